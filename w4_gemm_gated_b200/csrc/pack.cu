// One-off per-layer preparation kernels: RTN int4 quantiser, packing into the
// tiled nibble layout, unpacking, and the EC operand layouts.
//
// All of these are integer or exactly specified floating-point transforms and
// are bit-exact (see include/spear.h for each definition).
#include "common.cuh"
#include "kernels.h"

namespace spear {

// ---------------------------------------------------------------------------
// a-0 quantiser: one CTA per 32 output channels; 32 x 8 threads.
// Pass 1: max|w| per (block of k, channel); pass 2: codes, written through a
// shared-memory transpose so that q[n][k] rows are stored contiguously.
// ---------------------------------------------------------------------------
__device__ __forceinline__ __half rtn_scale(float m) {
  __half s = __float2half_rn(m / 7.0f);  // IEEE fp32 quotient, then fp16 RNE
  if (__hisinf(s)) s = __float2half_rn(65504.0f);
  return s;
}

__global__ void quantize_kernel(const float* __restrict__ W, int K, int N, int group, int8_t* __restrict__ q,
                                __half* __restrict__ s) {
  __shared__ float red[8][33];
  __shared__ int8_t tile[32][33];
  __shared__ float sc[32];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
  const int n0 = blockIdx.x * 32;
  const int n = n0 + tx;
  const int blk = group == 0 ? K : group;
  for (int kb = 0; kb < K; kb += blk) {
    float m = 0.f;
    for (int k = kb + ty; k < kb + blk; k += 8) m = fmaxf(m, fabsf(W[(size_t)k * N + n]));
    red[ty][tx] = m;
    __syncthreads();
    if (ty == 0) {
      float mm = red[0][tx];
      for (int i = 1; i < 8; ++i) mm = fmaxf(mm, red[i][tx]);
      __half hs = rtn_scale(mm);
      float sf = __half2float(hs);
      if (sf == 0.f) {
        hs = __float2half_rn(1.0f);
        sf = 0.f;  // marks "all codes zero"
      }
      sc[tx] = sf;
      const size_t si = group == 0 ? (size_t)n : (size_t)(kb / group) * N + n;
      s[si] = hs;
    }
    __syncthreads();
    for (int k0 = kb; k0 < kb + blk; k0 += 32) {
      // tile[k - k0][channel] then store q[channel][k0 .. k0+32)
      for (int kk = ty; kk < 32; kk += 8) {
        const float w = W[(size_t)(k0 + kk) * N + n];
        const float sf = sc[tx];
        int code = 0;
        if (sf != 0.f) {
          float v = rintf(w / sf);
          v = fminf(fmaxf(v, -7.f), 7.f);
          code = (int)v;
        }
        tile[kk][tx] = (int8_t)code;
      }
      __syncthreads();
      for (int nn = ty; nn < 32; nn += 8) q[(size_t)(n0 + nn) * K + k0 + tx] = tile[tx][nn];
      __syncthreads();
    }
  }
}

int launch_quantize(const float* W, int K, int N, int group, int8_t* q, __half* s, cudaStream_t st) {
  quantize_kernel<<<N / 32, 256, 0, st>>>(W, K, N, group, q, s);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SPEAR_OK : set_cuda_error("quantize launch", e);
}

// ---------------------------------------------------------------------------
// a-1 pack / unpack: one thread per 32-bit word of the packed layout.
// Word (tile (p, t), lane L, word s), slot i (bits 4i..4i+3) holds
//   n = 16p + rho + 8*(i & 1),  k = 64t + 16c + 4s + 2*((i & 3) >> 1) + (i >> 2),
// rho = L / 4, c = L % 4, value q + 8.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void word_coords(size_t wi, int K, int& nb, int& kb) {
  const int s = (int)(wi & 3);
  const int L = (int)((wi >> 2) & 31);
  const size_t tile = wi >> 7;
  const int KT = K / 64;
  const int p = (int)(tile / KT), t = (int)(tile % KT);
  nb = 16 * p + (L >> 2);
  kb = 64 * t + 16 * (L & 3) + 4 * s;
}

__global__ void pack_kernel(const int8_t* __restrict__ q, int N, int K, uint32_t* __restrict__ out) {
  const size_t nwords = (size_t)N * K / 8;
  for (size_t wi = (size_t)blockIdx.x * blockDim.x + threadIdx.x; wi < nwords; wi += (size_t)gridDim.x * blockDim.x) {
    int nb, kb;
    word_coords(wi, K, nb, kb);
    uint32_t word = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int n = nb + 8 * (i & 1);
      const int k = kb + 2 * ((i & 3) >> 1) + (i >> 2);
      const uint32_t u = (uint32_t)((int)q[(size_t)n * K + k] + 8) & 0xFu;
      word |= u << (4 * i);
    }
    out[wi] = word;
  }
}

__global__ void unpack_kernel(const uint32_t* __restrict__ in, int N, int K, int8_t* __restrict__ q) {
  const size_t nwords = (size_t)N * K / 8;
  for (size_t wi = (size_t)blockIdx.x * blockDim.x + threadIdx.x; wi < nwords; wi += (size_t)gridDim.x * blockDim.x) {
    int nb, kb;
    word_coords(wi, K, nb, kb);
    const uint32_t word = in[wi];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int n = nb + 8 * (i & 1);
      const int k = kb + 2 * ((i & 3) >> 1) + (i >> 2);
      q[(size_t)n * K + k] = (int8_t)((int)((word >> (4 * i)) & 0xFu) - 8);
    }
  }
}

static int grid_for(size_t work, int block) {
  size_t g = (work + block - 1) / block;
  if (g > 65535u * 8u) g = 65535u * 8u;
  return (int)(g ? g : 1);
}

int launch_pack(const int8_t* q, int N, int K, uint8_t* packed, cudaStream_t st) {
  const size_t nw = (size_t)N * K / 8;
  pack_kernel<<<grid_for(nw, 256), 256, 0, st>>>(q, N, K, reinterpret_cast<uint32_t*>(packed));
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SPEAR_OK : set_cuda_error("pack launch", e);
}

int launch_unpack(const uint8_t* packed, int N, int K, int8_t* q, cudaStream_t st) {
  const size_t nw = (size_t)N * K / 8;
  unpack_kernel<<<grid_for(nw, 256), 256, 0, st>>>(reinterpret_cast<const uint32_t*>(packed), N, K, q);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SPEAR_OK : set_cuda_error("unpack launch", e);
}

// ---------------------------------------------------------------------------
// EC operands
// ---------------------------------------------------------------------------
// B'[j][n] = bf16_rne(fp32(B[j][n] / s[n])); out is r x N, or N x r if transpose.
__global__ void prescale_kernel(const __nv_bfloat16* __restrict__ B, const __half* __restrict__ s, int r, int N,
                                __nv_bfloat16* __restrict__ out, bool transpose) {
  const size_t total = (size_t)r * N;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const int j = (int)(i / N), n = (int)(i % N);
    const float v = __bfloat162float(B[i]) / __half2float(s[n]);
    const __nv_bfloat16 o = __float2bfloat16_rn(v);
    if (transpose)
      out[(size_t)n * r + j] = o;
    else
      out[i] = o;
  }
}

int launch_prescale(const __nv_bfloat16* B, const __half* s, int r, int N, __nv_bfloat16* Bp, bool transpose,
                    cudaStream_t st) {
  prescale_kernel<<<grid_for((size_t)r * N, 256), 256, 0, st>>>(B, s, r, N, Bp, transpose);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SPEAR_OK : set_cuda_error("prescale launch", e);
}

// AgT[j][k] = A[k][j] (j < r), AgT[r][k] = w_g[k]
__global__ void agt_kernel(const __nv_bfloat16* __restrict__ A, const __nv_bfloat16* __restrict__ wg, int K, int r,
                           __nv_bfloat16* __restrict__ out) {
  const size_t total = (size_t)(r + 1) * K;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const int j = (int)(i / K), k = (int)(i % K);
    out[i] = j < r ? A[(size_t)k * r + j] : wg[k];
  }
}

int launch_agt(const __nv_bfloat16* A, const __nv_bfloat16* w_g, int K, int r, __nv_bfloat16* AgT, cudaStream_t st) {
  agt_kernel<<<grid_for((size_t)(r + 1) * K, 256), 256, 0, st>>>(A, w_g, K, r, AgT);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SPEAR_OK : set_cuda_error("ec pack (A) launch", e);
}

__global__ void transpose_b_kernel(const __nv_bfloat16* __restrict__ B, int r, int N, __nv_bfloat16* __restrict__ BT) {
  const size_t total = (size_t)r * N;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const int j = (int)(i / N), n = (int)(i % N);
    BT[(size_t)n * r + j] = B[i];
  }
}

int launch_transpose_b(const __nv_bfloat16* B, int r, int N, __nv_bfloat16* BT, cudaStream_t st) {
  transpose_b_kernel<<<grid_for((size_t)r * N, 256), 256, 0, st>>>(B, r, N, BT);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SPEAR_OK : set_cuda_error("ec pack (B) launch", e);
}

}  // namespace spear
