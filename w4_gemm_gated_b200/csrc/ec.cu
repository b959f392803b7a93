// Standalone Error-Compensator kernel of the unfused and semi-fused paths:
//     y <- bf16( y + g * ((x . A) . B) )     (in place)
// SPEAR runs the EC of the compute-bound prefill phase as a kernel of its own
// next to the low-bit GEMM (gist.science technical summary, section 2.2 A,
// "chemin semi-fusionne"); this is that kernel, run beside or after a GEMM
// whose own EC is disabled.
//
// Two launches, one kind of warp work item each:
//  phase 1, A items (m-block of 16 tokens, K part): partial [t | logit] =
//    x . [A | w_g] on the tensor cores (mma.sync), written to a partial
//    buffer; the last of the K parts (ticket) sums the parts in a fixed order,
//    applies the gate and writes gt = g * t (bf16), the gate outputs and the
//    mask count.  Nothing in it depends on y, so it can run concurrently with
//    the EC-disabled GEMM (the semi-fused DAG).
//  phase 2, B items (64 tokens, 32 output channels): gt . B' with MMA k-steps,
//    scaled by s_n (per-channel fold), read-modify-write of y.
// Stream order between the launches replaces any device-side wait: no item
// waits for another, and the CTAs need not be co-resident.
#include "common.cuh"
#include "kernels.h"

namespace spear {

constexpr int EC_WARPS = 8;
constexpr int EC_MAXE = 9;  // 16-row strips of [A^T ; w_g] for r <= 128

struct EcArgs {
  const __nv_bfloat16* x;
  __nv_bfloat16* y;
  const __nv_bfloat16* agt;
  const __nv_bfloat16* bpt;
  const __half* scales;
  float* part;       // [ksplit][Mpad][RT]
  int* tickets;      // [Mb16]
  __nv_bfloat16* gt; // [Mpad][r]
  float* gate_out;
  int* mask_count;
  WsHeader* hdr;
  int M, K, N, r, group;
  float b_g, tau;
  int ksplit, RT, Mb16, Mpad, E;
  int itemsA, itemsB;
  int phase;         // 1: A items (projection and gate), 2: B items (update of y)
  int gate_kind, gate_h;  // 0: scalar gate; 1: per-rank gamma(t) with bottleneck h
  const float *gw1, *gb1, *gw2, *gb2;
  float alpha;
};

__device__ __forceinline__ uint32_t w8(const uint4& a, const uint4& b, int i) {
  const uint4& v = i < 4 ? a : b;
  const int j = i & 3;
  return j == 0 ? v.x : j == 1 ? v.y : j == 2 ? v.z : v.w;
}

__device__ void ec_item_project(const EcArgs& a, int item, int lane) {
  const int mb = item / a.ksplit, ks = item % a.ksplit;
  const int KT = a.K / 64;
  const int kt0 = (int)((long long)ks * KT / a.ksplit), kt1 = (int)((long long)(ks + 1) * KT / a.ksplit);
  const int rho = lane >> 2, cq = lane & 3;
  float acc[EC_MAXE][2][4];
#pragma unroll
  for (int e = 0; e < EC_MAXE; ++e)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[e][nt][i] = 0.f;
  for (int kt = kt0; kt < kt1; ++kt) {
    const int col = kt * 64 + 16 * cq;
    uint4 xv[2][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int m = mb * 16 + nt * 8 + rho;
      if (m < a.M) {
        const uint4* p = reinterpret_cast<const uint4*>(a.x + (size_t)m * a.K + col);
        xv[nt][0] = __ldg(p);
        xv[nt][1] = __ldg(p + 1);
      } else {
        xv[nt][0] = xv[nt][1] = make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int e = 0; e < EC_MAXE; ++e) {
      if (e >= a.E) break;
      uint4 rv[2][2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int row = 16 * e + rho + 8 * h;
        if (row <= a.r) {
          const uint4* p = reinterpret_cast<const uint4*>(a.agt + (size_t)row * a.K + col);
          rv[h][0] = __ldg(p);
          rv[h][1] = __ldg(p + 1);
        } else {
          rv[h][0] = rv[h][1] = make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        uint32_t af[4] = {w8(rv[0][0], rv[0][1], 2 * s), w8(rv[1][0], rv[1][1], 2 * s),
                          w8(rv[0][0], rv[0][1], 2 * s + 1), w8(rv[1][0], rv[1][1], 2 * s + 1)};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
          mma_bf16_16816(acc[e][nt], af, w8(xv[nt][0], xv[nt][1], 2 * s), w8(xv[nt][0], xv[nt][1], 2 * s + 1));
      }
    }
  }
  // partial [t | logit] rows -> part[ks][m][row]
  float* P = a.part + (size_t)ks * a.Mpad * a.RT;
#pragma unroll
  for (int e = 0; e < EC_MAXE; ++e) {
    if (e >= a.E) break;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int row = 16 * e + rho;
      const int m = mb * 16 + nt * 8 + 2 * cq;
      P[(size_t)m * a.RT + row] = acc[e][nt][0];
      P[(size_t)(m + 1) * a.RT + row] = acc[e][nt][1];
      P[(size_t)m * a.RT + row + 8] = acc[e][nt][2];
      P[(size_t)(m + 1) * a.RT + row + 8] = acc[e][nt][3];
    }
  }
  __syncwarp();
  __threadfence();
  int prev = 0;
  if (lane == 0) prev = atomicAdd(&a.tickets[mb], 1);
  prev = __shfl_sync(0xffffffffu, prev, 0);
  if (prev != a.ksplit - 1) return;
  __threadfence();
  // last K part of this m-block: fixed-order sums, gate, gt
  const bool rank = a.gate_kind == 1;
  float gm = 0.f;
  if (!rank && lane < 16) {
    const int m = mb * 16 + lane;
    float l = 0.f;
    for (int k2 = 0; k2 < a.ksplit; ++k2) l += __ldcg(a.part + ((size_t)k2 * a.Mpad + m) * a.RT + a.r);
    gm = sigmoidf_(l + a.b_g);
  }
  // every lane owns (token, 4 columns) groups; K parts summed in order
  // 0..ksplit-1.  All parts of two groups are loaded before any sum, so a
  // lane has up to 16 independent 16-byte loads in flight.
  const int r4 = a.r / 4;
  const size_t stride = (size_t)a.Mpad * a.RT;
  for (int i0 = lane; i0 < 16 * r4; i0 += 64) {
    float4 v[2][8];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int idx = i0 + 32 * u;
      const int m = mb * 16 + idx / r4, j = 4 * (idx % r4);
      const float* src = a.part + (size_t)m * a.RT + j;
#pragma unroll
      for (int k2 = 0; k2 < 8; ++k2)
        if (idx < 16 * r4 && k2 < a.ksplit) v[u][k2] = __ldcg(reinterpret_cast<const float4*>(src + k2 * stride));
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int idx = i0 + 32 * u;
      // the gate of token mm lives in lane mm; every lane runs the shuffle
      const int mm = (idx < 16 * r4 ? idx : 0) / r4;
      const float g = __shfl_sync(0xffffffffu, gm, mm);
      if (idx >= 16 * r4) continue;
      const int m = mb * 16 + mm, j = 4 * (idx % r4);
      float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int k2 = 0; k2 < 8; ++k2)
        if (k2 < a.ksplit) {
          t.x += v[u][k2].x;
          t.y += v[u][k2].y;
          t.z += v[u][k2].z;
          t.w += v[u][k2].w;
        }
      if (rank) {
        // the rank gate needs whole rows of t: keep the sum in part 0's slot
        *reinterpret_cast<float4*>(a.part + (size_t)m * a.RT + j) = t;
      } else {
        uint2 o;
        o.x = pack_bf16x2(g * t.x, g * t.y);
        o.y = pack_bf16x2(g * t.z, g * t.w);
        *reinterpret_cast<uint2*>(a.gt + (size_t)m * a.r + j) = o;
      }
    }
  }
  if (rank) {
    // rank gate (summary section 2.1 A), one token per lane: u = relu(W1 t + b1),
    // gamma = sigmoid(W2 u + b2), gt = bf16(alpha gamma t); the gate is mean(gamma)
    __syncwarp();
    __threadfence_block();
    if (lane < 16) {
      const int m = mb * 16 + lane, h = a.gate_h;
      const float* trow = a.part + (size_t)m * a.RT;
      float u[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) u[i] = i < h ? __ldg(a.gb1 + i) : 0.f;
      for (int j = 0; j < a.r; j += 4) {
        const float4 tv = __ldcg(reinterpret_cast<const float4*>(trow + j));
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (i < h) {
            const float4 wv = __ldg(reinterpret_cast<const float4*>(a.gw1 + (size_t)i * a.r + j));
            u[i] = fmaf(wv.x, tv.x, u[i]);
            u[i] = fmaf(wv.y, tv.y, u[i]);
            u[i] = fmaf(wv.z, tv.z, u[i]);
            u[i] = fmaf(wv.w, tv.w, u[i]);
          }
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) u[i] = fmaxf(u[i], 0.f);
      float gsum = 0.f;
      for (int j = 0; j < a.r; j += 4) {
        const float4 tv = __ldcg(reinterpret_cast<const float4*>(trow + j));
        const float tt[4] = {tv.x, tv.y, tv.z, tv.w};
        float o[4];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          float z = __ldg(a.gb2 + j + jj);
          const float4* w = reinterpret_cast<const float4*>(a.gw2 + (size_t)(j + jj) * h);
#pragma unroll
          for (int i4 = 0; i4 < 8; ++i4)
            if (4 * i4 < h) {
              const float4 wv = __ldg(w + i4);
              z = fmaf(wv.x, u[4 * i4], z);
              z = fmaf(wv.y, u[4 * i4 + 1], z);
              z = fmaf(wv.z, u[4 * i4 + 2], z);
              z = fmaf(wv.w, u[4 * i4 + 3], z);
            }
          const float gam = sigmoidf_(z);
          gsum += gam;
          o[jj] = a.alpha * gam * tt[jj];
        }
        uint2 ov;
        ov.x = pack_bf16x2(o[0], o[1]);
        ov.y = pack_bf16x2(o[2], o[3]);
        *reinterpret_cast<uint2*>(a.gt + (size_t)m * a.r + j) = ov;
      }
      gm = gsum / (float)a.r;
    }
  }
  const bool valid = lane < 16 && mb * 16 + lane < a.M;
  if (a.gate_out && valid) a.gate_out[mb * 16 + lane] = gm;
  const unsigned below = __ballot_sync(0xffffffffu, valid && gm < a.tau);
  __syncwarp();
  if (lane == 0) {
    a.tickets[mb] = 0;
    if (a.mask_count) atomicAdd(&a.hdr->sf_count, __popc(below));
  }
}

template <int S>
__device__ __forceinline__ void ec_rowchunk(const __nv_bfloat16* base, int ld, int row, int jbase, int cq,
                                            uint32_t (&w)[8]) {
  const __nv_bfloat16* p = base + (size_t)row * ld + jbase + 4 * S * cq;
  if (S == 4) {
    const uint4 v0 = __ldcg(reinterpret_cast<const uint4*>(p)), v1 = __ldcg(reinterpret_cast<const uint4*>(p) + 1);
    w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w; w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
  } else if (S == 2) {
    const uint4 v0 = __ldcg(reinterpret_cast<const uint4*>(p));
    w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
  } else {
    const uint2 v0 = __ldcg(reinterpret_cast<const uint2*>(p));
    w[0] = v0.x; w[1] = v0.y;
  }
}

template <int S>
__device__ __forceinline__ void ec_up_chunk(const EcArgs& a, int m0, int pair, int lane, int jbase,
                                            float (&acc)[2][8][4]) {
  const int rho = lane >> 2, cq = lane & 3;
  uint32_t b[2][2][8];
#pragma unroll
  for (int si = 0; si < 2; ++si) {
    const int n0 = 16 * (2 * pair + si) + rho;
    ec_rowchunk<S>(a.bpt, a.r, n0, jbase, cq, b[si][0]);
    ec_rowchunk<S>(a.bpt, a.r, n0 + 8, jbase, cq, b[si][1]);
  }
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    uint32_t g[8];
    ec_rowchunk<S>(a.gt, a.r, m0 + nt * 8 + rho, jbase, cq, g);
#pragma unroll
    for (int si = 0; si < 2; ++si)
#pragma unroll
      for (int s = 0; s < S; ++s) {
        uint32_t af[4] = {b[si][0][2 * s], b[si][1][2 * s], b[si][0][2 * s + 1], b[si][1][2 * s + 1]};
        mma_bf16_16816(acc[si][nt], af, g[2 * s], g[2 * s + 1]);
      }
  }
}

__device__ void ec_item_update(const EcArgs& a, int item, int lane, __nv_bfloat16* stage) {
  const int P2 = a.N / 32;
  const int mb64 = item / P2, pair = item % P2;
  const int m0 = mb64 * 64;
  const int rho = lane >> 2, cq = lane & 3;
  float acc[2][8][4];
#pragma unroll
  for (int si = 0; si < 2; ++si)
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[si][nt][i] = 0.f;
  {
    if (a.r >= 64) {
      for (int jb = 0; jb < a.r; jb += 64) ec_up_chunk<4>(a, m0, pair, lane, jb, acc);
    } else if (a.r == 32) {
      ec_up_chunk<2>(a, m0, pair, lane, 0, acc);
    } else {
      ec_up_chunk<1>(a, m0, pair, lane, 0, acc);
    }
  }
  // y tile (64 tokens x 32 channels) -> stage, add, store
  for (int idx = lane; idx < 64 * 4; idx += 32) {
    const int m = idx >> 2, part = idx & 3;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (m0 + m < a.M) v = *reinterpret_cast<const uint4*>(a.y + (size_t)(m0 + m) * a.N + 32 * pair + part * 8);
    *reinterpret_cast<uint4*>(stage + m * 32 + part * 8) = v;
  }
  __syncwarp();
#pragma unroll
  for (int si = 0; si < 2; ++si) {
    const int n0 = 16 * (2 * pair + si) + rho;
    float s0 = 1.f, s1 = 1.f;
    if (a.group == 0) {
      s0 = __half2float(a.scales[n0]);
      s1 = __half2float(a.scales[n0 + 8]);
    }
    const int c0 = 16 * si + rho;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const int m = nt * 8 + 2 * cq;
      __nv_bfloat16* p00 = stage + m * 32 + c0;
      __nv_bfloat16* p10 = stage + (m + 1) * 32 + c0;
      *p00 = __float2bfloat16_rn(__bfloat162float(*p00) + s0 * acc[si][nt][0]);
      *p10 = __float2bfloat16_rn(__bfloat162float(*p10) + s0 * acc[si][nt][1]);
      *(p00 + 8) = __float2bfloat16_rn(__bfloat162float(*(p00 + 8)) + s1 * acc[si][nt][2]);
      *(p10 + 8) = __float2bfloat16_rn(__bfloat162float(*(p10 + 8)) + s1 * acc[si][nt][3]);
    }
  }
  __syncwarp();
  for (int idx = lane; idx < 64 * 4; idx += 32) {
    const int m = idx >> 2, part = idx & 3;
    if (m0 + m < a.M && SPEAR_DCHECK(32 * pair + 32 <= a.N, a.hdr))
      *reinterpret_cast<uint4*>(a.y + (size_t)(m0 + m) * a.N + 32 * pair + part * 8) =
          *reinterpret_cast<const uint4*>(stage + m * 32 + part * 8);
  }
  __syncwarp();
}

// Phase 1 and phase 2 are separate kernels, so the update keeps its own
// (smaller) register allocation.
__global__ void __launch_bounds__(EC_WARPS * 32) ec_project_kernel(const __grid_constant__ EcArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gw = blockIdx.x * EC_WARPS + warp, nw = gridDim.x * EC_WARPS;
  for (int it = gw; it < a.itemsA; it += nw) ec_item_project(a, it, lane);
  // the last CTA publishes the mask count of this launch
  __syncthreads();
  if (threadIdx.x == 0 && a.mask_count) {
    __threadfence();
    const int prev = atomicAdd(&a.hdr->sf_done, 1);
    if (prev == (int)gridDim.x - 1) {
      __threadfence();
      *a.mask_count = *reinterpret_cast<volatile int*>(&a.hdr->sf_count);
      a.hdr->sf_done = 0;
      a.hdr->sf_count = 0;
    }
  }
}

__global__ void __launch_bounds__(EC_WARPS * 32) ec_update_kernel(const __grid_constant__ EcArgs a) {
  __shared__ __align__(16) __nv_bfloat16 stage_all[EC_WARPS][64 * 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gw = blockIdx.x * EC_WARPS + warp, nw = gridDim.x * EC_WARPS;
  for (int it = gw; it < a.itemsB; it += nw) ec_item_update(a, it, lane, stage_all[warp]);
}

EcPlan plan_ec(int M, int K, int N, int r, int sm_count) {
  EcPlan p = {};
  const int Mb16 = (M + 15) / 16;
  const int KT = K / 64;
  const int warps = sm_count * 2 * EC_WARPS;
  int ks = (warps + Mb16 - 1) / Mb16;
  if (ks > KT) ks = KT;
  if (ks > 8) ks = 8;  // the last part of an m-block sums ksplit partials
  if (ks < 1) ks = 1;
  p.ksplit = ks;
  p.grid = sm_count * 2;
  p.RT = 16 * ((r + 16) / 16);
  const int Mpad = ((M + 63) / 64) * 64;
  p.part_floats = (size_t)ks * Mpad * p.RT;
  return p;
}

int launch_ec(const EcPlan& p, const LayerView& L, const __nv_bfloat16* x, int M, __nv_bfloat16* y, WsHeader* hdr,
              float* part, int* tickets, __nv_bfloat16* gt, float* gate_out, int* mask_count, cudaStream_t st,
              int phase) {
  if (phase != 1 && phase != 2) return set_error(SPEAR_ERR_INVALID_ARG, "EC launch phase must be 1 or 2");
  EcArgs a = {};
  a.x = x;
  a.y = y;
  a.agt = L.agt;
  a.bpt = L.bpt;
  a.scales = L.scales;
  a.part = part;
  a.tickets = tickets;
  a.gt = gt;
  a.gate_out = gate_out;
  a.mask_count = mask_count;
  a.hdr = hdr;
  a.M = M;
  a.K = L.K;
  a.N = L.N;
  a.r = L.r;
  a.group = L.group;
  a.b_g = L.b_g;
  a.tau = L.tau;
  a.ksplit = p.ksplit;
  a.RT = p.RT;
  a.Mb16 = (M + 15) / 16;
  a.Mpad = ((M + 63) / 64) * 64;
  a.E = (L.r + 16) / 16;
  a.itemsA = a.Mb16 * p.ksplit;
  a.itemsB = (a.Mpad / 64) * (L.N / 32);
  a.phase = phase;
  a.gate_kind = L.gate_kind;
  a.gate_h = L.gate_h;
  a.gw1 = L.gw1;
  a.gb1 = L.gb1;
  a.gw2 = L.gw2;
  a.gb2 = L.gb2;
  a.alpha = L.alpha;
  // no more CTAs than the items of this phase need
  const int items = phase == 1 ? a.itemsA : a.itemsB;
  const int need = (items + EC_WARPS - 1) / EC_WARPS;
  const int grid = need < p.grid ? need : p.grid;
  if (phase == 1)
    ec_project_kernel<<<grid, EC_WARPS * 32, 0, st>>>(a);
  else
    ec_update_kernel<<<grid, EC_WARPS * 32, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SPEAR_OK : set_cuda_error("ec kernel launch", e);
}

}  // namespace spear
