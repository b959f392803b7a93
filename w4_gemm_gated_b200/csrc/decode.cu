// Decode path (M <= 16): split-K GEMV-style kernel with the gated EC fused.
//
// SPEAR fuses the whole EC computation into the low-bit GEMM for the
// memory-bound decode phase (gist.science technical summary, section 2.2 A,
// "Phase de decodage ... M=1": one kernel, no inter-kernel launch on the
// critical path).  This kernel does that for 1 <= M <= 16 on sm_100a:
//
//  * Work is cut into 32-row strip pairs of the output (two 16-channel strips
//    of the packed layout) plus "EC pairs" (32 rows of [A^T ; w_g]).  A
//    thread-block cluster of CS CTAs owns a contiguous set of pairs and splits
//    K into CS parts, one per CTA; each CTA keeps its part of x in shared
//    memory.
//  * Inside a CTA the pair x k-tile units are split evenly over 16 warps.
//    Each warp streams its packed weights with 128-bit loads straight into
//    registers (double-buffered: the next unit's loads are in flight while
//    the current one is converted and multiplied), converts int4 -> bf16 in
//    registers and multiplies on the tensor cores (mma.sync m16n8k16, the
//    weights as the 16-row operand, tokens as the 8-wide operand).
//  * Partial sums go to per-warp slots in shared memory; an arrival counter
//    per pair (atomics on distributed shared memory) elects the last
//    contributor, which adds all slots of the cluster in a fixed order
//    (deterministic) through DSMEM.
//  * The EC rows (t = x.A and the gate logit x.w_g) are ordinary pairs that
//    are scheduled first.  Once all are reduced, one warp computes
//    g = sigmoid(logit + b_g) and gt = g * t, publishes them and raises an
//    epoch-tagged flag.  Weight pairs add gt . B' as r/16 extra MMA k-steps
//    (B' = B / s_n folded once per layer), apply s_n and store bf16 y with
//    16-byte stores.  A pair reduced before the flag is up is parked in its
//    slot and finished after the warp's last unit (bounded wait).
#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>

#include "common.cuh"
#include "kernels.h"

namespace spear {

constexpr int DEC_NW = 16;        // warps per CTA
constexpr int DEC_UK = 4;         // k-tiles (64 k each) per weight unit
constexpr int DEC_MAXSEG = 2;     // pairs one warp may touch
constexpr int DEC_MAXPAIRS = 64;  // pairs per cluster

struct DecodeArgs {
  const uint8_t* w;
  const __half* scales;
  const __nv_bfloat16* agt;
  const __nv_bfloat16* bpt;
  const __nv_bfloat16* x;
  __nv_bfloat16* y;
  float* gate_out;
  int* mask_count;
  WsHeader* hdr;
  float* ws_t;             // [MT][RT] fp32, RT = 32 * E2
  __nv_bfloat16* ws_gt;    // [MT][r] bf16
  int M, K, N, r, group;
  float b_g, tau;
  int CS, NC;              // cluster size (= K parts), clusters
  int kt_part;             // k-tiles per K part
  int E2, P2;              // EC pairs (0: EC off), weight pairs (N / 32)
  int ec_only;             // 1: skip the weights, y += EC term in place (unfused path)
};

struct DecodeShape {
  int E2, P2, NC, kt_part;
};

struct DecodeLayout {
  int ec_lo, n_ec, w_lo, n_w, upw, U;
  __host__ __device__ __forceinline__ int lp_of(int u, int kt_part) const {
    int ecu = n_ec * kt_part;
    return u < ecu ? u / kt_part : n_ec + (u - ecu) / upw;
  }
  __host__ __device__ __forceinline__ int first_unit(int lp, int kt_part) const {
    return lp < n_ec ? lp * kt_part : n_ec * kt_part + (lp - n_ec) * upw;
  }
  __host__ __device__ __forceinline__ int n_units(int lp, int kt_part) const { return lp < n_ec ? kt_part : upw; }
  __host__ __device__ __forceinline__ int warp_first(int w) const { return (int)(((long long)w * U) / DEC_NW); }
  __host__ __device__ __forceinline__ int warp_of(int u) const {
    return (int)((((long long)u + 1) * DEC_NW - 1) / U);
  }
  __host__ __device__ __forceinline__ bool warp_busy(int w) const { return warp_first(w) < warp_first(w + 1); }
  // warps (per CTA) that hold units of pair lp
  __host__ __device__ __forceinline__ int contributors(int lp, int kt_part) const {
    const int fu = first_unit(lp, kt_part);
    const int wlo = warp_of(fu), whi = warp_of(fu + n_units(lp, kt_part) - 1);
    int n = 0;
    for (int w = wlo; w <= whi; ++w) n += warp_busy(w) ? 1 : 0;
    return n;
  }
};

__host__ __device__ __forceinline__ int ceil_div_ll(long long n, long long d) { return (int)((n + d - 1) / d); }
__host__ __device__ __forceinline__ int clamp_ll(long long v, int hi) { return (int)(v < 0 ? 0 : (v > hi ? hi : v)); }

// Pairs of cluster cl: its EC pairs (at most one per cluster when E2 <= NC,
// spread evenly) followed by a contiguous range of weight pairs, chosen so
// that every cluster streams about the same number of bytes (an EC pair is
// DEC_UK times the bytes of a weight pair: bf16 instead of int4).
__host__ __device__ __forceinline__ DecodeLayout decode_layout(const DecodeShape& a, int cl) {
  DecodeLayout L;
  const int UK = DEC_UK;
  const int ec_lo = ceil_div_ll((long long)cl * a.E2, a.NC);
  const int ec_hi = ceil_div_ll((long long)(cl + 1) * a.E2, a.NC);
  const long long C = (long long)a.E2 * UK + a.P2;
  const long long s0 = (C * cl) / a.NC, s1 = (C * (cl + 1)) / a.NC;
  const int w0 = clamp_ll(s0 - (long long)UK * ec_lo, a.P2);
  int w1 = clamp_ll(s1 - (long long)UK * ec_hi, a.P2);
  if (cl == a.NC - 1) w1 = a.P2;
  L.ec_lo = ec_lo;
  L.n_ec = ec_hi - ec_lo;
  L.w_lo = w0;
  L.n_w = w1 > w0 ? w1 - w0 : 0;
  L.upw = (a.kt_part + UK - 1) / UK;
  L.U = L.n_ec * a.kt_part + L.n_w * L.upw;
  return L;
}

// Loads of one unit into 8 x 16 bytes per lane.
//   weight unit: 2 strips x up to 4 k-tiles, one 512-byte tile per 128-bit warp load;
//   EC unit:     2 EC strips x 1 k-tile, 2 rows x 32 bytes of [A^T ; w_g] per lane.
template <int MT>
__device__ __forceinline__ void decode_load_unit(const DecodeArgs& a, const DecodeLayout& L, int u, int q,
                                                 int lane, uint4 (&buf)[8]) {
  const int kt_part = a.kt_part;
  const int ecu = L.n_ec * kt_part;
  const int KT = a.K / 64;
  if (u < ecu) {
    const int e = L.ec_lo + u / kt_part;
    const int kt = q * kt_part + u % kt_part;
    const int rho = lane >> 2, cq = lane & 3;
    const int col = kt * 64 + 16 * cq;
#pragma unroll
    for (int si = 0; si < 2; ++si) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int row = 16 * (2 * e + si) + rho + 8 * h;
        if (row <= a.r) {
          const __nv_bfloat16* p = a.agt + (size_t)row * a.K + col;
          buf[si * 4 + h * 2 + 0] = ldg_stream(p);
          buf[si * 4 + h * 2 + 1] = ldg_stream(p + 8);
        } else {
          buf[si * 4 + h * 2 + 0] = make_uint4(0, 0, 0, 0);
          buf[si * 4 + h * 2 + 1] = make_uint4(0, 0, 0, 0);
        }
      }
    }
  } else if (!a.ec_only) {
    const int v = u - ecu;
    const int pair = L.w_lo + v / L.upw;
    const int kt0 = q * kt_part + (v % L.upw) * DEC_UK;
    const int kt_end = (q + 1) * kt_part;
#pragma unroll
    for (int si = 0; si < 2; ++si) {
      const uint8_t* base = a.w + ((size_t)(2 * pair + si) * KT) * 512 + lane * 16;
#pragma unroll
      for (int j = 0; j < DEC_UK; ++j) {
        const int kt = kt0 + j;
        buf[si * 4 + j] = kt < kt_end ? ldg_stream(base + (size_t)kt * 512) : make_uint4(0, 0, 0, 0);
      }
    }
  }
}

__device__ __forceinline__ uint32_t u4w(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// x fragments of one k-tile for n8-tile nt: 8 words = x[nt*8 + rho][kt*64 + 16c .. +16)
template <int MT>
__device__ __forceinline__ void load_x_frag(const __nv_bfloat16* xs, int xs_stride, int kt_local, int lane,
                                            uint32_t (&xf)[MT / 8][8]) {
  const int rho = lane >> 2, cq = lane & 3;
#pragma unroll
  for (int nt = 0; nt < MT / 8; ++nt) {
    const uint4* p = reinterpret_cast<const uint4*>(xs + (size_t)(nt * 8 + rho) * xs_stride + kt_local * 64 + 16 * cq);
    uint4 v0 = p[0], v1 = p[1];
    xf[nt][0] = v0.x; xf[nt][1] = v0.y; xf[nt][2] = v0.z; xf[nt][3] = v0.w;
    xf[nt][4] = v1.x; xf[nt][5] = v1.y; xf[nt][6] = v1.z; xf[nt][7] = v1.w;
  }
}

template <int MT, bool GROUP>
__device__ __forceinline__ void decode_compute_unit(const DecodeArgs& a, const DecodeLayout& L, int u, int q,
                                                    int lane, const uint4 (&buf)[8], const __nv_bfloat16* xs,
                                                    int xs_stride, float (&acc)[2][MT / 8][4]) {
  constexpr int NT = MT / 8;
  const int kt_part = a.kt_part;
  const int ecu = L.n_ec * kt_part;
  uint32_t xf[NT][8];
  if (u < ecu) {
    const int kt_local = u % kt_part;
    load_x_frag<MT>(xs, xs_stride, kt_local, lane, xf);
#pragma unroll
    for (int si = 0; si < 2; ++si) {
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        uint32_t af[4];
        // rows rho (h = 0) and rho + 8 (h = 1); words 2s (k + 0, 1) and 2s + 1 (k + 2, 3)
        af[0] = u4w(buf[si * 4 + 0 + (2 * s) / 4], (2 * s) % 4);
        af[1] = u4w(buf[si * 4 + 2 + (2 * s) / 4], (2 * s) % 4);
        af[2] = u4w(buf[si * 4 + 0 + (2 * s + 1) / 4], (2 * s + 1) % 4);
        af[3] = u4w(buf[si * 4 + 2 + (2 * s + 1) / 4], (2 * s + 1) % 4);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(acc[si][nt], af, xf[nt][2 * s], xf[nt][2 * s + 1]);
      }
    }
    return;
  }
  if (a.ec_only) return;
  const int v = u - ecu;
  const int pair = L.w_lo + v / L.upw;
  const int kt0_local = (v % L.upw) * DEC_UK;
  const int rho = lane >> 2;
#pragma unroll
  for (int j = 0; j < DEC_UK; ++j) {
    const int kt_local = kt0_local + j;
    if (kt_local >= kt_part) break;
    load_x_frag<MT>(xs, xs_stride, kt_local, lane, xf);
    float sc[2][2];
    float part[2][NT][4];
    if (GROUP) {
      const int g = (q * kt_part + kt_local) / 2;  // 128-k group of this 64-k tile
#pragma unroll
      for (int si = 0; si < 2; ++si) {
        const int n0 = 16 * (2 * pair + si) + rho;
        sc[si][0] = __half2float(a.scales[(size_t)g * a.N + n0]);
        sc[si][1] = __half2float(a.scales[(size_t)g * a.N + n0 + 8]);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int i = 0; i < 4; ++i) part[si][nt][i] = 0.f;
      }
    }
#pragma unroll
    for (int si = 0; si < 2; ++si) {
      const uint4 wv = buf[si * 4 + j];
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        uint32_t af[4];
        int4x8_to_bf16x8(u4w(wv, s), af);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          if (GROUP)
            mma_bf16_16816(part[si][nt], af, xf[nt][2 * s], xf[nt][2 * s + 1]);
          else
            mma_bf16_16816(acc[si][nt], af, xf[nt][2 * s], xf[nt][2 * s + 1]);
        }
      }
    }
    if (GROUP) {
#pragma unroll
      for (int si = 0; si < 2; ++si)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          acc[si][nt][0] = fmaf(sc[si][0], part[si][nt][0], acc[si][nt][0]);
          acc[si][nt][1] = fmaf(sc[si][0], part[si][nt][1], acc[si][nt][1]);
          acc[si][nt][2] = fmaf(sc[si][1], part[si][nt][2], acc[si][nt][2]);
          acc[si][nt][3] = fmaf(sc[si][1], part[si][nt][3], acc[si][nt][3]);
        }
    }
  }
}

// 8*S bytes of row `row` of a row-major [.. x r] bf16 matrix at columns
// jbase + 4*S*cq, as words w[0 .. 2S).
template <int S>
__device__ __forceinline__ void load_rowchunk(const __nv_bfloat16* base, int r, int row, int jbase, int cq,
                                              uint32_t (&w)[8]) {
  const __nv_bfloat16* p = base + (size_t)row * r + jbase + 4 * S * cq;
  if (S == 4) {
    uint4 v0 = __ldcg(reinterpret_cast<const uint4*>(p));
    uint4 v1 = __ldcg(reinterpret_cast<const uint4*>(p) + 1);
    w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w; w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
  } else if (S == 2) {
    uint4 v0 = __ldcg(reinterpret_cast<const uint4*>(p));
    w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
  } else {
    uint2 v0 = __ldcg(reinterpret_cast<const uint2*>(p));
    w[0] = v0.x; w[1] = v0.y;
  }
}

template <int MT, int S>
__device__ __forceinline__ void ec_upproject_chunk(const DecodeArgs& a, int pair, int lane, int jbase,
                                                   float (&acc)[2][MT / 8][4]) {
  const int rho = lane >> 2, cq = lane & 3;
  uint32_t g[MT / 8][8];
#pragma unroll
  for (int nt = 0; nt < MT / 8; ++nt) load_rowchunk<S>(a.ws_gt, a.r, nt * 8 + rho, jbase, cq, g[nt]);
#pragma unroll
  for (int si = 0; si < 2; ++si) {
    const int n0 = 16 * (2 * pair + si) + rho;
    uint32_t b0[8], b1[8];
    load_rowchunk<S>(a.bpt, a.r, n0, jbase, cq, b0);
    load_rowchunk<S>(a.bpt, a.r, n0 + 8, jbase, cq, b1);
#pragma unroll
    for (int s = 0; s < S; ++s) {
      uint32_t af[4] = {b0[2 * s], b1[2 * s], b0[2 * s + 1], b1[2 * s + 1]};
#pragma unroll
      for (int nt = 0; nt < MT / 8; ++nt) mma_bf16_16816(acc[si][nt], af, g[nt][2 * s], g[nt][2 * s + 1]);
    }
  }
}

// Final epilogue of a weight pair: + gt . B', scale, bf16, 16-byte stores.
template <int MT, bool GROUP>
__device__ void decode_store_pair(const DecodeArgs& a, int pair, int lane, bool ec_ok, __nv_bfloat16* stage,
                                  float (&acc)[2][MT / 8][4]) {
  constexpr int NT = MT / 8;
  const int rho = lane >> 2, cq = lane & 3;
  if (a.E2 > 0 && ec_ok) {
    if (a.r >= 64) {
      for (int jb = 0; jb < a.r; jb += 64) ec_upproject_chunk<MT, 4>(a, pair, lane, jb, acc);
    } else if (a.r == 32) {
      ec_upproject_chunk<MT, 2>(a, pair, lane, 0, acc);
    } else {
      ec_upproject_chunk<MT, 1>(a, pair, lane, 0, acc);
    }
  }
#pragma unroll
  for (int si = 0; si < 2; ++si) {
    const int n0 = 16 * (2 * pair + si) + rho;
    float s0 = 1.f, s1 = 1.f;
    if (!GROUP) {
      s0 = __half2float(a.scales[n0]);
      s1 = __half2float(a.scales[n0 + 8]);
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int m0 = nt * 8 + 2 * cq;
      const int c0 = 16 * si + rho;
      stage[(m0 + 0) * 32 + c0] = __float2bfloat16_rn(s0 * acc[si][nt][0]);
      stage[(m0 + 1) * 32 + c0] = __float2bfloat16_rn(s0 * acc[si][nt][1]);
      stage[(m0 + 0) * 32 + c0 + 8] = __float2bfloat16_rn(s1 * acc[si][nt][2]);
      stage[(m0 + 1) * 32 + c0 + 8] = __float2bfloat16_rn(s1 * acc[si][nt][3]);
    }
  }
  __syncwarp();
  for (int idx = lane; idx < MT * 4; idx += 32) {
    const int m = idx >> 2, part = idx & 3;
    if (m < a.M) {
      uint4 v = *reinterpret_cast<const uint4*>(stage + m * 32 + part * 8);
      uint4* dst = reinterpret_cast<uint4*>(a.y + (size_t)m * a.N + 32 * pair + part * 8);
      if (a.ec_only) {
        // y already holds the EC-disabled GEMM result: add the EC term in fp32, round once
        const uint4 old = *dst;
        const uint32_t* o = reinterpret_cast<const uint32_t*>(&old);
        uint32_t* nv = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 a2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(o + i));
          const float2 b2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(nv + i));
          nv[i] = pack_bf16x2(a2.x + b2.x, a2.y + b2.y);
        }
      }
      *dst = v;
    }
  }
  __syncwarp();
}

// The warp that finalises the last EC pair: gate, gt = g * t, gate outputs, flag.
template <int MT>
__device__ void decode_finish_gate(const DecodeArgs& a, int lane, int epoch) {
  const int RT = 32 * a.E2;
  float gm = 0.f;
  if (lane < MT) {
    const float l = __ldcg(a.ws_t + (size_t)lane * RT + a.r);
    gm = sigmoidf_(l + a.b_g);
  }
  const bool valid = lane < a.M;
  if (a.gate_out && valid) a.gate_out[lane] = gm;
  const unsigned below = __ballot_sync(0xffffffffu, valid && gm < a.tau);
  if (a.mask_count && lane == 0) *a.mask_count = __popc(below);
  // gt[m][j] = bf16(g_m * t[m][j]); every lane handles whole tokens so the
  // gate value comes from a shuffle with a warp-uniform source lane.
  for (int m = 0; m < MT; ++m) {
    const float g = __shfl_sync(0xffffffffu, gm, m);
    for (int j = lane; j < a.r; j += 32) {
      const float t = __ldcg(a.ws_t + (size_t)m * RT + j);
      a.ws_gt[(size_t)m * a.r + j] = __float2bfloat16_rn(g * t);
    }
  }
  __syncwarp();
  __threadfence();
  if (lane == 0) st_release_gpu(&a.hdr->ec_flag, epoch + 1);
}

template <int MT, bool GROUP>
__global__ void __launch_bounds__(DEC_NW * 32, 1) decode_kernel(const __grid_constant__ DecodeArgs a) {
  constexpr int NT = MT / 8;
  constexpr int NF4 = 2 * NT;  // float4 fragments per lane per slot
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = (int)cluster_rank();
  const int cl = blockIdx.x / a.CS;
  const int xs_stride = a.kt_part * 64 + 8;
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(smem);
  float4* slots = reinterpret_cast<float4*>(smem + (size_t)MT * xs_stride * 2);
  __nv_bfloat16* stage_all = reinterpret_cast<__nv_bfloat16*>(slots + DEC_NW * DEC_MAXSEG * NF4 * 32);
  uint32_t* cnt = reinterpret_cast<uint32_t*>(stage_all + DEC_NW * MT * 32);
  __nv_bfloat16* stage = stage_all + warp * MT * 32;

  const int epoch = *reinterpret_cast<volatile int*>(&a.hdr->epoch);
  const DecodeLayout L = decode_layout(DecodeShape{a.E2, a.P2, a.NC, a.kt_part}, cl);
  const int u0 = L.warp_first(warp), u1 = L.warp_first(warp + 1);

  uint4 bufA[8], bufB[8];
  if (u0 < u1) decode_load_unit<MT>(a, L, u0, q, lane, bufA);

  // x part of this CTA -> shared memory (rows >= M are zero)
  {
    const int kp = a.kt_part * 64;
    const int chunks = MT * (kp / 8);
    for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
      const int m = c / (kp / 8), kk = (c % (kp / 8)) * 8;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (m < a.M) v = __ldg(reinterpret_cast<const uint4*>(a.x + (size_t)m * a.K + (size_t)q * kp + kk));
      *reinterpret_cast<uint4*>(xs + (size_t)m * xs_stride + kk) = v;
    }
  }
  if (q == 0)
    for (int i = threadIdx.x; i < DEC_MAXPAIRS; i += blockDim.x) cnt[i] = 0;
  if (a.E2 == 0 && blockIdx.x == 0 && warp == 0) {
    if (a.gate_out && lane < a.M) a.gate_out[lane] = 0.f;
    if (a.mask_count && lane == 0) *a.mask_count = a.M;
  }
  __syncthreads();
  cluster_sync_all();

  float acc[2][NT][4];
  auto zero_acc = [&]() {
#pragma unroll
    for (int si = 0; si < 2; ++si)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[si][nt][i] = 0.f;
  };
  zero_acc();

  int stash_lp[DEC_MAXSEG];
  int stash_seg[DEC_MAXSEG];
  int n_stash = 0;
  const int lp_first = u0 < u1 ? L.lp_of(u0, a.kt_part) : 0;
  const uint32_t cnt_base = map_rank(smem_u32(cnt), 0);

  // Flush acc as this warp's contribution to pair lp; finalise if last.
  auto flush = [&](int lp) {
    const int seg = lp - lp_first;
    float4* my = slots + (size_t)((warp * DEC_MAXSEG + seg) * NF4) * 32;
#pragma unroll
    for (int si = 0; si < 2; ++si)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        my[(si * NT + nt) * 32 + lane] = make_float4(acc[si][nt][0], acc[si][nt][1], acc[si][nt][2], acc[si][nt][3]);
    __syncwarp();
    uint32_t old = 0;
    if (lane == 0) old = atom_add_dsmem_acqrel(cnt_base + 4 * lp, 1u);
    old = __shfl_sync(0xffffffffu, old, 0);
    const int fu = L.first_unit(lp, a.kt_part);
    const int wlo = L.warp_of(fu), whi = L.warp_of(fu + L.n_units(lp, a.kt_part) - 1);
    const uint32_t need = (uint32_t)(a.CS * L.contributors(lp, a.kt_part));
    zero_acc();
    if (old + 1 != need) return;
    fence_acq_rel_cluster();
    // last contributor: fixed-order sum over (CTA rank, warp)
    for (int qq = 0; qq < a.CS; ++qq) {
      for (int w2 = wlo; w2 <= whi; ++w2) {
        if (!L.warp_busy(w2)) continue;  // empty range: no slot written
        const int seg2 = lp - L.lp_of(L.warp_first(w2), a.kt_part);
        const uint32_t base = map_rank(smem_u32(slots + (size_t)((w2 * DEC_MAXSEG + seg2) * NF4) * 32), qq);
#pragma unroll
        for (int si = 0; si < 2; ++si)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const float4 v = ld_dsmem_f4(base + 16u * ((si * NT + nt) * 32 + lane));
            acc[si][nt][0] += v.x;
            acc[si][nt][1] += v.y;
            acc[si][nt][2] += v.z;
            acc[si][nt][3] += v.w;
          }
      }
    }
    if (lp < L.n_ec) {
      // EC rows: t (rows < r) and the gate logit (row r) -> ws_t[m][row]
      const int e = L.ec_lo + lp;
      const int RT = 32 * a.E2;
      const int rho = lane >> 2, cq = lane & 3;
#pragma unroll
      for (int si = 0; si < 2; ++si)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int row0 = 16 * (2 * e + si) + rho;
          const int m0 = nt * 8 + 2 * cq;
          a.ws_t[(size_t)m0 * RT + row0] = acc[si][nt][0];
          a.ws_t[(size_t)(m0 + 1) * RT + row0] = acc[si][nt][1];
          a.ws_t[(size_t)m0 * RT + row0 + 8] = acc[si][nt][2];
          a.ws_t[(size_t)(m0 + 1) * RT + row0 + 8] = acc[si][nt][3];
        }
      __syncwarp();
      __threadfence();
      int prev = 0;
      if (lane == 0) prev = atomicAdd(&a.hdr->ec_done, 1);
      prev = __shfl_sync(0xffffffffu, prev, 0);
      if (prev == a.E2 - 1) {
        __threadfence();
        decode_finish_gate<MT>(a, lane, epoch);
      }
      zero_acc();
      return;
    }
    const int pair = L.w_lo + (lp - L.n_ec);
    const bool ready = a.E2 == 0 || ld_acquire_gpu(&a.hdr->ec_flag) == epoch + 1;
    if (ready) {
      decode_store_pair<MT, GROUP>(a, pair, lane, true, stage, acc);
    } else {
      // park the reduced sum in this warp's own slot for the end
#pragma unroll
      for (int si = 0; si < 2; ++si)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          my[(si * NT + nt) * 32 + lane] =
              make_float4(acc[si][nt][0], acc[si][nt][1], acc[si][nt][2], acc[si][nt][3]);
      stash_lp[n_stash] = lp;
      stash_seg[n_stash] = seg;
      ++n_stash;
    }
    zero_acc();
  };

  int u = u0;
  while (u < u1) {
    if (u + 1 < u1) decode_load_unit<MT>(a, L, u + 1, q, lane, bufB);
    decode_compute_unit<MT, GROUP>(a, L, u, q, lane, bufA, xs, xs_stride, acc);
    {
      const int lp = L.lp_of(u, a.kt_part);
      if (u + 1 == u1 || L.lp_of(u + 1, a.kt_part) != lp) flush(lp);
    }
    ++u;
    if (u >= u1) break;
    if (u + 1 < u1) decode_load_unit<MT>(a, L, u + 1, q, lane, bufA);
    decode_compute_unit<MT, GROUP>(a, L, u, q, lane, bufB, xs, xs_stride, acc);
    {
      const int lp = L.lp_of(u, a.kt_part);
      if (u + 1 == u1 || L.lp_of(u + 1, a.kt_part) != lp) flush(lp);
    }
    ++u;
  }

  // parked pairs: wait (bounded) for the gated EC projection, then finish
  for (int i = 0; i < n_stash; ++i) {
    bool ok = true;
    if (lane == 0) ok = wait_flag_eq(&a.hdr->ec_flag, epoch + 1, a.hdr);
    ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
    const float4* my = slots + (size_t)((warp * DEC_MAXSEG + stash_seg[i]) * NF4) * 32;
#pragma unroll
    for (int si = 0; si < 2; ++si)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const float4 v = my[(si * NT + nt) * 32 + lane];
        acc[si][nt][0] = v.x;
        acc[si][nt][1] = v.y;
        acc[si][nt][2] = v.z;
        acc[si][nt][3] = v.w;
      }
    decode_store_pair<MT, GROUP>(a, L.w_lo + (stash_lp[i] - L.n_ec), lane, ok, stage, acc);
  }

  __syncthreads();
  cluster_sync_all();  // no CTA leaves while others may still read its slots
  if (threadIdx.x == 0) {
    __threadfence();
    const int prev = atomicAdd(&a.hdr->done_ctas, 1);
    if (prev == (int)gridDim.x - 1) {
      a.hdr->done_ctas = 0;
      a.hdr->ec_done = 0;
      __threadfence();
      atomicAdd(&a.hdr->epoch, 1);
    }
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
static size_t decode_smem_bytes(int MT, int kt_part) {
  const size_t xs = (size_t)MT * (kt_part * 64 + 8) * 2;
  const size_t slots = (size_t)DEC_NW * DEC_MAXSEG * (2 * MT / 8) * 32 * 16;
  const size_t stage = (size_t)DEC_NW * MT * 32 * 2;
  return xs + slots + stage + DEC_MAXPAIRS * 4;
}

template <int MT, bool GROUP>
static cudaError_t ensure_smem_attr(size_t smem) {
  // per kernel instantiation, the largest dynamic shared memory opted into so far
  static std::mutex mu;
  static size_t opted = 0;
  std::lock_guard<std::mutex> lk(mu);
  if (smem <= opted) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<MT, GROUP>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess) {
    cudaFuncSetAttribute(decode_kernel<MT, GROUP>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    opted = smem;
  }
  return e;
}

template <int MT, bool GROUP>
static int launch_decode_t(const DecodeArgs& a, size_t smem, cudaStream_t st) {
  cudaError_t e = ensure_smem_attr<MT, GROUP>(smem);
  if (e != cudaSuccess) return set_cuda_error("cudaFuncSetAttribute(decode)", e);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.NC * a.CS);
  cfg.blockDim = dim3(DEC_NW * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = a.CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, decode_kernel<MT, GROUP>, a);
  if (e != cudaSuccess) return set_cuda_error("decode launch", e);
  return SPEAR_OK;
}

// Largest number of co-resident clusters of size CS for this kernel.
template <int MT, bool GROUP>
static int max_clusters_t(int CS, size_t smem) {
  if (ensure_smem_attr<MT, GROUP>(smem) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CS);
  cfg.blockDim = dim3(DEC_NW * 32);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, decode_kernel<MT, GROUP>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

static DecodePlan make_decode_plan(int MT, int K, int N, int r, int group, int sm_count) {
  DecodePlan p = {};
  p.MT = MT;
  const int KT = K / 64;
  // K split: the smallest cluster size (1, 2, 4, 8 dividing K/64) whose x part
  // is at most 40 KB and 32 k-tiles; larger splits cut the x bytes each CTA
  // reads from L2 at the price of more partial sums.
  int CS = 1;
  const int cands[4] = {1, 2, 4, 8};
  for (int i = 0; i < 4; ++i) {
    const int c = cands[i];
    if (KT % c) continue;
    CS = c;
    const size_t xbytes = (size_t)p.MT * (KT / c) * 64 * 2;
    if (xbytes <= 40 * 1024 && (KT / c) <= 32) break;
  }
  p.CS = CS;
  p.kt_part = KT / CS;
  p.smem = decode_smem_bytes(p.MT, p.kt_part);
  p.E2 = r > 0 ? (r / 16 + 1 + 1) / 2 : 0;
  p.P2 = N / 32;
  p.RT = 32 * p.E2;
  int mc = 0;
  if (p.MT == 8)
    mc = group ? max_clusters_t<8, true>(CS, p.smem) : max_clusters_t<8, false>(CS, p.smem);
  else
    mc = group ? max_clusters_t<16, true>(CS, p.smem) : max_clusters_t<16, false>(CS, p.smem);
  if (mc <= 0) mc = sm_count / CS;
  int NC = std::min(mc, sm_count / CS);
  // every cluster gets at least DEC_UK pairs' worth of bytes
  const long long C = (long long)p.E2 * DEC_UK + p.P2;
  NC = (int)std::min<long long>(NC, std::max<long long>(1, C / DEC_UK));
  // one EC pair per cluster at most
  NC = std::max(NC, std::min(p.E2, mc > 0 ? mc : 1));
  p.NC = std::max(NC, 1);
  return p;
}

DecodePlan plan_decode(int M, int K, int N, int r, int group, int sm_count) {
  static std::mutex mu;
  static std::map<std::tuple<int, int, int, int, int, int, int>, DecodePlan> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  const int MT = M <= 8 ? 8 : 16;
  const auto key = std::make_tuple(dev, MT, K, N, r, group, sm_count);
  {
    std::lock_guard<std::mutex> lk(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
  }
  DecodePlan p = make_decode_plan(MT, K, N, r, group, sm_count);
  std::lock_guard<std::mutex> lk(mu);
  cache[key] = p;
  return p;
}

const char* check_decode_plan(const DecodePlan& p) {
  if (p.NC < 1 || p.kt_part < 1) return "empty plan";
  const DecodeShape sh{p.E2, p.P2, p.NC, p.kt_part};
  int prev_end = 0;
  for (int cl = 0; cl < p.NC; ++cl) {
    const DecodeLayout L = decode_layout(sh, cl);
    if (L.w_lo != prev_end) return "weight pairs are not partitioned contiguously";
    prev_end = L.w_lo + L.n_w;
    if (L.n_ec + L.n_w > DEC_MAXPAIRS) return "too many pairs per cluster";
    for (int w = 0; w < DEC_NW; ++w) {
      const int u0 = L.warp_first(w), u1 = L.warp_first(w + 1);
      if (u0 < u1 && L.lp_of(u1 - 1, p.kt_part) - L.lp_of(u0, p.kt_part) + 1 > DEC_MAXSEG)
        return "a warp's unit range spans too many pairs";
    }
  }
  if (prev_end != p.P2) return "weight pairs not covered";
  return nullptr;
}

int launch_decode(const DecodePlan& p, const LayerView& Lv, const __nv_bfloat16* x, int M, __nv_bfloat16* y,
                  WsHeader* hdr, float* ws_t, __nv_bfloat16* ws_gt, float* gate_out, int* mask_count, bool ec_only,
                  cudaStream_t st) {
  DecodeArgs a = {};
  a.w = Lv.w;
  a.scales = Lv.scales;
  a.agt = Lv.agt;
  a.bpt = Lv.bpt;
  a.x = x;
  a.y = y;
  a.gate_out = gate_out;
  a.mask_count = mask_count;
  a.hdr = hdr;
  a.ws_t = ws_t;
  a.ws_gt = ws_gt;
  a.M = M;
  a.K = Lv.K;
  a.N = Lv.N;
  a.r = Lv.r;
  a.group = Lv.group;
  a.b_g = Lv.b_g;
  a.tau = Lv.tau;
  a.CS = p.CS;
  a.NC = p.NC;
  a.kt_part = p.kt_part;
  a.E2 = p.E2;
  a.P2 = p.P2;
  a.ec_only = ec_only ? 1 : 0;
  if (p.MT == 8)
    return Lv.group ? launch_decode_t<8, true>(a, p.smem, st) : launch_decode_t<8, false>(a, p.smem, st);
  return Lv.group ? launch_decode_t<16, true>(a, p.smem, st) : launch_decode_t<16, false>(a, p.smem, st);
}

}  // namespace spear
