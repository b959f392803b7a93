// Decode path (M <= 16): split-K GEMV-style kernel with the gated EC fused.
//
// SPEAR fuses the whole EC computation into the low-bit GEMM for the
// memory-bound decode phase (gist.science technical summary, section 2.2 A,
// "Phase de decodage ... M=1": one kernel, no inter-kernel launch on the
// critical path).  This kernel does that for 1 <= M <= 16 on sm_100a.
//
// Work.  The output is cut into 32-channel "pairs" (two 16-channel strips of
// the packed layout) plus "EC pairs" (32 rows of [A^T ; w_g]).  A cluster of
// CS CTAs owns a contiguous set of pairs and splits K into CS parts, one per
// CTA.  A unit is 4 KB of operand bytes: a weight pair over 4 k-tiles (int4)
// or an EC pair over one k-tile (bf16).
//
// Streaming.  One producer warp issues TMA loads for every unit of the CTA
// into a ring of 4 KB shared-memory slots (dozens of KB in flight per SM, so
// the weights stream at HBM rate), after one TMA load of the CTA's part of x
// (128-byte swizzled, rows beyond M zero-filled).  Consumer warps own
// contiguous unit ranges; the producer issues units interleaved across the
// consumers so that every consumer finds its next unit in the ring.
//
// Math.  A consumer turns 8 nibbles into 4 bf16 pairs with one LOP3 each
// (bf16 128 + u, exact) and multiplies on the tensor cores (mma.sync
// m16n8k16, weights as the 16-row operand); the +136 offset of every code is
// removed once per k-tile in fp32 from per-k-tile token sums of x.
//
// Reduction.  A consumer writes its partial sum of a pair to a shared-memory
// slot and bumps the pair's arrival counter (atomics on distributed shared
// memory of CTA 0 of the cluster).  The last contributor adds every slot of
// the cluster in a fixed order (deterministic) through DSMEM.
//
// EC.  EC pairs are scheduled first.  Their reduced rows (t = x . A and the
// gate logit x . w_g) go to a small global buffer; the last one computes
// g = sigmoid(logit + b_g), gt = g * t (bf16) and raises an epoch-tagged flag.
// Weight pairs add gt . B' as r/16 MMA k-steps (B' = B / s_n folded once per
// layer), apply s_n and store bf16 y with 16-byte stores.  A pair reduced
// before the flag is up is parked in its slot and finished after the warp's
// last unit.  Every wait is bounded.
#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>

#include "common.cuh"
#include "kernels.h"
#include "tma.cuh"

namespace spear {

constexpr int DEC_NWC = 12;       // consumer warps
constexpr int DEC_THREADS = (DEC_NWC + 1) * 32;
constexpr int DEC_UK = 4;         // k-tiles (64 k each) per weight unit
constexpr int DEC_UNIT = 4096;    // bytes per unit
constexpr int DEC_MAXSEG = 2;     // pairs one consumer may touch
constexpr int DEC_MAXPAIRS = 64;  // pairs per cluster
constexpr int DEC_MAXRING = 40;
constexpr int DEC_MAXCL = 160;
constexpr int DEC_PREWAIT = 8;     // units requested before the grid-dependency wait     // clusters described in the kernel parameters

struct DecodeArgs {
  const __half* scales;
  const __nv_bfloat16* bpt;
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
  int ring;                // ring slots
  int ec_only;             // 1: skip the weights, y += EC term in place (unfused path)
  short4 cl_tab[DEC_MAXCL];  // per cluster: EC pair start, EC pairs, weight pair start, weight pairs
};

struct DecodeShape {
  int E2, P2, NC, kt_part;
};

// Units of one CTA: n_ec EC pairs x kt_part units, then n_w weight pairs x upw
// units.  Consumer w owns units [start(w), start(w) + len(w)), longer ranges
// first, so that consumer w's i-th unit is the producer's (i * NWC + w)-th.
struct DecodeLayout {
  int ec_lo, n_ec, w_lo, n_w, upw, U, base, rem;
  __host__ __device__ __forceinline__ int lp_of(int u, int kt_part) const {
    const int ecu = n_ec * kt_part;
    return u < ecu ? u / kt_part : n_ec + (u - ecu) / upw;
  }
  __host__ __device__ __forceinline__ int first_unit(int lp, int kt_part) const {
    return lp < n_ec ? lp * kt_part : n_ec * kt_part + (lp - n_ec) * upw;
  }
  __host__ __device__ __forceinline__ int n_units(int lp, int kt_part) const { return lp < n_ec ? kt_part : upw; }
  __host__ __device__ __forceinline__ int start(int w) const { return w * base + (w < rem ? w : rem); }
  __host__ __device__ __forceinline__ int len(int w) const { return base + (w < rem ? 1 : 0); }
  __host__ __device__ __forceinline__ int warp_of(int u) const {
    const int big = rem * (base + 1);
    return u < big ? u / (base + 1) : rem + (u - big) / base;
  }
  // consumers (per CTA) holding units of pair lp
  __host__ __device__ __forceinline__ int contributors(int lp, int kt_part) const {
    const int fu = first_unit(lp, kt_part);
    return warp_of(fu + n_units(lp, kt_part) - 1) - warp_of(fu) + 1;
  }
};

__host__ __device__ __forceinline__ int ceil_div_ll(long long n, long long d) { return (int)((n + d - 1) / d); }
__host__ __device__ __forceinline__ int clamp_ll(long long v, int hi) { return (int)(v < 0 ? 0 : (v > hi ? hi : v)); }

// Pairs of cluster cl: its EC pairs (spread evenly, at most one per cluster
// when E2 <= NC) followed by a contiguous range of weight pairs, chosen so that
// every cluster streams about the same number of bytes (an EC pair streams
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
  L.base = L.U / DEC_NWC;
  L.rem = L.U % DEC_NWC;
  return L;
}

__device__ __forceinline__ uint32_t u4w(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// Swizzled 128-byte-row tile (TMA SWIZZLE_128B): 16-byte chunk ch of row r.
__device__ __forceinline__ uint4 ld_sw128(const uint8_t* tile, int row, int ch) {
  return *reinterpret_cast<const uint4*>(tile + row * 128 + ((ch ^ (row & 7)) << 4));
}

// x fragments of k-tile kt for n8-tile nt: 8 words = x[nt*8 + rho][16c .. 16c + 16)
template <int MT>
__device__ __forceinline__ void load_x_frag(const uint8_t* xs, int kt, int lane, uint32_t (&xf)[MT / 8][8]) {
  const int rho = lane >> 2, cq = lane & 3;
  const uint8_t* tile = xs + kt * (MT * 128);
#pragma unroll
  for (int nt = 0; nt < MT / 8; ++nt) {
    const uint4 v0 = ld_sw128(tile, nt * 8 + rho, 2 * cq), v1 = ld_sw128(tile, nt * 8 + rho, 2 * cq + 1);
    xf[nt][0] = v0.x; xf[nt][1] = v0.y; xf[nt][2] = v0.z; xf[nt][3] = v0.w;
    xf[nt][4] = v1.x; xf[nt][5] = v1.y; xf[nt][6] = v1.z; xf[nt][7] = v1.w;
  }
}

// 8 nibbles -> 4 bf16x2 (128 + u each, exact): register pi = nibbles (pi, pi + 4)
__device__ __forceinline__ void nib_to_bf16_biased(uint32_t w, uint32_t (&o)[4]) {
#pragma unroll
  for (int pi = 0; pi < 4; ++pi) {
    uint32_t v;
    asm("lop3.b32 %0, %1, %2, %3, 0xea;" : "=r"(v) : "r"(w >> (4 * pi)), "r"(0x000F000Fu), "r"(0x43004300u));
    o[pi] = v;
  }
}

// One weight unit: 2 strips x up to 4 k-tiles from ring slot `src`
// (layout [strip][k-tile][32 lanes x 16 bytes]).  The MMAs see 136 + q for
// every code (bf16 128 + u, u = q + 8): per-channel scales accumulate
// directly and subtract 136 * sum(x) once per unit; group scales need one
// partial sum per 64-k tile.
template <int MT, bool GROUP>
__device__ __forceinline__ void compute_w_unit(const DecodeArgs& a, const uint8_t* src, const uint8_t* xs,
                                               const float* xsum, int kt0_local, int nkt, int pair, int q,
                                               int lane, float (&acc)[2][MT / 8][4]) {
  constexpr int NT = MT / 8;
  const int rho = lane >> 2, cq = lane & 3;
  if (!GROUP) {
    float xs0[NT], xs1[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) xs0[nt] = xs1[nt] = 0.f;
#pragma unroll
    for (int j = 0; j < DEC_UK; ++j) {
      if (j >= nkt) break;
      const int kt = kt0_local + j;
      uint32_t xf[NT][8];
      load_x_frag<MT>(xs, kt, lane, xf);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        xs0[nt] += xsum[kt * MT + nt * 8 + 2 * cq];
        xs1[nt] += xsum[kt * MT + nt * 8 + 2 * cq + 1];
      }
#pragma unroll
      for (int si = 0; si < 2; ++si) {
        const uint4 wv = *reinterpret_cast<const uint4*>(src + (si * DEC_UK + j) * 512 + lane * 16);
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          uint32_t af[4];
          nib_to_bf16_biased(u4w(wv, s), af);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(acc[si][nt], af, xf[nt][2 * s], xf[nt][2 * s + 1]);
        }
      }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const float b0 = 136.f * xs0[nt], b1 = 136.f * xs1[nt];
#pragma unroll
      for (int si = 0; si < 2; ++si) {
        acc[si][nt][0] -= b0;
        acc[si][nt][1] -= b1;
        acc[si][nt][2] -= b0;
        acc[si][nt][3] -= b1;
      }
    }
    return;
  }
#pragma unroll
  for (int j = 0; j < DEC_UK; ++j) {
    if (j >= nkt) break;
    const int kt = kt0_local + j;
    uint32_t xf[NT][8];
    load_x_frag<MT>(xs, kt, lane, xf);
    float part[2][NT][4];
#pragma unroll
    for (int si = 0; si < 2; ++si)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) part[si][nt][i] = 0.f;
#pragma unroll
    for (int si = 0; si < 2; ++si) {
      const uint4 wv = *reinterpret_cast<const uint4*>(src + (si * DEC_UK + j) * 512 + lane * 16);
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        uint32_t af[4];
        nib_to_bf16_biased(u4w(wv, s), af);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(part[si][nt], af, xf[nt][2 * s], xf[nt][2 * s + 1]);
      }
    }
    const int g = (q * a.kt_part + kt) >> 1;  // 128-k group of this 64-k tile
    float sc[2][2];
#pragma unroll
    for (int si = 0; si < 2; ++si) {
      const int n0 = 16 * (2 * pair + si) + rho;
      sc[si][0] = __half2float(a.scales[(size_t)g * a.N + n0]);
      sc[si][1] = __half2float(a.scales[(size_t)g * a.N + n0 + 8]);
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const float b0 = 136.f * xsum[kt * MT + nt * 8 + 2 * cq];
      const float b1 = 136.f * xsum[kt * MT + nt * 8 + 2 * cq + 1];
#pragma unroll
      for (int si = 0; si < 2; ++si) {
        acc[si][nt][0] = fmaf(sc[si][0], part[si][nt][0] - b0, acc[si][nt][0]);
        acc[si][nt][1] = fmaf(sc[si][0], part[si][nt][1] - b1, acc[si][nt][1]);
        acc[si][nt][2] = fmaf(sc[si][1], part[si][nt][2] - b0, acc[si][nt][2]);
        acc[si][nt][3] = fmaf(sc[si][1], part[si][nt][3] - b1, acc[si][nt][3]);
      }
    }
  }
}

// One EC unit: rows [32e, 32e + 32) of [A^T ; w_g] x one k-tile, TMA tile
// [32 rows][64 k] bf16 with 128-byte swizzle (rows beyond r zero-filled).
template <int MT>
__device__ __forceinline__ void compute_ec_unit(const uint8_t* src, const uint8_t* xs, int kt, int lane,
                                                float (&acc)[2][MT / 8][4]) {
  constexpr int NT = MT / 8;
  const int rho = lane >> 2, cq = lane & 3;
  uint32_t xf[NT][8];
  load_x_frag<MT>(xs, kt, lane, xf);
#pragma unroll
  for (int si = 0; si < 2; ++si) {
    const int r0 = 16 * si + rho, r1 = r0 + 8;
    const uint4 a00 = ld_sw128(src, r0, 2 * cq), a01 = ld_sw128(src, r0, 2 * cq + 1);
    const uint4 a10 = ld_sw128(src, r1, 2 * cq), a11 = ld_sw128(src, r1, 2 * cq + 1);
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      // words 2s (k + 0, 1) and 2s + 1 (k + 2, 3) of rows rho and rho + 8
      const uint4& lo0 = s < 2 ? a00 : a01;
      const uint4& lo1 = s < 2 ? a10 : a11;
      uint32_t af[4] = {u4w(lo0, (2 * s) & 3), u4w(lo1, (2 * s) & 3), u4w(lo0, (2 * s + 1) & 3),
                        u4w(lo1, (2 * s + 1) & 3)};
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(acc[si][nt], af, xf[nt][2 * s], xf[nt][2 * s + 1]);
    }
  }
}

// 8*S bytes of row `row` of a row-major [.. x ld] bf16 matrix at columns
// jbase + 4*S*cq, as words w[0 .. 2S).
template <int S>
__device__ __forceinline__ void load_rowchunk(const __nv_bfloat16* base, int ld, int row, int jbase, int cq,
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

template <int MT, int S>
__device__ __forceinline__ void ec_upproject_chunk(const DecodeArgs& a, int pair, int lane, int jbase,
                                                   float (&acc)[2][MT / 8][4]) {
  const int rho = lane >> 2, cq = lane & 3;
  uint32_t g[MT / 8][8], b[2][2][8];
#pragma unroll
  for (int nt = 0; nt < MT / 8; ++nt) load_rowchunk<S>(a.ws_gt, a.r, nt * 8 + rho, jbase, cq, g[nt]);
#pragma unroll
  for (int si = 0; si < 2; ++si) {
    const int n0 = 16 * (2 * pair + si) + rho;
    load_rowchunk<S>(a.bpt, a.r, n0, jbase, cq, b[si][0]);
    load_rowchunk<S>(a.bpt, a.r, n0 + 8, jbase, cq, b[si][1]);
  }
#pragma unroll
  for (int si = 0; si < 2; ++si)
#pragma unroll
    for (int s = 0; s < S; ++s) {
      uint32_t af[4] = {b[si][0][2 * s], b[si][1][2 * s], b[si][0][2 * s + 1], b[si][1][2 * s + 1]};
#pragma unroll
      for (int nt = 0; nt < MT / 8; ++nt) mma_bf16_16816(acc[si][nt], af, g[nt][2 * s], g[nt][2 * s + 1]);
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
    if (m < a.M && SPEAR_DCHECK(32 * pair + 32 <= a.N, a.hdr)) {
      uint4 v = *reinterpret_cast<const uint4*>(stage + m * 32 + part * 8);
      uint4* dst = reinterpret_cast<uint4*>(a.y + (size_t)m * a.N + 32 * pair + part * 8);
      if (a.ec_only) {
        // y already holds the EC-disabled GEMM result: add the EC term in fp32, round once more
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
  if (lane < MT) gm = sigmoidf_(__ldcg(a.ws_t + (size_t)lane * RT + a.r) + a.b_g);
  const bool valid = lane < a.M;
  if (a.gate_out && valid) a.gate_out[lane] = gm;
  const unsigned below = __ballot_sync(0xffffffffu, valid && gm < a.tau);
  if (a.mask_count && lane == 0) *a.mask_count = __popc(below);
  // gt[m][j] = bf16(g_m t[m][j]); each lane owns column pairs of every token
  for (int m = 0; m < MT; ++m) {
    const float g = __shfl_sync(0xffffffffu, gm, m);
    const float* trow = a.ws_t + (size_t)m * RT;
    for (int j = 2 * lane; j < a.r; j += 64) {
      const float2 t = __ldcg(reinterpret_cast<const float2*>(trow + j));
      *reinterpret_cast<uint32_t*>(a.ws_gt + (size_t)m * a.r + j) = pack_bf16x2(g * t.x, g * t.y);
    }
  }
  __syncwarp();
  __threadfence();
  if (lane == 0) st_release_gpu(&a.hdr->ec_flag, epoch + 1);
}

template <int MT, bool GROUP>
__global__ void __launch_bounds__(DEC_THREADS, 1)
    decode_kernel(const __grid_constant__ DecodeArgs a, const __grid_constant__ CUtensorMap tm_x,
                  const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_agt) {
  constexpr int NT = MT / 8;
  constexpr int NF4 = 2 * NT;  // float4 fragments per lane per slot
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, derived from the shared array itself so that the
  // compiler keeps every access in the shared window (ld/st.shared)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* ring = smem;                                       // [ring][4 KB]
  uint8_t* xs = ring + (size_t)a.ring * DEC_UNIT;             // [kt_part][MT x 128 B], swizzled
  float4* slots = reinterpret_cast<float4*>(xs + (size_t)a.kt_part * MT * 128);
  float* xsum = reinterpret_cast<float*>(slots + DEC_NWC * DEC_MAXSEG * NF4 * 32);  // [kt_part][MT]
  uint64_t* full = reinterpret_cast<uint64_t*>(xsum + a.kt_part * MT);
  uint64_t* empty = full + DEC_MAXRING;
  uint64_t* xbar = empty + DEC_MAXRING;
  uint32_t* cnt = reinterpret_cast<uint32_t*>(xbar + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = (int)cluster_rank();
  const int cl = blockIdx.x / a.CS;
  DecodeLayout L;
  {
    const short4 t = a.cl_tab[cl];
    L.ec_lo = t.x;
    L.n_ec = t.y;
    L.w_lo = t.z;
    L.n_w = t.w;
    L.upw = (a.kt_part + DEC_UK - 1) / DEC_UK;
    L.U = L.n_ec * a.kt_part + L.n_w * L.upw;
    L.base = L.U / DEC_NWC;
    L.rem = L.U - L.base * DEC_NWC;
  }
  const int ecu = L.n_ec * a.kt_part;

  // TMA job of producer issue index j (consumer j % NWC, its (j / NWC)-th unit):
  // kind 0 = weight unit (3-D box at {0, kt0, 2 * pair}), 1 = EC unit (2-D box
  // at {kt * 64, 32 * e}), 2 = nothing to load (EC-only launch, weight unit).
  // Computed by all producer lanes in parallel; lane 0 issues.
  auto job_of = [&](int j, int& kind, int& c1, int& c2) {
    const int w = j % DEC_NWC, i = j / DEC_NWC;
    const int u = L.start(w) + i;
    if (u < ecu) {
      kind = 1;
      c1 = (q * a.kt_part + u % a.kt_part) * 64;
      c2 = 32 * (L.ec_lo + u / a.kt_part);
    } else {
      const int v = u - ecu;
      kind = a.ec_only ? 2 : 0;
      c1 = q * a.kt_part + (v % L.upw) * DEC_UK;
      c2 = 2 * (L.w_lo + v / L.upw);
    }
  };
  auto issue_job = [&](int slot, int kind, int c1, int c2) {
    uint8_t* dst = ring + (size_t)slot * DEC_UNIT;
    if (kind == 2) {
      mbar_arrive(&full[slot]);  // EC-only launch: the weights are not needed
      return;
    }
    mbar_arrive_tx(&full[slot], DEC_UNIT);
    if (kind == 1)
      tma_load_2d(smem_u32(dst), &tm_agt, &full[slot], c1, c2);
    else
      tma_load_3d(smem_u32(dst), &tm_w, &full[slot], 0, c1, c2);
  };

  // weights (and [A^T ; w_g]) do not depend on the previous kernel in the
  // stream: a few units are requested before the grid-dependency wait; x goes
  // right after the wait, ahead of the rest of the ring (so it does not queue
  // behind megabytes of weight requests)
  const int first_batch = L.U < a.ring ? L.U : a.ring;
  const int pre_batch = first_batch < DEC_PREWAIT ? first_batch : DEC_PREWAIT;
  if (warp == 0) {
    for (int s = lane; s < a.ring; s += 32) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    if (lane == 0) mbar_init(xbar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    __syncwarp();
    for (int j = lane; j < pre_batch; j += 32) {
      int kind, c1, c2;
      job_of(j, kind, c1, c2);
      issue_job(j, kind, c1, c2);
    }
  } else if (q == 0) {
    for (int i = threadIdx.x - 32; i < DEC_MAXPAIRS; i += DEC_NWC * 32) cnt[i] = 0;
  }
  __syncthreads();
  // cluster phase: counters initialised (arrive now, wait before the first remote
  // atomic).  The producer wrote nothing to publish and must not wait here for
  // its TMA loads, so it arrives relaxed.
  if (warp == 0)
    asm volatile("barrier.cluster.arrive.relaxed;" ::: "memory");
  else
    asm volatile("barrier.cluster.arrive.release;" ::: "memory");
  // let the next kernel in the stream start its own weight prefetch as our CTAs drain
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // x, the workspace and y may belong to the previous kernel in the stream
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int epoch = *reinterpret_cast<volatile int*>(&a.hdr->epoch);
  if (a.E2 == 0 && blockIdx.x == 0 && warp == 1) {
    if (a.gate_out && lane < a.M) a.gate_out[lane] = 0.f;
    if (a.mask_count && lane == 0) *a.mask_count = a.M;
  }

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      const int kp = a.kt_part * 64;
      mbar_arrive_tx(xbar, a.kt_part * MT * 128);
      for (int kt = 0; kt < a.kt_part; ++kt)
        tma_load_2d(smem_u32(xs + kt * MT * 128), &tm_x, xbar, q * kp + kt * 64, 0);
    }
    __syncwarp();
    for (int j = pre_batch + lane; j < first_batch; j += 32) {
      int kind, c1, c2;
      job_of(j, kind, c1, c2);
      issue_job(j, kind, c1, c2);
    }
    // remaining units: slot s is always refilled by lane s % 32, in issue
    // order, so no lane waits on a slot more than one phase ahead
    int abort_local = 0;
    for (int j = first_batch; j < L.U; ++j) {
      const int slot = j % a.ring;
      if ((slot & 31) != lane) continue;
      if (!mbar_wait(&empty[slot], ((j / a.ring) & 1) ^ 1, &abort_local, a.hdr)) break;
      int kind, c1, c2;
      job_of(j, kind, c1, c2);
      issue_job(slot, kind, c1, c2);
    }
    __syncwarp();
    asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
  } else {
    // ---------------------------------------------------------------- consumers
    const int cw = warp - 1;
    int abort_local = 0;
    // per-k-tile token sums of x (for removing the +136 code bias)
    const bool xok = __all_sync(0xffffffffu, mbar_wait(xbar, 0, &abort_local, a.hdr));
    if (xok) {
      for (int e = threadIdx.x - 32; e < a.kt_part * MT; e += DEC_NWC * 32) {
        const int kt = e / MT, m = e % MT;
        const uint8_t* tile = xs + kt * (MT * 128);
        float sum = 0.f;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint4 v = ld_sw128(tile, m, ch);
          const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[i]));
            sum += f.x + f.y;
          }
        }
        xsum[e] = sum;
      }
    }
    asm volatile("bar.sync 1, %0;" ::"r"(DEC_NWC * 32) : "memory");  // consumers only
    asm volatile("barrier.cluster.wait.acquire;" ::: "memory");

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
    int stash_lp0 = 0, stash_lp1 = 0, n_stash = 0;
    const int u0 = L.start(cw), nu = L.len(cw);
    const int lp_first = nu > 0 ? L.lp_of(u0, a.kt_part) : 0;
    const uint32_t cnt_base = map_rank(smem_u32(cnt), 0);

    auto flush = [&](int lp) {
      const int seg = lp - lp_first;
      float4* my = slots + (size_t)((cw * DEC_MAXSEG + seg) * NF4) * 32;
#pragma unroll
      for (int si = 0; si < 2; ++si)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          my[(si * NT + nt) * 32 + lane] = make_float4(acc[si][nt][0], acc[si][nt][1], acc[si][nt][2], acc[si][nt][3]);
      __syncwarp();
      uint32_t old = 0;
      if (lane == 0) old = atom_add_dsmem_acqrel(cnt_base + 4 * lp, 1u);
      old = __shfl_sync(0xffffffffu, old, 0);
      const uint32_t need = (uint32_t)(a.CS * L.contributors(lp, a.kt_part));
      zero_acc();
      if (old + 1 != need) return;
      fence_acq_rel_cluster();
      // last contributor: fixed-order sum over (CTA rank, consumer)
      const int fu = L.first_unit(lp, a.kt_part);
      const int wlo = L.warp_of(fu), whi = L.warp_of(fu + L.n_units(lp, a.kt_part) - 1);
      for (int qq = 0; qq < a.CS; ++qq) {
        for (int w2 = wlo; w2 <= whi; ++w2) {
          const int seg2 = lp - L.lp_of(L.start(w2), a.kt_part);
          const uint32_t base = map_rank(smem_u32(slots + (size_t)((w2 * DEC_MAXSEG + seg2) * NF4) * 32), qq);
          float4 v[2][NT];
#pragma unroll
          for (int si = 0; si < 2; ++si)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) v[si][nt] = ld_dsmem_f4(base + 16u * ((si * NT + nt) * 32 + lane));
#pragma unroll
          for (int si = 0; si < 2; ++si)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              acc[si][nt][0] += v[si][nt].x;
              acc[si][nt][1] += v[si][nt].y;
              acc[si][nt][2] += v[si][nt].z;
              acc[si][nt][3] += v[si][nt].w;
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
            const int row0 = 32 * e + 16 * si + rho;
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
        // the last contributor's own slot is no longer read by anyone: use it as staging
        __syncwarp();
        decode_store_pair<MT, GROUP>(a, pair, lane, true, reinterpret_cast<__nv_bfloat16*>(my), acc);
      } else {
        // park the reduced sum in this consumer's own slot for the end
        __syncwarp();
#pragma unroll
        for (int si = 0; si < 2; ++si)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            my[(si * NT + nt) * 32 + lane] =
                make_float4(acc[si][nt][0], acc[si][nt][1], acc[si][nt][2], acc[si][nt][3]);
        if (n_stash == 0)
          stash_lp0 = lp;
        else
          stash_lp1 = lp;
        ++n_stash;
      }
      zero_acc();
    };

    bool ok = xok;
    for (int i = 0; i < nu && ok; ++i) {
      const int j = i * DEC_NWC + cw;
      const int slot = j % a.ring;
      ok = __all_sync(0xffffffffu, mbar_wait(&full[slot], (j / a.ring) & 1, &abort_local, a.hdr));
      if (!ok) break;
      const int u = u0 + i;
      const uint8_t* src = ring + (size_t)slot * DEC_UNIT;
      if (a.E2 > 0 && u >= ecu && (i == 0 || L.lp_of(u - 1, a.kt_part) != L.lp_of(u, a.kt_part))) {
        // this consumer starts a weight pair: warm L2 with its 32 rows of B' for the epilogue
        const __nv_bfloat16* row = a.bpt + (size_t)(32 * (L.w_lo + (u - ecu) / L.upw) + lane) * a.r;
        for (int off = 0; off < a.r; off += 64) asm volatile("prefetch.global.L2 [%0];" ::"l"(row + off));
      }
      if (u < ecu) {
        compute_ec_unit<MT>(src, xs, u % a.kt_part, lane, acc);
      } else if (!a.ec_only) {
        const int v = u - ecu;
        const int kt0 = (v % L.upw) * DEC_UK;
        const int nkt = min(DEC_UK, a.kt_part - kt0);
        compute_w_unit<MT, GROUP>(a, src, xs, xsum, kt0, nkt, L.w_lo + v / L.upw, q, lane, acc);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
      const int lp = L.lp_of(u, a.kt_part);
      if (i + 1 == nu || L.lp_of(u + 1, a.kt_part) != lp) flush(lp);
    }

    // parked pairs: wait (bounded) for the gated EC projection, then finish
    for (int i = 0; i < n_stash; ++i) {
      const int lp = i == 0 ? stash_lp0 : stash_lp1;
      bool fl = true;
      if (lane == 0) fl = wait_flag_eq(&a.hdr->ec_flag, epoch + 1, a.hdr);
      fl = __shfl_sync(0xffffffffu, (int)fl, 0) != 0;
      float4* my = slots + (size_t)((cw * DEC_MAXSEG + (lp - lp_first)) * NF4) * 32;
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
      __syncwarp();
      decode_store_pair<MT, GROUP>(a, L.w_lo + (lp - L.n_ec), lane, fl, reinterpret_cast<__nv_bfloat16*>(my), acc);
    }
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
static size_t decode_fixed_smem(int MT, int kt_part) {
  const size_t xs = (size_t)kt_part * MT * 128;
  const size_t slots = (size_t)DEC_NWC * DEC_MAXSEG * (2 * MT / 8) * 32 * 16;
  const size_t xsum = (size_t)kt_part * MT * 4;
  const size_t bars = (2 * DEC_MAXRING + 1) * 8 + DEC_MAXPAIRS * 4;
  return xs + slots + xsum + bars + 1024 /* alignment */;
}

template <int MT, bool GROUP>
static cudaError_t ensure_smem_attr(size_t smem) {
  // per kernel instantiation, the largest dynamic shared memory opted into so far
  static std::mutex mu;
  static size_t opted = 0;
  std::lock_guard<std::mutex> lk(mu);
  if (smem <= opted) return cudaSuccess;
  cudaError_t e =
      cudaFuncSetAttribute(decode_kernel<MT, GROUP>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess) {
    cudaFuncSetAttribute(decode_kernel<MT, GROUP>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    opted = smem;
  }
  return e;
}

template <int MT, bool GROUP>
static int launch_decode_t(const DecodeArgs& a, const CUtensorMap* maps, size_t smem, cudaStream_t st) {
  cudaError_t e = ensure_smem_attr<MT, GROUP>(smem);
  if (e != cudaSuccess) return set_cuda_error("cudaFuncSetAttribute(decode)", e);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.NC * a.CS);
  cfg.blockDim = dim3(DEC_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = a.CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // programmatic dependent launch: this grid may start while the previous
  // kernel in the stream drains; it waits for it before touching x / y / ws
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, decode_kernel<MT, GROUP>, a, maps[0], maps[1], maps[2]);
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
  cfg.blockDim = dim3(DEC_THREADS);
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

static constexpr size_t kDecodeSmemCap = 226 * 1024;

static DecodePlan make_decode_plan(int MT, int K, int N, int r, int group, int sm_count) {
  DecodePlan p = {};
  p.MT = MT;
  const int KT = K / 64;
  // K split: the smallest cluster size (1, 2, 4, 8 dividing K/64) whose x part
  // is at most 32 KB; larger splits cut the x bytes each CTA reads from L2
  // at the price of more partial sums.
  int CS = 1;
  const int cands[4] = {1, 2, 4, 8};
  for (int i = 0; i < 4; ++i) {
    const int c = cands[i];
    if (KT % c) continue;
    CS = c;
    if ((size_t)MT * (KT / c) * 128 <= 32 * 1024) break;
  }
  // tuning override of the K split (cluster size), honoured when it divides K/64
  if (const char* e = getenv("SPEAR_DECODE_CS")) {
    const int c = atoi(e);
    if ((c == 1 || c == 2 || c == 4 || c == 8) && KT % c == 0) CS = c;
  }
  p.CS = CS;
  p.kt_part = KT / CS;
  const size_t fixed = decode_fixed_smem(MT, p.kt_part);
  int ring = (int)((kDecodeSmemCap - std::min(fixed, kDecodeSmemCap)) / DEC_UNIT);
  ring = std::min(ring, DEC_MAXRING);
  p.ring = ring;
  p.smem = fixed + (size_t)ring * DEC_UNIT;
  p.E2 = r > 0 ? (r / 16 + 1 + 1) / 2 : 0;
  p.P2 = N / 32;
  p.RT = 32 * p.E2;
  int mc = 0;
  if (ring >= 4) {
    if (MT == 8)
      mc = group ? max_clusters_t<8, true>(CS, p.smem) : max_clusters_t<8, false>(CS, p.smem);
    else
      mc = group ? max_clusters_t<16, true>(CS, p.smem) : max_clusters_t<16, false>(CS, p.smem);
  }
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
  if (p.ring < 4 || p.ring > DEC_MAXRING) return "x part of K too large for shared memory (use the tensor-core path)";
  const DecodeShape sh{p.E2, p.P2, p.NC, p.kt_part};
  int prev_end = 0;
  for (int cl = 0; cl < p.NC; ++cl) {
    const DecodeLayout L = decode_layout(sh, cl);
    if (L.w_lo != prev_end) return "weight pairs are not partitioned contiguously";
    prev_end = L.w_lo + L.n_w;
    if (L.n_ec + L.n_w > DEC_MAXPAIRS) return "too many pairs per cluster";
    for (int w = 0; w < DEC_NWC; ++w) {
      const int u0 = L.start(w), n = L.len(w);
      if (n > 0 && L.lp_of(u0 + n - 1, p.kt_part) - L.lp_of(u0, p.kt_part) + 1 > DEC_MAXSEG)
        return "a consumer's unit range spans too many pairs";
    }
  }
  if (prev_end != p.P2) return "weight pairs not covered";
  return nullptr;
}

int launch_decode(const DecodePlan& p, const LayerView& Lv, const __nv_bfloat16* x, int M, __nv_bfloat16* y,
                  WsHeader* hdr, float* ws_t, __nv_bfloat16* ws_gt, float* gate_out, int* mask_count, bool ec_only,
                  cudaStream_t st) {
  DecodeArgs a = {};
  a.scales = Lv.scales;
  a.bpt = Lv.bpt;
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
  a.E2 = Lv.r > 0 ? p.E2 : 0;
  a.P2 = p.P2;
  a.ring = p.ring;
  a.ec_only = ec_only ? 1 : 0;
  if (p.NC > DEC_MAXCL) return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "too many clusters for the decode path");
  for (int c = 0; c < p.NC; ++c) {
    const DecodeLayout Lc = decode_layout(DecodeShape{a.E2, p.P2, p.NC, p.kt_part}, c);
    a.cl_tab[c] = make_short4((short)Lc.ec_lo, (short)Lc.n_ec, (short)Lc.w_lo, (short)Lc.n_w);
  }
  CUtensorMap maps[3];
  memset(maps, 0, sizeof(maps));
  bool ok = tmap_2d_bf16(&maps[0], x, Lv.K, M, 64, p.MT) && tmap_packed_box(&maps[1], Lv.w, Lv.K, Lv.N, DEC_UK, 2);
  if (ok && a.E2 > 0) ok = tmap_2d_bf16(&maps[2], Lv.agt, Lv.K, Lv.r + 1, 64, 32);
  if (!ok) return set_error(SPEAR_ERR_CUDA, "cuTensorMapEncodeTiled failed (decode)");
  if (p.MT == 8)
    return Lv.group ? launch_decode_t<8, true>(a, maps, p.smem, st) : launch_decode_t<8, false>(a, maps, p.smem, st);
  return Lv.group ? launch_decode_t<16, true>(a, maps, p.smem, st) : launch_decode_t<16, false>(a, maps, p.smem, st);
}

}  // namespace spear
