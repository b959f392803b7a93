// Decode path (1 <= M <= 16) on sm_100a: W4 GEMV with the gated EC fused,
// built for back-to-back launches.
//
// SPEAR fuses the whole EC computation into the low-bit GEMM for the
// memory-bound decode phase (gist.science technical summary, section 2.2 A,
// decode at M = 1: one kernel, no inter-kernel launch on the critical path).
//
// Residency.  Two CTAs per SM per launch, each half an SM (192 threads, at
// most 112 KB of shared memory), so the whole grid is resident at once.  The
// next launch in the stream (programmatic dependent launch) takes an SM's
// halves as this one leaves them and streams its own weights before it waits.
//
// Split.  K is cut into CS parts, one per CTA of a cluster, and each part into
// 4 warp slices of KTW 64-wide k-tiles.  A consumer warp loads the activations
// of its slice once, as mma.sync B fragments in registers, and applies them to
// every 16-channel strip of its cluster.
//
// Streaming.  The producer warp issues TMA loads of units of at most 8 KB into
// a shared-memory ring.  Weights, [A^T ; w_g] and the epilogue operands (B'
// rows, scales) do not depend on the previous kernel in the stream: the
// epilogue operands and the first two ring units are requested before the
// grid-dependency wait, the rest of the ring after it (a full ring requested
// early delays the activation load that follows the wait).
//
// Reduction, in a fixed order.  The 4 warp partials of a strip go through
// shared memory to the reducer warp.  With CS > 1 the CTA partials go to the
// strip's owner CTA (strip index mod CS) by st.async into its shared memory and
// are added in rank order.  The owner runs the strip's epilogue.
//
// EC.  The r + 1 rows of [A^T ; w_g] form 16-row EC strips, scheduled first in
// a few clusters.  The owner of an EC strip stores its reduced rows x . [A ; w_g]
// as 64-bit words (value, launch tag) in the workspace, so readers need no
// counter: the reducer of every CTA fetches the words (cp.async, without
// blocking), and once every tag is this launch's it computes the gate
// g = sigmoid(x . w_g + b_g) and gt = g * (x . A) in shared memory.  Strips
// reduced before that are parked in shared memory.  The epilogue adds gt . B'
// on the tensor cores (B' = B / s_n per channel, B for group scales), scales,
// and stores bf16 y with 16-byte stores.
//
// Every wait is bounded; a timeout is reported in the workspace status word.
#include <algorithm>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include "common.cuh"
#include "kernels.h"
#include "tma.cuh"

namespace spear {

constexpr int D2_NWC = 4;                       // consumer warps (one per SM sub-partition)
constexpr int D2_THREADS = (D2_NWC + 2) * 32;   // + one producer and one reducer warp
constexpr int D2_SLOT = 8192;                   // ring slot bytes
constexpr int D2_MAXSLOT = 16;
// partial-sum buffers (jobs in flight per CTA) and weight strips per job
__host__ __device__ constexpr int d2_nbuf(int MT) { return 4; }
__host__ __device__ constexpr int d2_bj(int MT) { return MT > 0 ? 1 : 1; }
constexpr int D2_PRE_UNITS = 2;                 // ring units requested before the grid-dependency wait
constexpr int D2_MAXCL = 160;                   // clusters described in the kernel parameters
constexpr int D2_MAXOWN = 16;                   // strips one CTA finishes per launch
constexpr int D2_KTW_MAX = 8;                   // warp slice (k-tiles): KTW * NT * 8 activation registers
constexpr size_t D2_SMEM_CAP = 112 * 1024;      // two CTAs per SM

template <int MT>
struct D2T {
  static constexpr int NT = MT / 8;             // n8 token tiles
  static constexpr int ACCS = MT == 8 ? 4 : 2;  // accumulator sets per strip (k16 step mod ACCS)
};
// warps sharing one ring unit and EC tiles per warp in one unit (units <= 8 KB)
__host__ __device__ constexpr int d2_wpu(int ktw) { return ktw >= 5 ? 2 : 4; }
__host__ __device__ constexpr int d2_ecu(int ktw) { return 4 / d2_wpu(ktw); }

struct D2Args {
  const __half* scales;
  const __nv_bfloat16* x;
  __nv_bfloat16* y;
  float* gate_out;
  int* mask_count;
  WsHeader* hdr;
  unsigned long long* tt;   // [ES][MT][16]: EC projection rows as (fp32 bits, launch tag) words
  int M, K, N, r, group;
  float b_g, tau;
  int CS, NC, G;            // cluster size (= K parts), clusters, CTAs
  int KTP;                  // k-tiles per part
  int ES;                   // EC strips (0: EC off)
  int nslot, own_cap;
  int ec_only;              // 1: no weights, y += EC term in place (unfused path)
  int gate_kind, gate_h;    // 0: scalar gate; 1: per-rank gamma(t) with bottleneck h
  const float *gw1, *gb1, *gw2, *gb2;
  float alpha;
  short4 cl_tab[D2_MAXCL];  // per cluster: first EC strip, EC strips, first weight strip, weight strips
};

// Shared-memory carve-up (same on host and device).
struct D2Smem {
  uint32_t ring, red, recv, park, bps, scs, ts, gts, gsc, gpar, stage, bars, total;
};
// rank-gate parameters staged in shared memory: W1 [h][r], W2 [r][h], b1 [h], b2 [r] (fp32)
__host__ __device__ __forceinline__ uint32_t d2_gpar_floats(int h, int r) { return 2 * h * r + h + r; }
__host__ __device__ __forceinline__ uint32_t d2_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }
__host__ __device__ __forceinline__ D2Smem d2_smem(int MT, int nslot, int CS, int own_cap, int r, int ES,
                                                   int gate_kind, int gate_h) {
  D2Smem s;
  const uint32_t NT = MT / 8;
  uint32_t off = 0;
  s.ring = off;
  off += nslot * D2_SLOT;
  s.red = off;
  off += d2_nbuf(MT) * D2_NWC * d2_bj(MT) * NT * 512;
  s.recv = off;
  off += CS > 1 ? own_cap * (CS - 1) * NT * 512 : 0;
  s.park = off;
  off += own_cap * NT * 512;
  s.bps = off;  // B' rows of the strips this CTA finishes: [own][16][r] bf16
  off += d2_up(own_cap * 32 * r, 128);
  s.scs = off;  // their per-channel scales: [own][16] fp16
  off += own_cap * 32;
  s.ts = off;   // staged EC projection words
  off += ES * MT * 16 * 8;
  s.gts = off;  // gt [MT][r + 8] bf16
  off += d2_up(MT * (r + 8) * 2, 16);
  s.gsc = off;  // rank gate: hidden activations [MT][32] fp32
  off += gate_kind ? MT * 32 * 4 : 0;
  s.gpar = off;  // rank gate: W1, W2, b1, b2
  off += gate_kind ? d2_up(d2_gpar_floats(gate_h, r) * 4, 16) : 0;
  s.stage = off;
  off += MT * 32;
  s.bars = off;
  off += (2 * nslot + 2 * d2_nbuf(MT) + own_cap + 2) * 8;
  s.total = off + 1024;  // base alignment slack
  return s;
}

__device__ __forceinline__ uint32_t d2_w(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// 8 nibbles -> 4 bf16x2 holding 128 + u (exact): register pi = nibbles (pi, pi + 4)
__device__ __forceinline__ void d2_nib_biased(uint32_t w, uint32_t (&o)[4]) {
#pragma unroll
  for (int pi = 0; pi < 4; ++pi) {
    uint32_t v;
    asm("lop3.b32 %0, %1, %2, %3, 0xea;" : "=r"(v) : "r"(w >> (4 * pi)), "r"(0x000F000Fu), "r"(0x43004300u));
    o[pi] = v;
  }
}

// Bounded wait on an mbarrier phase; the warp sleeps in hardware (up to
// `sleep_ns` per try) until the phase completes.  `idle` runs between tries.
// False after a timeout (reported) or once another role has given up.
template <typename Idle>
__device__ __forceinline__ bool d2_wait_idle(uint64_t* bar, uint32_t parity, volatile int* abort_flag, WsHeader* h,
                                             uint32_t sleep_ns, Idle&& idle) {
  if (mbar_test(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait_sleep(bar, parity, sleep_ns)) {
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitCycles) {
      report_status(h, SPEAR_ERR_TIMEOUT);
      *abort_flag = 1;
      return false;
    }
    idle();
  }
  return true;
}
__device__ __forceinline__ bool d2_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, WsHeader* h) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  for (int it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63) == 0) {
      if (*abort_flag) return false;
      if (clock64() - t0 > kWaitCycles) {
        report_status(h, SPEAR_ERR_TIMEOUT);
        *abort_flag = 1;
        return false;
      }
    }
  }
}

// Bounded wait for warps that must not take issue slots from the consumer
// warps: a non-blocking test, then sleeps of growing length (up to max_ns).
__device__ __forceinline__ bool d2_wait_polite(uint64_t* bar, uint32_t parity, volatile int* abort_flag, WsHeader* h,
                                               uint32_t max_ns) {
  if (mbar_test(bar, parity)) return true;
  const long long t0 = clock64();
  uint32_t ns = 32;
  while (true) {
    __nanosleep(ns);
    if (mbar_test(bar, parity)) return true;
    ns = ns * 2 < max_ns ? ns * 2 : max_ns;
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitCycles) {
      report_status(h, SPEAR_ERR_TIMEOUT);
      *abort_flag = 1;
      return false;
    }
  }
}

// Swizzled 128-byte-row tile (TMA SWIZZLE_128B): 16-byte chunk ch of row r.
__device__ __forceinline__ uint4 d2_sw128(const uint8_t* tile, int row, int ch) {
  return *reinterpret_cast<const uint4*>(tile + row * 128 + ((ch ^ (row & 7)) << 4));
}

// One EC tile: 16 rows of [A^T ; w_g] x 64 k (bf16, SW128) against the
// activations of the same k-tile.  Lane (rho, c) feeds k [16c, 16c + 16) of
// rows rho and rho + 8, the k order the activation fragments use.
template <int NT>
__device__ __forceinline__ void d2_ec_tile(const uint8_t* src, const uint32_t (&xf)[NT][8], int lane,
                                           float (&acc)[NT][4]) {
  const int rho = lane >> 2, c = lane & 3;
  const uint4 a00 = d2_sw128(src, rho, 2 * c), a01 = d2_sw128(src, rho, 2 * c + 1);
  const uint4 a10 = d2_sw128(src, rho + 8, 2 * c), a11 = d2_sw128(src, rho + 8, 2 * c + 1);
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    const uint4& lo0 = s < 2 ? a00 : a01;
    const uint4& lo1 = s < 2 ? a10 : a11;
    const uint32_t af[4] = {d2_w(lo0, (2 * s) & 3), d2_w(lo1, (2 * s) & 3), d2_w(lo0, (2 * s + 1) & 3),
                            d2_w(lo1, (2 * s + 1) & 3)};
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(acc[nt], af, xf[nt][2 * s], xf[nt][2 * s + 1]);
  }
}

// 2S consecutive words of a bf16 row in shared memory (S = 1, 2 or 4).
template <int S>
__device__ __forceinline__ void d2_lds_words(const __nv_bfloat16* p, uint32_t (&w)[8]) {
  if (S == 4) {
    const uint4 v0 = reinterpret_cast<const uint4*>(p)[0], v1 = reinterpret_cast<const uint4*>(p)[1];
    w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w; w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
  } else if (S == 2) {
    const uint4 v0 = *reinterpret_cast<const uint4*>(p);
    w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
  } else {
    const uint2 v0 = *reinterpret_cast<const uint2*>(p);
    w[0] = v0.x; w[1] = v0.y;
  }
}

// acc(16 channels x tokens) += B'[strip rows][0 .. r) . gt[tokens][0 .. r), both
// operands in shared memory (B' rows [16][r], gt [MT][r + 8]).  Lane c feeds 4S
// consecutive columns of each 16S-column chunk; NCH chunks of 64 columns.
template <int MT, int S, int NCH>
__device__ __forceinline__ void d2_ecterm(const __nv_bfloat16* bp, const __nv_bfloat16* gts, int r, int lane,
                                          float (&acc)[MT / 8][4]) {
  constexpr int NT = MT / 8;
  const int rho = lane >> 2, c = lane & 3, gs = r + 8;
#pragma unroll
  for (int ch = 0; ch < NCH; ++ch) {
    uint32_t b0[8], b1[8], g[NT][8];
    d2_lds_words<S>(bp + rho * r + 64 * ch + 4 * S * c, b0);
    d2_lds_words<S>(bp + (rho + 8) * r + 64 * ch + 4 * S * c, b1);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) d2_lds_words<S>(gts + (nt * 8 + rho) * gs + 64 * ch + 4 * S * c, g[nt]);
#pragma unroll
    for (int s = 0; s < S; ++s) {
      const uint32_t af[4] = {b0[2 * s], b1[2 * s], b0[2 * s + 1], b1[2 * s + 1]};
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(acc[nt], af, g[nt][2 * s], g[nt][2 * s + 1]);
    }
  }
}

template <int MT>
__device__ __forceinline__ void d2_ecterm_r(const __nv_bfloat16* bp, const __nv_bfloat16* gts, int r, int lane,
                                            float (&acc)[MT / 8][4]) {
  if (r == 16)
    d2_ecterm<MT, 1, 1>(bp, gts, r, lane, acc);
  else if (r == 32)
    d2_ecterm<MT, 2, 1>(bp, gts, r, lane, acc);
  else if (r == 64)
    d2_ecterm<MT, 4, 1>(bp, gts, r, lane, acc);
  else
    d2_ecterm<MT, 4, 2>(bp, gts, r, lane, acc);
}

// Epilogue of weight strip p: acc is the sum over all of K (fp32, m16n8
// accumulator layout: rows rho / rho + 8, tokens nt*8 + 2c and + 1).  Adds the
// gated EC term, scales by (s0, s1) for rows (rho, rho + 8), rounds to bf16 and
// stores with 16-byte stores through a staging tile ([MT tokens][16 channels]).
template <int MT>
__device__ void d2_store_strip(const D2Args& a, int p, float (&acc)[MT / 8][4], const __nv_bfloat16* bp, float s0,
                               float s1, const __nv_bfloat16* gts, __nv_bfloat16* stage, int lane) {
  constexpr int NT = MT / 8;
  const int rho = lane >> 2, c = lane & 3;
  if (a.ES > 0) d2_ecterm_r<MT>(bp, gts, a.r, lane, acc);
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int t0 = nt * 8 + 2 * c;
    stage[t0 * 16 + rho] = __float2bfloat16_rn(s0 * acc[nt][0]);
    stage[(t0 + 1) * 16 + rho] = __float2bfloat16_rn(s0 * acc[nt][1]);
    stage[t0 * 16 + rho + 8] = __float2bfloat16_rn(s1 * acc[nt][2]);
    stage[(t0 + 1) * 16 + rho + 8] = __float2bfloat16_rn(s1 * acc[nt][3]);
  }
  __syncwarp();
  const int m = lane >> 1, h = lane & 1;
  if (m < a.M && SPEAR_DCHECK(16 * p + 16 <= a.N, a.hdr)) {
    uint4 v = *reinterpret_cast<const uint4*>(stage + m * 16 + 8 * h);
    uint4* dst = reinterpret_cast<uint4*>(a.y + (size_t)m * a.N + 16 * p + 8 * h);
    if (a.ec_only) {
      // y holds the EC-disabled GEMM result: add the EC term in fp32, round once more
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
  __syncwarp();
}

// ---- EC projection words: (fp32 bits, launch tag), single-copy atomic 64-bit stores
__device__ __forceinline__ void d2_st_tagged(unsigned long long* p, float v, uint32_t tag) {
  const unsigned long long w = ((unsigned long long)tag << 32) | __float_as_uint(v);
  asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}
__device__ __forceinline__ void d2_cp16(void* smem_dst, const void* gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gsrc) : "memory");
}

// Copy 16-byte chunks [c0, c1) (stride 32 over the lanes) of the EC projection
// words into shared memory.  Asynchronous: every lane then arrives on `bar`
// when its copies have landed (32 arrivals complete the phase).
__device__ __forceinline__ void d2_ts_fetch(const unsigned long long* tt, unsigned long long* ts, int c0, int c1,
                                            int cstride, uint64_t* bar, int lane) {
  for (int ch = c0 + lane * cstride; ch < c1; ch += 32 * cstride) d2_cp16(ts + 2 * ch, tt + 2 * ch);
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Rank gate (summary section 2.1 A) from the staged projection, one warp:
// u = relu(W1 t + b1), gamma = sigmoid(W2 u + b2), gt[m][j] = bf16(alpha
// gamma_j t[m][j]); padded tokens get zero rows.  Returns, on lane m of CTA 0
// (report), token m's mean of gamma.  Kept out of line so that the scalar-gate
// kernel body, and the inlining of its per-strip code, do not change with it.
template <int MT>
__device__ __noinline__ float d2_rank_gate(const unsigned long long* ts, __nv_bfloat16* gts, float* gsc,
                                           const float* gpar, int M, int r, int h, float alpha, bool report,
                                           int lane) {
  auto tval = [&](int m, int row) {
    return __uint_as_float((uint32_t)ts[((row >> 4) * MT + m) * 16 + (row & 15)]);
  };
  const int gs = r + 8;
  const float* W1 = gpar;              // [h][r]
  const float* W2 = gpar + h * r;      // [r][h]
  const float* B1 = gpar + 2 * h * r;  // [h]
  const float* B2 = B1 + h;            // [r]
  // One warp builds this on every CTA's critical path, so the loops run over
  // the live tokens only and every sum is four independent FMA chains.
  // Hidden activations u[m][i]: M * h pairs; with fewer than 32 pairs, L
  // adjacent lanes share a pair, each summing r / L of its products, and add
  // them by a fixed shuffle tree.
  const int P1 = M * h, r4 = r / 4;
  int L = 1;
  while (L < 4 && P1 * L * 2 <= 32) L *= 2;  // h >= 8, r >= 16: r4 / L >= 1
  const int seg = r4 / L;
  for (int base = 0; base < P1 * L; base += 32) {
    const int idx = base + lane;
    const int p = idx / L, sub = idx - p * L;
    const bool live = p < P1;
    const int m = live ? p / h : 0, i = live ? p - m * h : 0;
    float v0 = 0.f, v1 = 0.f, v2 = 0.f, v3 = 0.f;
    if (live) {
      const float4* w = reinterpret_cast<const float4*>(W1 + i * r) + sub * seg;
      const int j0 = 4 * sub * seg;
#pragma unroll 4
      for (int q4 = 0; q4 < seg; ++q4) {
        const float4 wv = w[q4];
        v0 = fmaf(wv.x, tval(m, j0 + 4 * q4), v0);
        v1 = fmaf(wv.y, tval(m, j0 + 4 * q4 + 1), v1);
        v2 = fmaf(wv.z, tval(m, j0 + 4 * q4 + 2), v2);
        v3 = fmaf(wv.w, tval(m, j0 + 4 * q4 + 3), v3);
      }
    }
    float v = (v0 + v1) + (v2 + v3);
    for (int off = L >> 1; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if (live && sub == 0) gsc[m * 32 + i] = fmaxf(v + B1[i], 0.f);
  }
  __syncwarp();
  // gamma and gt by (token, rank): M * r pairs, a multiple of 16; a batch of
  // 32 pairs holds one token (r >= 32) or two (r = 16)
  float gsum = 0.f;
  for (int base = 0; base < M * r; base += 32) {
    const int idx = base + lane;
    const int m = idx / r, j = idx - m * r;
    float gam = 0.f;
    if (idx < M * r) {
      const float4* w = reinterpret_cast<const float4*>(W2 + j * h);
      const float4* u = reinterpret_cast<const float4*>(gsc + m * 32);
      float z0 = 0.f, z1 = 0.f, z2 = 0.f, z3 = 0.f;
#pragma unroll
      for (int i4 = 0; i4 < 8; ++i4) {
        if (4 * i4 >= h) break;
        const float4 wv = w[i4], uv = u[i4];
        z0 = fmaf(wv.x, uv.x, z0);
        z1 = fmaf(wv.y, uv.y, z1);
        z2 = fmaf(wv.z, uv.z, z2);
        z3 = fmaf(wv.w, uv.w, z3);
      }
      gam = sigmoidf_(B2[j] + ((z0 + z1) + (z2 + z3)));
      gts[m * gs + j] = __float2bfloat16_rn(alpha * gam * tval(m, j));
    }
    if (report) {
      // only CTA 0 reports the gate: this batch's gamma sum per token, by a
      // fixed shuffle tree
      float v = gam;
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1)
        if (off < r) v += __shfl_xor_sync(0xffffffffu, v, off);
      const int m0 = base / r;
      if (r >= 32) {
        if (lane == m0) gsum += v;
      } else {
        const float va = __shfl_sync(0xffffffffu, v, 0), vb = __shfl_sync(0xffffffffu, v, 16);
        if (lane == m0) gsum += va;
        if (lane == m0 + 1) gsum += vb;
      }
    }
  }
  // the padded tokens' rows of gt are zero
  for (int idx = lane; idx < (MT - M) * (r / 2); idx += 32) {
    const int m = M + idx / (r / 2), j = 2 * (idx - (idx / (r / 2)) * (r / 2));
    *reinterpret_cast<uint32_t*>(gts + m * gs + j) = 0u;
  }
  return gsum / (float)r;
}

// Gate and gt from the staged projection (one warp).  Scalar gate:
// g_m = sigmoid(t[m][r] + b_g), gt[m][j] = bf16(g_m t[m][j]); rank gate: see
// d2_rank_gate, with the mean of gamma as the reported gate.  CTA 0 also writes
// the gate outputs and the mask count.
template <int MT>
__device__ void d2_build_gt(const D2Args& a, const unsigned long long* ts, __nv_bfloat16* gts, float* gsc,
                            const float* gpar, int lane) {
  auto tval = [&](int m, int row) {
    return __uint_as_float((uint32_t)ts[((row >> 4) * MT + m) * 16 + (row & 15)]);
  };
  const int gs = a.r + 8;
  float g;  // lane m: token m's gate
  if (a.gate_kind == 1) {
    g = d2_rank_gate<MT>(ts, gts, gsc, gpar, a.M, a.r, a.gate_h, a.alpha, blockIdx.x == 0, lane);
  } else {
    g = lane < MT ? sigmoidf_(tval(lane, a.r) + a.b_g) : 0.f;
    const int half = a.r / 2;
    for (int base = 0; base < MT * half; base += 32) {
      const int idx = base + lane;
      const int m = idx / half;
      const float gm = __shfl_sync(0xffffffffu, g, m < MT ? m : 0);
      if (idx < MT * half) {
        const int j = 2 * (idx - m * half);
        *reinterpret_cast<uint32_t*>(gts + m * gs + j) = pack_bf16x2(gm * tval(m, j), gm * tval(m, j + 1));
      }
    }
  }
  if (blockIdx.x == 0) {
    const bool valid = lane < a.M;
    if (a.gate_out && valid) a.gate_out[lane] = g;
    const unsigned below = __ballot_sync(0xffffffffu, valid && g < a.tau);
    if (a.mask_count && lane == 0) *a.mask_count = __popc(below);
  }
  __syncwarp();
}

template <int MT, int KTW, bool GROUP>
__global__ void __launch_bounds__(D2_THREADS, 2)
    decode2_kernel(const __grid_constant__ D2Args a, const __grid_constant__ CUtensorMap tm_w,
                   const __grid_constant__ CUtensorMap tm_agt, const __grid_constant__ CUtensorMap tm_bp) {
  constexpr int NT = D2T<MT>::NT, ACCS = D2T<MT>::ACCS;
  constexpr int NBUF = d2_nbuf(MT), BJ = d2_bj(MT);
  constexpr int WPU = d2_wpu(KTW), ECU = d2_ecu(KTW) < KTW ? d2_ecu(KTW) : KTW;
  constexpr int UPJ = D2_NWC / WPU;  // units per job and pass
  constexpr int R = KTW / ECU;       // passes over an EC strip (ECU tiles per warp each)
  constexpr unsigned FULL = 0xffffffffu;
  extern __shared__ uint8_t smem_raw[];
  __shared__ int s_abort;
  // 1024-byte aligned base, derived from the shared array itself so that the
  // compiler keeps every access in the shared window (ld/st.shared)
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const D2Smem SL = d2_smem(MT, a.nslot, a.CS, a.own_cap, a.r, a.ES, a.gate_kind, a.gate_h);
  uint8_t* ring = sm + SL.ring;
  float4* red = reinterpret_cast<float4*>(sm + SL.red);
  float4* recv = reinterpret_cast<float4*>(sm + SL.recv);
  float4* park = reinterpret_cast<float4*>(sm + SL.park);
  __nv_bfloat16* bps = reinterpret_cast<__nv_bfloat16*>(sm + SL.bps);
  __half* scs = reinterpret_cast<__half*>(sm + SL.scs);
  unsigned long long* ts = reinterpret_cast<unsigned long long*>(sm + SL.ts);
  __nv_bfloat16* gts = reinterpret_cast<__nv_bfloat16*>(sm + SL.gts);
  float* gsc = reinterpret_cast<float*>(sm + SL.gsc);
  float* gpar = reinterpret_cast<float*>(sm + SL.gpar);
  __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(sm + SL.stage);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + SL.bars);
  uint64_t* empty = full + a.nslot;
  uint64_t* redfull = empty + a.nslot;
  uint64_t* redempty = redfull + NBUF;
  uint64_t* recvbar = redempty + NBUF;
  uint64_t* epibar = recvbar + a.own_cap;
  uint64_t* tsbar = epibar + 1;  // completion of the reducer's cp.async fetches (one arrival per lane)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = a.CS > 1 ? (int)cluster_rank() : 0;
  const short4 ct = a.cl_tab[blockIdx.x / a.CS];
  const int ec_lo = ct.x, n_ec = ct.y, w_lo = ct.z, n_w = ct.w;
  const int n_jobs = n_ec + n_w;                           // items: EC strips, then weight strips
  // jobs (units of synchronisation): one per EC strip, then weight strips in groups of BJ
  const int n_jb = n_ec + (n_w + BJ - 1) / BJ;
  auto job_first = [&](int j) { return j < n_ec ? j : n_ec + (j - n_ec) * BJ; };
  auto job_len = [&](int j) { return j < n_ec ? 1 : min(BJ, n_jobs - (n_ec + (j - n_ec) * BJ)); };
  const int ecU = n_ec * R * UPJ;                          // EC units come first
  const int U = ecU + (a.ec_only ? 0 : n_w * UPJ);
  const bool has_ec = a.ES > 0;
  const int n_own = n_jobs > q ? (n_jobs - q + a.CS - 1) / a.CS : 0;  // jobs i = o * CS + q

  // ring unit u into slot `slot`
  auto issue = [&](int slot, int u) {
    uint64_t* bar = &full[slot];
    const uint32_t dst = smem_u32(ring + (size_t)slot * D2_SLOT);
    if (u < ecU) {
      const int i = u / (R * UPJ), rem = u - i * (R * UPJ), rr = rem / UPJ, g = rem - rr * UPJ;
      mbar_arrive_tx(bar, WPU * ECU * 2048);
#pragma unroll
      for (int wi = 0; wi < WPU; ++wi)
#pragma unroll
        for (int t = 0; t < ECU; ++t) {
          const int kt = q * a.KTP + (g * WPU + wi) * KTW + rr * ECU + t;
          tma_load_2d(dst + (wi * ECU + t) * 2048, &tm_agt, bar, kt * 64, 16 * (ec_lo + i));
        }
    } else {
      const int v = u - ecU, i = n_ec + v / UPJ, g = v - (v / UPJ) * UPJ;
      mbar_arrive_tx(bar, WPU * KTW * 512);
      tma_load_3d(dst, &tm_w, bar, 0, q * a.KTP + g * WPU * KTW, w_lo + (i - n_ec));
    }
  };

  if (warp == 0) {
    for (int s = lane; s < a.nslot; s += 32) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], WPU);
    }
    if (lane < NBUF) {
      mbar_init(&redfull[lane], D2_NWC);
      mbar_init(&redempty[lane], 1);
    }
    for (int o = lane; o < a.own_cap; o += 32) mbar_init(&recvbar[o], 1);
    if (lane == 0) {
      mbar_init(epibar, 1);
      mbar_init(tsbar, 32);
      s_abort = 0;
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    __syncwarp();
    if (a.CS > 1) {
      // partials of the strips this CTA finishes arrive by st.async from the other ranks
      const uint32_t rx = (uint32_t)(a.CS - 1) * NT * 512;
      for (int o = lane; o < n_own; o += 32) {
        const int i = o * a.CS + q;
        if (!(a.ec_only && i >= n_ec)) mbar_arrive_tx(&recvbar[o], rx);
      }
    }
    // epilogue operands of the strips this CTA finishes: B' rows and scales
    int n_epi = 0;
    for (int o = 0; o < n_own; ++o) n_epi += (o * a.CS + q) >= n_ec ? 1 : 0;
    const uint32_t epi_bytes = (uint32_t)n_epi * ((has_ec ? 32u * a.r : 0u) + (GROUP ? 0u : 32u));
    if (lane == 0) {
      if (epi_bytes)
        mbar_arrive_tx(epibar, epi_bytes);
      else
        mbar_arrive(epibar);
    }
    __syncwarp();
    for (int o = lane; o < n_own; o += 32) {
      const int i = o * a.CS + q;
      if (i < n_ec) continue;
      const int p = w_lo + (i - n_ec);
      if (has_ec) tma_load_2d(smem_u32(bps + (size_t)o * 16 * a.r), &tm_bp, epibar, 0, 16 * p);
      if (!GROUP) bulk_g2s(scs + o * 16, a.scales + 16 * p, 32, epibar);
    }
    // the weights and [A^T ; w_g] do not depend on the previous kernel in the
    // stream: the first units go out before the grid-dependency wait.  Only
    // two: a full ring in flight at that point delays the activation load that
    // follows the wait (measured: 15.4 vs 16.2 us per launch at M = 1).
    const int first = U < D2_PRE_UNITS ? U : D2_PRE_UNITS;
    for (int u = lane; u < first; u += 32) issue(u, u);
  }
  __syncthreads();
  if (a.CS > 1) {
    // cluster phase 1: barriers initialised (the producer must not wait here for its loads)
    if (warp == 0)
      asm volatile("barrier.cluster.arrive.relaxed;" ::: "memory");
    else
      asm volatile("barrier.cluster.arrive.release;" ::: "memory");
  }
  // the next kernel in the stream may start (and request its own weights) now
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // x, y and the workspace may belong to the previous kernel in the stream
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (!has_ec && blockIdx.x == 0 && warp == 1) {
    if (a.gate_out && lane < a.M) a.gate_out[lane] = 0.f;
    if (a.mask_count && lane == 0) *a.mask_count = a.M;
  }
  volatile int* abortp = &s_abort;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    // units in order: wait (sleeping) for the slot to drain, lane 0 refills it
    const int first = U < D2_PRE_UNITS ? U : D2_PRE_UNITS;
    int slot = first % a.nslot;
    uint32_t round = first / a.nslot;  // u / nslot
    for (int u = first; u < U; ++u) {
      if (!__all_sync(FULL, d2_wait_polite(&empty[slot], (round & 1) ^ 1, abortp, a.hdr, 256u))) break;
      if (lane == 0) issue(slot, u);
      __syncwarp();
      if (++slot == a.nslot) {
        slot = 0;
        ++round;
      }
    }
    if (a.CS > 1) asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
  } else if (warp <= D2_NWC) {
    // ---------------------------------------------------------------- consumers
    const int w = warp - 1, g = w / WPU, wi = w - g * WPU;
    const int rho = lane >> 2, c = lane & 3;
    // activations of this warp's k slice as B fragments: word i of xf[kt][nt]
    // = x[nt*8 + rho][64 (kt0 + kt) + 16c + 2i .. + 1]
    uint32_t xf[KTW][NT][8];
    const int kt0 = q * a.KTP + w * KTW;
#pragma unroll
    for (int kt = 0; kt < KTW; ++kt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int m = nt * 8 + rho;
        uint4 v0 = make_uint4(0u, 0u, 0u, 0u), v1 = v0;
        if (m < a.M) {
          const uint4* src = reinterpret_cast<const uint4*>(a.x + (size_t)m * a.K + (size_t)(kt0 + kt) * 64 + 16 * c);
          v0 = __ldcg(src);
          v1 = __ldcg(src + 1);
        }
        xf[kt][nt][0] = v0.x; xf[kt][nt][1] = v0.y; xf[kt][nt][2] = v0.z; xf[kt][nt][3] = v0.w;
        xf[kt][nt][4] = v1.x; xf[kt][nt][5] = v1.y; xf[kt][nt][6] = v1.z; xf[kt][nt][7] = v1.w;
      }
    // per-channel codes enter the MMAs as 136 + q: remove 136 * sum(x) of the slice
    // per token (accumulator columns 2c and 2c + 1 of each n8 tile)
    float xsA[NT], xsB[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      xsA[nt] = xsB[nt] = 0.f;
      if (!GROUP) {
        float s = 0.f;
#pragma unroll
        for (int kt = 0; kt < KTW; ++kt)
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xf[kt][nt][i]));
            s += f.x + f.y;
          }
        s += __shfl_xor_sync(FULL, s, 1);
        s += __shfl_xor_sync(FULL, s, 2);
        xsA[nt] = 136.f * __shfl_sync(FULL, s, 8 * c);
        xsB[nt] = 136.f * __shfl_sync(FULL, s, 8 * c + 4);
      }
    }
    if (a.CS > 1) asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
    bool ok = true;
    // this warp's units are g, g + UPJ, g + 2 UPJ, ...: ring slot and phase of the next one
    int cslot = g;
    uint32_t cphase = 0;
    auto next_unit = [&](int& slot, uint32_t& phase) {
      slot = cslot;
      phase = cphase;
      cslot += UPJ;
      if (cslot >= a.nslot) {
        cslot -= a.nslot;
        cphase ^= 1u;
      }
    };
    // one item (an EC strip or a weight strip) of this warp's slice into acc
    auto compute_item = [&](int i, float (&acc)[NT][4]) -> bool {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
      if (i < n_ec) {
        // EC strip: every tile of this warp's slice, ECU tiles per unit
        int slot = 0;
        const uint8_t* src = ring;
#pragma unroll
        for (int kt = 0; kt < KTW; ++kt) {
          if (kt % ECU == 0) {
            uint32_t phase;
            next_unit(slot, phase);
            ok = ok && __all_sync(FULL, d2_wait(&full[slot], phase, abortp, a.hdr));
            src = ring + (size_t)slot * D2_SLOT + wi * ECU * 2048;
          }
          if (ok) d2_ec_tile<NT>(src + (kt % ECU) * 2048, xf[kt], lane, acc);
          if (kt % ECU == ECU - 1) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);
          }
        }
        if (!ok) return false;
      } else {
        int slot;
        uint32_t phase;
        next_unit(slot, phase);
        if (!__all_sync(FULL, d2_wait(&full[slot], phase, abortp, a.hdr))) return false;
        const uint8_t* src = ring + (size_t)slot * D2_SLOT + wi * KTW * 512 + lane * 16;
        if (GROUP) {
          const int p = w_lo + (i - n_ec);
          float sc[KTW][2];
#pragma unroll
          for (int kt = 0; kt < KTW; ++kt) {
            const __half* srow = a.scales + (size_t)((kt0 + kt) >> 1) * a.N + 16 * p + rho;
            sc[kt][0] = __half2float(srow[0]);
            sc[kt][1] = __half2float(srow[8]);
          }
#pragma unroll
          for (int kt = 0; kt < KTW; ++kt) {
            const uint4 wv = *reinterpret_cast<const uint4*>(src + kt * 512);
            float part[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) part[nt][0] = part[nt][1] = part[nt][2] = part[nt][3] = 0.f;
#pragma unroll
            for (int s = 0; s < 4; ++s) {
              uint32_t af[4];
              int4x8_to_bf16x8(d2_w(wv, s), af);
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(part[nt], af, xf[kt][nt][2 * s], xf[kt][nt][2 * s + 1]);
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              acc[nt][0] = fmaf(sc[kt][0], part[nt][0], acc[nt][0]);
              acc[nt][1] = fmaf(sc[kt][0], part[nt][1], acc[nt][1]);
              acc[nt][2] = fmaf(sc[kt][1], part[nt][2], acc[nt][2]);
              acc[nt][3] = fmaf(sc[kt][1], part[nt][3], acc[nt][3]);
            }
          }
        } else {
          // consecutive MMAs go to different accumulator sets (k16 step mod ACCS)
          float accs[ACCS][NT][4];
#pragma unroll
          for (int h = 0; h < ACCS; ++h)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) accs[h][nt][0] = accs[h][nt][1] = accs[h][nt][2] = accs[h][nt][3] = 0.f;
#pragma unroll
          for (int kt = 0; kt < KTW; ++kt) {
            const uint4 wv = *reinterpret_cast<const uint4*>(src + kt * 512);
#pragma unroll
            for (int s = 0; s < 4; ++s) {
              uint32_t af[4];
              d2_nib_biased(d2_w(wv, s), af);
#pragma unroll
              for (int nt = 0; nt < NT; ++nt)
                mma_bf16_16816(accs[s % ACCS][nt], af, xf[kt][nt][2 * s], xf[kt][nt][2 * s + 1]);
            }
          }
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int h = 0; h < ACCS; ++h)
#pragma unroll
              for (int e = 0; e < 4; ++e) acc[nt][e] += accs[h][nt][e];
            acc[nt][0] -= xsA[nt];
            acc[nt][1] -= xsB[nt];
            acc[nt][2] -= xsA[nt];
            acc[nt][3] -= xsB[nt];
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
      }
      return true;
    };
    const int n_jp = a.ec_only ? n_ec : n_jb;  // jobs with weight or EC partials
    for (int j = 0; j < n_jp && ok; ++j) {
      const int t0 = job_first(j), nb = job_len(j);
      float accb[BJ][NT][4];
#pragma unroll
      for (int sb = 0; sb < BJ; ++sb)
        if (sb < nb && ok) ok = compute_item(t0 + sb, accb[sb]);
      if (!ok) break;
      // the partials go to the reducer warp through buffer b
      const int b = j % NBUF, k = j / NBUF;
      if (!__all_sync(FULL, d2_wait(&redempty[b], (k & 1) ^ 1, abortp, a.hdr))) break;
#pragma unroll
      for (int sb = 0; sb < BJ; ++sb)
        if (sb < nb) {
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            red[(((b * D2_NWC + w) * BJ + sb) * NT + nt) * 32 + lane] =
                make_float4(accb[sb][nt][0], accb[sb][nt][1], accb[sb][nt][2], accb[sb][nt][3]);
        }
      __syncwarp();
      if (lane == 0) mbar_arrive(&redfull[b]);
    }
  } else {
    // ---------------------------------------------------------------- reducer
    // Sums the warp partials of every job in warp order, exchanges CTA partials
    // within the cluster (rank order), publishes EC strips, fetches the whole EC
    // projection without blocking, and runs (or parks) the strip epilogues.
    const int rho = lane >> 2, c = lane & 3;
    if (a.gate_kind == 1) {
      // rank-gate parameters into shared memory while the first partials are
      // computed (all four arrays have a multiple of 4 floats, 16-byte aligned)
      const int h = a.gate_h, r = a.r;
      auto stage4 = [&](const float* src, float* dst, int n) {
        for (int i = lane; i < n / 4; i += 32)
          reinterpret_cast<float4*>(dst)[i] = __ldg(reinterpret_cast<const float4*>(src) + i);
      };
      stage4(a.gw1, gpar, h * r);
      stage4(a.gw2, gpar + h * r, r * h);
      stage4(a.gb1, gpar + 2 * h * r, h);
      stage4(a.gb2, gpar + 2 * h * r + h, r);
      __syncwarp();
    }
    if (a.CS > 1) asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
    const uint32_t tag = (uint32_t)(*reinterpret_cast<volatile int*>(&a.hdr->d2_epoch)) + 1u;
    // EC projection state: 0 idle, 1 probe in flight, 2 full fetch in flight, 3 gate and gt ready.
    // Fetches complete on tsbar (phase = fetch count); nothing here blocks.
    int gst = has_ec ? 0 : 3, nfetch = 0;
    int obs_prev = -1;
    uint32_t parked = 0;
    bool epi_ready = false, ok = true;
    const int words = a.ES * MT * 16;
    auto gt_step = [&]() {
      if (gst == 1 || gst == 2) {
        if (!__all_sync(FULL, mbar_test(tsbar, (nfetch - 1) & 1))) return;  // still in flight
        bool tok = true;
        if (gst == 1) {
          // probe: the last 16 bytes of every EC strip
          if (lane < a.ES) {
            const int ch = (lane * MT + MT - 1) * 8 + 7;
            tok = (uint32_t)(ts[2 * ch] >> 32) == tag && (uint32_t)(ts[2 * ch + 1] >> 32) == tag;
          }
        } else {
          for (int i = lane; i < words; i += 32) tok = tok && (uint32_t)(ts[i] >> 32) == tag;
        }
        tok = __all_sync(FULL, tok);
        if (tok && gst == 2) {
          d2_build_gt<MT>(a, ts, gts, gsc, gpar, lane);
          gst = 3;
          // every CTA reads the projection once; the last reader advances the epoch
          if (lane == 0) obs_prev = atomicAdd(&a.hdr->gt_obs, 1);
          return;
        }
        if (tok) {
          d2_ts_fetch(a.tt, ts, 0, words / 2, 1, tsbar, lane);
          ++nfetch;
          gst = 2;
          return;
        }
        gst = 0;
      }
      if (gst == 0) {
        // probe chunk of EC strip e: (e * MT + MT - 1) * 8 + 7 = 8 MT e + 8 MT - 1
        d2_ts_fetch(a.tt, ts, 8 * MT - 1, a.ES * 8 * MT, 8 * MT, tsbar, lane);
        ++nfetch;
        gst = 1;
      }
    };
    // warp-uniform wait that keeps the projection fetch moving
    auto rwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      if (__all_sync(FULL, mbar_test(bar, parity))) return true;
      const long long t0 = clock64();
      uint32_t ns = 32;
      while (true) {
        __nanosleep(ns);
        ns = ns < 256 ? ns * 2 : 256;
        const bool d = mbar_test(bar, parity);
        if (__all_sync(FULL, d)) return true;
        int stop = 0;
        if (lane == 0) {
          if (*abortp) {
            stop = 1;
          } else if (clock64() - t0 > kWaitCycles) {
            report_status(a.hdr, SPEAR_ERR_TIMEOUT);
            *abortp = 1;
            stop = 1;
          }
        }
        if (__shfl_sync(FULL, stop, 0)) return false;
        if (gst < 3) gt_step();
      }
    };
    auto epilogue = [&](int o, float (&tot)[NT][4]) {
      if (!epi_ready) {
        ok = rwait(epibar, 0);
        epi_ready = true;
        if (!ok) return;
      }
      const int p = w_lo + (o * a.CS + q - n_ec);
      float s0 = 1.f, s1 = 1.f;
      if (!GROUP) {
        s0 = __half2float(scs[o * 16 + rho]);
        s1 = __half2float(scs[o * 16 + rho + 8]);
      }
      d2_store_strip<MT>(a, p, tot, bps + (size_t)o * 16 * a.r, s0, s1, gts, stage, lane);
    };
    auto flush_parked = [&]() {
      while (parked && ok) {
        const int o = __ffs(parked) - 1;
        parked &= parked - 1;
        float tot[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const float4 v = park[(o * NT + nt) * 32 + lane];
          tot[nt][0] = v.x;
          tot[nt][1] = v.y;
          tot[nt][2] = v.z;
          tot[nt][3] = v.w;
        }
        epilogue(o, tot);
      }
    };

    // a finished sum of job i: publish an EC strip, run or park a strip epilogue
    auto finalize = [&](int i, float (&tot)[NT][4]) {
      const int o = i / a.CS;
      if (i < n_ec) {
        // the reduced rows of EC strip e: [MT tokens][16 rows] tagged words
        unsigned long long* dst = a.tt + (size_t)(ec_lo + i) * MT * 16;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int t0 = nt * 8 + 2 * c;
          d2_st_tagged(dst + t0 * 16 + rho, tot[nt][0], tag);
          d2_st_tagged(dst + (t0 + 1) * 16 + rho, tot[nt][1], tag);
          d2_st_tagged(dst + t0 * 16 + rho + 8, tot[nt][2], tag);
          d2_st_tagged(dst + (t0 + 1) * 16 + rho + 8, tot[nt][3], tag);
        }
        return;
      }
      if (gst == 3) {
        flush_parked();
        epilogue(o, tot);
      } else {
        // gt not in yet: park the reduced strip
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          park[(o * NT + nt) * 32 + lane] = make_float4(tot[nt][0], tot[nt][1], tot[nt][2], tot[nt][3]);
        __syncwarp();
        parked |= 1u << o;
      }
    };
    // Owned jobs whose own partial waits in park[o] for the other ranks'
    // partials: finish those that have arrived (or wait for all of them).
    uint32_t pending = 0;
    auto finish_pending = [&](bool block) {
      uint32_t m = pending;
      while (m && ok) {
        const int o = __ffs(m) - 1;
        m &= m - 1;
        if (block) {
          if (!rwait(&recvbar[o], 0)) {
            ok = false;
            return;
          }
        } else if (!__all_sync(FULL, mbar_test(&recvbar[o], 0))) {
          continue;
        }
        pending &= ~(1u << o);
        float tot[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) tot[nt][0] = tot[nt][1] = tot[nt][2] = tot[nt][3] = 0.f;
        for (int q2 = 0; q2 < a.CS; ++q2) {
          const int sidx = q2 - (q2 > q ? 1 : 0);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const float4 v = q2 == q ? park[(o * NT + nt) * 32 + lane]
                                     : recv[((o * (a.CS - 1) + sidx) * NT + nt) * 32 + lane];
            tot[nt][0] += v.x;
            tot[nt][1] += v.y;
            tot[nt][2] += v.z;
            tot[nt][3] += v.w;
          }
        }
        __syncwarp();
        finalize(o * a.CS + q, tot);
      }
    };

    for (int j = 0; j < n_jb && ok; ++j) {
      if (gst < 3) gt_step();
      const int t0 = job_first(j), nb = job_len(j);
      const bool has_part = !(a.ec_only && j >= n_ec);
      const int b = j % NBUF, k = j / NBUF;
      if (has_part && !rwait(&redfull[b], k & 1)) {
        ok = false;
        break;
      }
      for (int sb = 0; sb < nb; ++sb) {
        const int i = t0 + sb;  // item
        const int owner = i % a.CS, o = i / a.CS;
        const bool mine = owner == q;
        float tot[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) tot[nt][0] = tot[nt][1] = tot[nt][2] = tot[nt][3] = 0.f;
        if (has_part) {
          for (int w2 = 0; w2 < D2_NWC; ++w2)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              const float4 v = red[(((b * D2_NWC + w2) * BJ + sb) * NT + nt) * 32 + lane];
              tot[nt][0] += v.x;
              tot[nt][1] += v.y;
              tot[nt][2] += v.z;
              tot[nt][3] += v.w;
            }
          if (a.CS > 1) {
            if (!mine) {
              // this CTA's partial to the owner, which adds the ranks in order
              const int sidx = q - (q > owner ? 1 : 0);
              const uint32_t rbar = map_rank(smem_u32(&recvbar[o]), owner);
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) {
                const uint32_t dst =
                    map_rank(smem_u32(recv + ((o * (a.CS - 1) + sidx) * NT + nt) * 32 + lane), owner);
                st_async_f4(dst, make_float4(tot[nt][0], tot[nt][1], tot[nt][2], tot[nt][3]), rbar);
              }
            } else {
#pragma unroll
              for (int nt = 0; nt < NT; ++nt)
                park[(o * NT + nt) * 32 + lane] = make_float4(tot[nt][0], tot[nt][1], tot[nt][2], tot[nt][3]);
              __syncwarp();
              pending |= 1u << o;
            }
            continue;
          }
        } else if (!mine) {
          continue;
        }
        finalize(i, tot);
        if (!ok) break;
      }
      if (has_part) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&redempty[b]);
      }
      if (a.CS > 1) finish_pending(false);
    }
    if (ok) finish_pending(true);
    if (ok && has_ec) {
      // the rest of the projection (bounded), then the parked strips
      const long long t0 = clock64();
      while (gst < 3) {
        gt_step();
        if (gst == 3) break;
        int stop = 0;
        if (lane == 0) {
          if (*abortp) {
            stop = 1;
          } else if (clock64() - t0 > kWaitCycles) {
            report_status(a.hdr, SPEAR_ERR_TIMEOUT);
            *abortp = 1;
            stop = 1;
          }
        }
        if (__shfl_sync(FULL, stop, 0)) {
          ok = false;
          break;
        }
        __nanosleep(256);
      }
      flush_parked();
      if (lane == 0 && obs_prev == a.G - 1) {
        a.hdr->gt_obs = 0;
        a.hdr->d2_epoch = (int)tag;
      }
    }
  }
  // no CTA of the cluster leaves while st.async writes into it may be in flight.
  // Lifetime only: nothing is read after the barrier, so the arrival is relaxed
  // and does not wait for this thread's global stores (a release would).
  if (a.CS > 1) asm volatile("barrier.cluster.arrive.relaxed;\n\tbarrier.cluster.wait;" ::: "memory");
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
struct D2Plan {
  int MT, CS, NC, KTP, KTW, ES, nslot, own_cap;
  size_t smem;
  const char* why;            // non-null: the decode kernel cannot run this shape
  std::vector<short4> cl_tab;
};

template <int MT, int KTW, bool GROUP>
static cudaError_t d2_attrs(size_t smem) {
  static std::mutex mu;
  static size_t opted = 0;
  std::lock_guard<std::mutex> lk(mu);
  if (smem <= opted) return cudaSuccess;
  cudaError_t e =
      cudaFuncSetAttribute(decode2_kernel<MT, KTW, GROUP>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // two CTAs per SM need the largest shared-memory carve-out
  e = cudaFuncSetAttribute(decode2_kernel<MT, KTW, GROUP>, cudaFuncAttributePreferredSharedMemoryCarveout,
                           (int)cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  opted = smem;
  return cudaSuccess;
}

static D2Plan make_d2_plan(int MT, int K, int N, int r, int sms, int gate_kind, int gate_h, int nc_cap) {
  D2Plan p = {};
  p.MT = MT;
  p.why = nullptr;
  const int KT = K / 64;
  if (K % (64 * D2_NWC)) {
    p.why = "K must be a multiple of 256";
    return p;
  }
  // warp slice: the largest power of two <= 8 dividing K / (64 * warps)
  const int SW = KT / D2_NWC;
  int ktw = 1;
  for (int d = D2_KTW_MAX; d >= 1; d /= 2)
    if (SW % d == 0) {
      ktw = d;
      break;
    }
  p.KTW = ktw;
  p.CS = SW / ktw;
  if (p.CS > 8) {
    p.why = "K too large for the decode kernel's cluster";
    return p;
  }
  p.KTP = KT / p.CS;
  p.ES = r > 0 ? (r + 1 + 15) / 16 : 0;
  const int NS = N / 16;
  // two CTAs per SM per launch: the next launch takes an SM's halves as this
  // one leaves them (measured faster than one CTA per SM beside the next
  // launch); never more clusters than can be resident at once (nc_cap), since
  // every CTA waits for the EC strips of other clusters
  int NC = std::max(1, std::min(2 * sms / p.CS, nc_cap));
  NC = std::min(NC, std::max(1, NS + p.ES));
  NC = std::min(NC, D2_MAXCL);
  p.NC = NC;
  // balance bytes per cluster: a weight strip streams KTW int4 tiles (512 B) per
  // warp, an EC strip KTW bf16 tiles (2 KB) per warp
  const long long cw = 1, ce = 4;
  const long long C = (long long)p.ES * ce + (long long)NS * cw;
  std::vector<int> eb(NC + 1), wb(NC + 1);
  for (int c = 0; c <= NC; ++c) eb[c] = (int)(((long long)c * p.ES + NC - 1) / NC);
  wb[0] = 0;
  for (int c = 1; c < NC; ++c) {
    const long long s = C * c / NC - (long long)eb[c] * ce;
    long long v = std::max<long long>(s, wb[c - 1]);
    wb[c] = (int)std::min<long long>(v, NS);
  }
  wb[NC] = NS;
  p.cl_tab.resize(NC);
  int own = 1;
  for (int c = 0; c < NC; ++c) {
    const int ne = eb[c + 1] - eb[c], nw = wb[c + 1] - wb[c];
    p.cl_tab[c] = make_short4((short)eb[c], (short)ne, (short)wb[c], (short)nw);
    own = std::max(own, (ne + nw + p.CS - 1) / p.CS);
  }
  p.own_cap = own;
  if (own > D2_MAXOWN) {
    p.why = "too many strips per CTA for the decode kernel";
    return p;
  }
  const D2Smem s0 = d2_smem(MT, 0, p.CS, own, r, p.ES, gate_kind, gate_h);
  const size_t per_slot = D2_SLOT + 16;
  p.nslot = (int)std::min<size_t>(D2_MAXSLOT, (D2_SMEM_CAP - std::min<size_t>(s0.total, D2_SMEM_CAP)) / per_slot);
  if (p.nslot < 3) {
    p.why = "shared memory too small for the decode kernel's ring";
    return p;
  }
  p.smem = d2_smem(MT, p.nslot, p.CS, own, r, p.ES, gate_kind, gate_h).total;
  return p;
}

// Clusters of this kernel instance that fit on the device at once (cluster
// size CS, `smem` bytes each); 0 if the query fails.
template <int MT, int KTW>
static int d2_max_clusters_t(int CS, size_t smem) {
  if (d2_attrs<MT, KTW, false>(smem) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  int n = 0;
  if (CS == 1) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode2_kernel<MT, KTW, false>, D2_THREADS, smem) !=
        cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    return per_sm * device_sm_count();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CS);
  cfg.blockDim = dim3(D2_THREADS);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeClusterSchedulingPolicyPreference;
  attr[1].val.clusterSchedulingPolicyPreference = cudaClusterSchedulingPolicySpread;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (cudaOccupancyMaxActiveClusters(&n, decode2_kernel<MT, KTW, false>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

static int d2_max_clusters(int MT, int KTW, int CS, size_t smem) {
  if (MT == 8) {
    switch (KTW) {
      case 8: return d2_max_clusters_t<8, 8>(CS, smem);
      case 4: return d2_max_clusters_t<8, 4>(CS, smem);
      case 2: return d2_max_clusters_t<8, 2>(CS, smem);
      default: return d2_max_clusters_t<8, 1>(CS, smem);
    }
  }
  switch (KTW) {
    case 8: return d2_max_clusters_t<16, 8>(CS, smem);
    case 4: return d2_max_clusters_t<16, 4>(CS, smem);
    case 2: return d2_max_clusters_t<16, 2>(CS, smem);
    default: return d2_max_clusters_t<16, 1>(CS, smem);
  }
}

// The plan for a shape, with its clusters capped at what is resident at once.
static const D2Plan& d2_plan(int MT, int K, int N, int r, int sms, int gate_kind, int gate_h) {
  static std::mutex mu;
  static std::map<std::tuple<int, int, int, int, int, int, int, int>, D2Plan> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  const int gh = gate_kind ? gate_h : 0;
  const auto key = std::make_tuple(dev, MT, K, N, r, sms, gate_kind, gh);
  std::lock_guard<std::mutex> lk(mu);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  D2Plan p = make_d2_plan(MT, K, N, r, sms, gate_kind, gh, 1 << 30);
  // fewer clusters give each more strips (more shared memory), which does not
  // change residency while a CTA stays within the two-per-SM cap; re-check anyway
  for (int iter = 0; !p.why; ++iter) {
    const int mc = d2_max_clusters(MT, p.KTW, p.CS, p.smem);
    if (mc <= 0) {
      p.why = "cluster occupancy query failed for the decode kernel";
    } else if (p.NC > mc) {
      if (iter == 3)
        p.why = "the decode kernel's clusters do not fit on the device at once";
      else
        p = make_d2_plan(MT, K, N, r, sms, gate_kind, gh, mc);
    } else {
      break;
    }
  }
  return cache.emplace(key, std::move(p)).first->second;
}

size_t decode2_tt_bytes(int r) {
  const int ES = r > 0 ? (r + 1 + 15) / 16 : 0;
  return (size_t)ES * 16 * 16 * 8;
}

const char* decode2_unsupported(int M, int K, int N, int r, int gate_kind, int gate_h) {
  if (M < 1 || M > 16) return "the decode kernel needs 1 <= M <= 16";
  return d2_plan(M <= 8 ? 8 : 16, K, N, r, device_sm_count(), gate_kind, gate_h).why;
}

template <int MT, int KTW, bool GROUP>
static int d2_launch_t(const D2Args& a, const CUtensorMap* maps, size_t smem, cudaStream_t st) {
  cudaError_t e = d2_attrs<MT, KTW, GROUP>(smem);
  if (e != cudaSuccess) return set_cuda_error("cudaFuncSetAttribute(decode)", e);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.NC * a.CS);
  cfg.blockDim = dim3(D2_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[3];
  int na = 0;
  // programmatic dependent launch: this grid may start while the previous
  // kernel in the stream drains; it waits for it before touching x, y, ws
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  if (a.CS > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = a.CS;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
    // one CTA of this launch per SM: the other half of each SM is for the next launch
    attr[na].id = cudaLaunchAttributeClusterSchedulingPolicyPreference;
    attr[na].val.clusterSchedulingPolicyPreference = cudaClusterSchedulingPolicySpread;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  e = cudaLaunchKernelEx(&cfg, decode2_kernel<MT, KTW, GROUP>, a, maps[0], maps[1], maps[2]);
  if (e != cudaSuccess) return set_cuda_error("decode launch", e);
  return SPEAR_OK;
}

template <int MT, int KTW>
static int d2_dispatch_g(bool group, const D2Args& a, const CUtensorMap* maps, size_t smem, cudaStream_t st) {
  return group ? d2_launch_t<MT, KTW, true>(a, maps, smem, st) : d2_launch_t<MT, KTW, false>(a, maps, smem, st);
}

template <int MT>
static int d2_dispatch_k(int ktw, bool group, const D2Args& a, const CUtensorMap* maps, size_t smem,
                         cudaStream_t st) {
  switch (ktw) {
    case 8: return d2_dispatch_g<MT, 8>(group, a, maps, smem, st);
    case 4: return d2_dispatch_g<MT, 4>(group, a, maps, smem, st);
    case 2: return d2_dispatch_g<MT, 2>(group, a, maps, smem, st);
    default: return d2_dispatch_g<MT, 1>(group, a, maps, smem, st);
  }
}

int launch_decode2(const LayerView& Lv, const __nv_bfloat16* x, int M, __nv_bfloat16* y, WsHeader* hdr, void* tt,
                   float* gate_out, int* mask_count, bool ec_only, cudaStream_t st) {
  if (M < 1 || M > 16) return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "decode path needs 1 <= M <= 16 (M=%d)", M);
  const int MT = M <= 8 ? 8 : 16;
  const int gk = Lv.r > 0 ? Lv.gate_kind : 0;
  const D2Plan& p = d2_plan(MT, Lv.K, Lv.N, Lv.r, device_sm_count(), gk, Lv.gate_h);
  if (p.why) return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "decode path: %s", p.why);
  if (ec_only && Lv.r == 0) return set_error(SPEAR_ERR_INVALID_ARG, "EC-only launch without an EC");
  D2Args a = {};
  a.scales = Lv.scales;
  a.x = x;
  a.y = y;
  a.gate_out = gate_out;
  a.mask_count = mask_count;
  a.hdr = hdr;
  a.tt = static_cast<unsigned long long*>(tt);
  a.M = M;
  a.K = Lv.K;
  a.N = Lv.N;
  a.r = Lv.r;
  a.group = Lv.group;
  a.b_g = Lv.b_g;
  a.tau = Lv.tau;
  a.CS = p.CS;
  a.NC = p.NC;
  a.G = p.NC * p.CS;
  a.KTP = p.KTP;
  a.ES = Lv.r > 0 ? p.ES : 0;
  a.nslot = p.nslot;
  a.own_cap = p.own_cap;
  a.ec_only = ec_only ? 1 : 0;
  a.gate_kind = gk;
  a.gate_h = Lv.gate_h;
  a.gw1 = Lv.gw1;
  a.gb1 = Lv.gb1;
  a.gw2 = Lv.gw2;
  a.gb2 = Lv.gb2;
  a.alpha = Lv.alpha;
  for (int c = 0; c < p.NC; ++c) a.cl_tab[c] = p.cl_tab[c];
  CUtensorMap maps[3];
  memset(maps, 0, sizeof(maps));
  bool ok = tmap_packed_box(&maps[0], Lv.w, Lv.K, Lv.N, d2_wpu(p.KTW) * p.KTW, 1);
  if (ok && a.ES > 0) ok = tmap_2d_bf16(&maps[1], Lv.agt, Lv.K, Lv.r + 1, 64, 16);
  if (ok && a.ES > 0) ok = tmap_2d_bf16(&maps[2], Lv.bpt, Lv.r, Lv.N, Lv.r, 16, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!ok) return set_error(SPEAR_ERR_CUDA, "cuTensorMapEncodeTiled failed (decode)");
  return MT == 8 ? d2_dispatch_k<8>(p.KTW, Lv.group != 0, a, maps, p.smem, st)
                 : d2_dispatch_k<16>(p.KTW, Lv.group != 0, a, maps, p.smem, st);
}

}  // namespace spear
