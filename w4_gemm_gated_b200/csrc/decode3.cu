// Decode path (1 <= M <= 16) on sm_100a: W4 GEMV with the gated EC fused,
// laid out so that no single warp serialises the work of its CTA.
//
// SPEAR fuses the whole EC computation into the low-bit GEMM for the
// memory-bound decode phase (gist.science technical summary, section 2.2 A,
// decode at M = 1: one kernel, no inter-kernel launch on the critical path).
//
// Work.  K is cut into CS <= 2 parts, one per CTA of a cluster; each part
// into 8 warp slices of CH 64-wide k-tiles (CH <= 4), whose activations a
// consumer warp holds in registers as mma.sync B fragments for the whole
// launch.  A cluster owns a run of items, the same run for both of its CTAs:
//   - at most one EC item, first: a 16-row strip of A^T, or the gate row w_g
//     (scalar gate), both read from [A^T ; w_g];
//   - then 16-channel weight strips.
// Items are balanced over the clusters by the bytes they stream.
//
// Streaming.  One producer warp fills a ring of 16-17 KB units by TMA: a
// weight strip's K part (with its group scales), or one k-tile per warp of an
// EC strip.  Nothing here depends on the previous kernel in the stream, so the
// whole ring is requested before the grid-dependency wait.  With one CTA per
// SM and at most 112 KB of shared memory, the next launch's CTA fits beside
// this one and fills its own ring while this one computes.
//
// Reduction, in a fixed order (deterministic).  Each consumer warp writes its
// partial of an item into one of two shared buffers; the warp whose turn it is
// (item index mod 8) adds the 8 partials in warp order one item later, so the
// reduction work rotates over the warps.  With CS = 2 the non-owner CTA of an
// item (item index mod 2) sends its partial to the owner by st.async into the
// owner's shared memory.
//
// EC.  The owner of an EC item adds the two K parts and publishes the rows of
// t = x . A (or the gate logit x . w_g) for the live tokens to the workspace,
// then raises that item's flag to this launch's tag.  The producer warp, once
// its last unit is issued, waits for every flag and loads t.  At the end all
// warps build g and gt = bf16(g t) (or the pages' per-rank gate) in shared
// memory and finish the owned strips: y = bf16(s (acc + gt . B')), 16-byte
// stores.
//
// Every wait is bounded; a timeout is reported in the workspace status word
// and every role falls through to the end (no early exit while copies or
// cluster stores may be in flight).
#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include "common.cuh"
#include "kernels.h"
#include "tma.cuh"

namespace spear {

constexpr int D3_NW = 8;                       // consumer warps
constexpr int D3_THREADS = (D3_NW + 1) * 32;   // + the producer warp
constexpr int D3_NB = 2;                       // partial buffers
constexpr int D3_MAXCL = 160;                  // clusters described in the kernel parameters
constexpr int D3_MAXOWN = 24;                  // items one CTA finishes per launch
constexpr int D3_MAXE = 9;                     // EC items: 8 strips of A^T (r <= 128) + the gate row

struct D3Args {
  const __half* scales;
  const __nv_bfloat16* x;
  __nv_bfloat16* y;
  float* gate_out;
  int* mask_count;
  WsHeader* hdr;
  float* tf;                // [D3_MAXE][MT][16] fp32: published EC rows (t, then the gate logit in row 0)
  const float *gw1, *gb1, *gw2, *gb2;
  int M, K, N, r;
  float b_g, tau, alpha;
  int CS, G;                // cluster size (= K parts), CTAs
  int KTC;                  // k-tiles per CTA (8 * CH)
  int ES;                   // strips of A^T (r / 16); 0 with the EC off
  int gate_item;            // 1: the gate row w_g is an EC item (scalar gate)
  int nslot, slot, own_cap;
  int ec_only;              // 1: no weights; y += EC term in place (unfused path)
  int gate_kind, gate_h;
  int tag_skew;             // test injection: publication flags are awaited at tag + skew (0 normally)
  long long pub_wait;       // bound of that wait (SM cycles)
  short4 cl_tab[D3_MAXCL];  // per cluster: EC item (-1 none), first weight strip, weight strips, 0
};

// Shared-memory carve-up (same on host and device).
struct D3Smem {
  uint32_t ring, red, park, recv, bps, scs, ts, gts, gv, stage, bars, total;
};
// Reduction buffers are idle in the end phase: the epilogue staging tiles and
// gt live there then.
__host__ __device__ __forceinline__ uint32_t d3_red_bytes(int MT, int r) {
  const uint32_t red = D3_NB * D3_NW * (MT / 8) * 512;
  const uint32_t end = (D3_NW + 1) * MT * 32 + (r > 0 ? (uint32_t)MT * (r + 8) * 2 : 0u);
  return red > end ? red : end;
}
__host__ __device__ __forceinline__ uint32_t d3_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }
__host__ __device__ __forceinline__ D3Smem d3_smem(int MT, int nslot, int slot, int CS, int own_cap, int r) {
  D3Smem s;
  const uint32_t NT = MT / 8;
  uint32_t off = 0;
  s.ring = off;
  off += nslot * slot;
  s.red = off;  // [NB][8 warps][NT][32 lanes] float4; in the end phase: staging tiles, then gt
  s.stage = off;  // per warp [MT tokens][16 channels] bf16
  s.gts = off + (D3_NW + 1) * MT * 32;  // gt [MT][r + 8] bf16
  off += d3_up(d3_red_bytes(MT, r), 128);
  s.park = off;  // own partials of the owned items [own][NT][32] float4
  off += own_cap * NT * 512;
  s.recv = off;  // the other rank's partials [own][NT][32] float4
  off += CS > 1 ? own_cap * NT * 512 : 0;
  s.bps = off;  // B' rows of the owned strips [own][16][r] bf16
  off += d3_up(own_cap * 32 * r, 128);
  s.scs = off;  // per-channel scales of the owned strips [own][16] fp16
  off += d3_up(own_cap * 32, 16);
  s.ts = off;  // t [MT][r] fp32, then the gate logits [MT]
  off += r > 0 ? d3_up((MT * r + MT) * 4, 16) : 0;
  s.gv = off;  // per-token gate g (fp32) [MT]
  off += 64;
  s.bars = off;
  off += (2 * nslot + 2 * D3_NB + own_cap + 2) * 8 + 16;
  s.total = off + 1024;  // base alignment slack
  return s;
}

__device__ __forceinline__ uint32_t d3_w(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// 8 nibbles -> 4 bf16x2 holding 128 + u (exact): register pi = nibbles (pi, pi + 4)
__device__ __forceinline__ void d3_nib_biased(uint32_t w, uint32_t (&o)[4]) {
#pragma unroll
  for (int pi = 0; pi < 4; ++pi) {
    uint32_t v;
    asm("lop3.b32 %0, %1, %2, %3, 0xea;" : "=r"(v) : "r"(w >> (4 * pi)), "r"(0x000F000Fu), "r"(0x43004300u));
    o[pi] = v;
  }
}

// Bounded spin on an mbarrier phase.  False after a timeout (reported) or once
// another role has given up.
__device__ __forceinline__ bool d3_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, WsHeader* h) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  for (int it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31) == 0) {
      if (*abort_flag) return false;
      if (clock64() - t0 > kWaitCycles) {
        report_status(h, SPEAR_ERR_TIMEOUT);
        *abort_flag = 1;
        return false;
      }
    }
  }
}

// Bounded wait that sleeps between tests (for the producer warp, which must
// not take issue slots from the consumers).
__device__ __forceinline__ bool d3_wait_sleep(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                              WsHeader* h) {
  if (mbar_test(bar, parity)) return true;
  const long long t0 = clock64();
  uint32_t ns = 32;
  while (true) {
    __nanosleep(ns);
    if (mbar_test(bar, parity)) return true;
    ns = ns < 256 ? ns * 2 : 256;
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitCycles) {
      report_status(h, SPEAR_ERR_TIMEOUT);
      *abort_flag = 1;
      return false;
    }
  }
}

// Wait, bounded and without reporting, for copies already issued into this
// CTA's shared memory (used before exit after another role gave up).
__device__ __forceinline__ void d3_drain(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > kWaitCycles) break;
}

// Swizzled 128-byte-row tile (TMA SWIZZLE_128B): 16-byte chunk ch of row r.
__device__ __forceinline__ uint4 d3_sw128(const uint8_t* tile, int row, int ch) {
  return *reinterpret_cast<const uint4*>(tile + row * 128 + ((ch ^ (row & 7)) << 4));
}

// One EC tile: 16 rows of A^T x 64 k (bf16, SW128) against the activations of
// the same k-tile.  Lane (rho, c) feeds k [16c, 16c + 16) of rows rho and
// rho + 8, the k order the activation fragments use.
template <int NT>
__device__ __forceinline__ void d3_ec_tile(const uint8_t* src, const uint32_t (&xf)[NT][8], int lane,
                                           float (&acc)[NT][4]) {
  const int rho = lane >> 2, c = lane & 3;
  const uint4 a00 = d3_sw128(src, rho, 2 * c), a01 = d3_sw128(src, rho, 2 * c + 1);
  const uint4 a10 = d3_sw128(src, rho + 8, 2 * c), a11 = d3_sw128(src, rho + 8, 2 * c + 1);
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    const uint4& lo0 = s < 2 ? a00 : a01;
    const uint4& lo1 = s < 2 ? a10 : a11;
    const uint32_t af[4] = {d3_w(lo0, (2 * s) & 3), d3_w(lo1, (2 * s) & 3), d3_w(lo0, (2 * s + 1) & 3),
                            d3_w(lo1, (2 * s + 1) & 3)};
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(acc[nt], af, xf[nt][2 * s], xf[nt][2 * s + 1]);
  }
}

// The gate row as the only live row of a 16-row MMA operand: tile t of this
// warp's slice holds row w_g, k [64 t, 64 t + 64) unswizzled (128 bytes);
// lanes of rows 1..15 feed zeros.  Row 0 of acc receives x . w_g.
template <int NT>
__device__ __forceinline__ void d3_gate_tile(const uint8_t* src, const uint32_t (&xf)[NT][8], int lane,
                                             float (&acc)[NT][4]) {
  const int rho = lane >> 2, c = lane & 3;
  uint4 lo = make_uint4(0u, 0u, 0u, 0u), hi = lo;
  if (rho == 0) {
    lo = *reinterpret_cast<const uint4*>(src + 32 * c);
    hi = *reinterpret_cast<const uint4*>(src + 32 * c + 16);
  }
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    const uint4& v = s < 2 ? lo : hi;
    const uint32_t af[4] = {d3_w(v, (2 * s) & 3), 0u, d3_w(v, (2 * s + 1) & 3), 0u};
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(acc[nt], af, xf[nt][2 * s], xf[nt][2 * s + 1]);
  }
}

// 2S consecutive words of a bf16 row in shared memory (S = 1, 2 or 4).
template <int S>
__device__ __forceinline__ void d3_lds_words(const __nv_bfloat16* p, uint32_t (&w)[8]) {
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
__device__ __forceinline__ void d3_ecterm(const __nv_bfloat16* bp, const __nv_bfloat16* gts, int r, int lane,
                                          float (&acc)[MT / 8][4]) {
  constexpr int NT = MT / 8;
  const int rho = lane >> 2, c = lane & 3, gs = r + 8;
#pragma unroll
  for (int ch = 0; ch < NCH; ++ch) {
    uint32_t b0[8], b1[8], g[NT][8];
    d3_lds_words<S>(bp + rho * r + 64 * ch + 4 * S * c, b0);
    d3_lds_words<S>(bp + (rho + 8) * r + 64 * ch + 4 * S * c, b1);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) d3_lds_words<S>(gts + (nt * 8 + rho) * gs + 64 * ch + 4 * S * c, g[nt]);
#pragma unroll
    for (int s = 0; s < S; ++s) {
      const uint32_t af[4] = {b0[2 * s], b1[2 * s], b0[2 * s + 1], b1[2 * s + 1]};
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(acc[nt], af, g[nt][2 * s], g[nt][2 * s + 1]);
    }
  }
}

template <int MT>
__device__ __forceinline__ void d3_ecterm_r(const __nv_bfloat16* bp, const __nv_bfloat16* gts, int r, int lane,
                                            float (&acc)[MT / 8][4]) {
  if (r == 16)
    d3_ecterm<MT, 1, 1>(bp, gts, r, lane, acc);
  else if (r == 32)
    d3_ecterm<MT, 2, 1>(bp, gts, r, lane, acc);
  else if (r == 64)
    d3_ecterm<MT, 4, 1>(bp, gts, r, lane, acc);
  else
    d3_ecterm<MT, 4, 2>(bp, gts, r, lane, acc);
}

// This warp's partial of one weight strip: CH packed tiles of its slice,
// dequantised in registers, against the activation fragments.  Per channel,
// the codes enter the MMAs as 136 + q and 136 * sum(x) is removed at the end;
// with group scales, every tile's partial is scaled by its group's scale.
template <int MT, int CH, bool GROUP>
__device__ __forceinline__ void d3_w_item(const uint8_t* base, int KTC, int w, int lane,
                                          const uint32_t (&xf)[CH][MT / 8][8], const float (&xsA)[MT / 8],
                                          const float (&xsB)[MT / 8], float (&acc)[MT / 8][4]) {
  constexpr int NT = MT / 8;
  constexpr int ACCS = MT == 8 ? 4 : 2;  // independent accumulator sets (k16 step mod ACCS)
  const int rho = lane >> 2;
  const uint8_t* src = base + w * CH * 512 + lane * 16;
  if (GROUP) {
    // a partial per tile (its own scale group); at M = 16 two tiles at a time
    constexpr int TB = MT == 8 ? CH : (CH < 2 ? CH : 2);
    const __half* sc = reinterpret_cast<const __half*>(base + KTC * 512);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
    for (int t0 = 0; t0 < CH; t0 += TB) {
      float part[TB][NT][4];
#pragma unroll
      for (int tb = 0; tb < TB; ++tb)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) part[tb][nt][0] = part[tb][nt][1] = part[tb][nt][2] = part[tb][nt][3] = 0.f;
#pragma unroll
      for (int tb = 0; tb < TB; ++tb) {
        if (t0 + tb >= CH) break;
        const int t = t0 + tb;
        const uint4 wv = *reinterpret_cast<const uint4*>(src + t * 512);
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          uint32_t af[4];
          int4x8_to_bf16x8(d3_w(wv, s), af);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(part[tb][nt], af, xf[t][nt][2 * s], xf[t][nt][2 * s + 1]);
        }
      }
#pragma unroll
      for (int tb = 0; tb < TB; ++tb) {
        if (t0 + tb >= CH) break;
        const int g = (w * CH + t0 + tb) >> 1;
        const float s0 = __half2float(sc[g * 16 + rho]), s1 = __half2float(sc[g * 16 + rho + 8]);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          acc[nt][0] = fmaf(s0, part[tb][nt][0], acc[nt][0]);
          acc[nt][1] = fmaf(s0, part[tb][nt][1], acc[nt][1]);
          acc[nt][2] = fmaf(s1, part[tb][nt][2], acc[nt][2]);
          acc[nt][3] = fmaf(s1, part[tb][nt][3], acc[nt][3]);
        }
      }
    }
  } else {
    float accs[ACCS][NT][4];
#pragma unroll
    for (int h = 0; h < ACCS; ++h)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) accs[h][nt][0] = accs[h][nt][1] = accs[h][nt][2] = accs[h][nt][3] = 0.f;
#pragma unroll
    for (int t = 0; t < CH; ++t) {
      const uint4 wv = *reinterpret_cast<const uint4*>(src + t * 512);
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        uint32_t af[4];
        d3_nib_biased(d3_w(wv, s), af);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          mma_bf16_16816(accs[(4 * t + s) % ACCS][nt], af, xf[t][nt][2 * s], xf[t][nt][2 * s + 1]);
      }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float v = accs[0][nt][e];
#pragma unroll
        for (int h = 1; h < ACCS; ++h) v += accs[h][nt][e];
        acc[nt][e] = v;
      }
      acc[nt][0] -= xsA[nt];
      acc[nt][1] -= xsB[nt];
      acc[nt][2] -= xsA[nt];
      acc[nt][3] -= xsB[nt];
    }
  }
}

// Reduction of item i by one warp: the 8 warp partials in warp order, then to
// the owner rank (or parked here); the owner of the EC item adds the ranks
// (rank order) and publishes its rows for the live tokens, then raises the
// item's flag.  Out of line: it runs for one item in eight per warp.
template <int MT>
__device__ __noinline__ bool d3_reduce(const D3Args& a, uint8_t* sm, int i, int q, int n_ec, int ec_item, int tag,
                                       volatile int* abortp, int lane) {
  constexpr int NT = MT / 8;
  constexpr unsigned FULL = 0xffffffffu;
  const D3Smem SL = d3_smem(MT, a.nslot, a.slot, a.CS, a.own_cap, a.r);
  const float4* red = reinterpret_cast<const float4*>(sm + SL.red);
  float4* park = reinterpret_cast<float4*>(sm + SL.park);
  float4* recv = reinterpret_cast<float4*>(sm + SL.recv);
  uint64_t* redfull = reinterpret_cast<uint64_t*>(sm + SL.bars) + 2 * a.nslot;
  uint64_t* redempty = redfull + D3_NB;
  uint64_t* recvbar = redempty + D3_NB;
  const int rho = lane >> 2, c = lane & 3;
  const int b = i % D3_NB, k = i / D3_NB;
  if (!__all_sync(FULL, d3_wait(&redfull[b], k & 1, abortp, a.hdr))) return false;
  float tot[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) tot[nt][0] = tot[nt][1] = tot[nt][2] = tot[nt][3] = 0.f;
#pragma unroll
  for (int w2 = 0; w2 < D3_NW; ++w2)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const float4 v = red[((b * D3_NW + w2) * NT + nt) * 32 + lane];
      tot[nt][0] += v.x;
      tot[nt][1] += v.y;
      tot[nt][2] += v.z;
      tot[nt][3] += v.w;
    }
  __syncwarp();
  if (lane == 0) mbar_arrive_relaxed(&redempty[b]);
  const int owner = i % a.CS, o = i / a.CS;
  if (owner != q) {
    const uint32_t rbar = map_rank(smem_u32(&recvbar[o]), owner);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const uint32_t dst = map_rank(smem_u32(recv + (o * NT + nt) * 32 + lane), owner);
      st_async_f4(dst, make_float4(tot[nt][0], tot[nt][1], tot[nt][2], tot[nt][3]), rbar);
    }
    return true;
  }
  if (i >= n_ec) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
      park[(o * NT + nt) * 32 + lane] = make_float4(tot[nt][0], tot[nt][1], tot[nt][2], tot[nt][3]);
    return true;
  }
  if (a.CS > 1) {
    if (!__all_sync(FULL, d3_wait(&recvbar[o], 0, abortp, a.hdr))) return false;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const float4 v = recv[(o * NT + nt) * 32 + lane];
      tot[nt][0] += v.x;
      tot[nt][1] += v.y;
      tot[nt][2] += v.z;
      tot[nt][3] += v.w;
    }
  }
  float* dst = a.tf + (size_t)ec_item * MT * 16;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int t0 = nt * 8 + 2 * c;
    if (t0 < a.M) {
      dst[t0 * 16 + rho] = tot[nt][0];
      dst[t0 * 16 + rho + 8] = tot[nt][2];
    }
    if (t0 + 1 < a.M) {
      dst[(t0 + 1) * 16 + rho] = tot[nt][1];
      dst[(t0 + 1) * 16 + rho + 8] = tot[nt][3];
    }
  }
  __threadfence();
  __syncwarp();
  if (lane == 0) st_release_gpu(&a.hdr->d3_flag[ec_item], tag);
  return true;
}

// Gate and gt for the live tokens (every thread of the CTA; t and the gate
// logits are in shared memory), then the reported gate and mask count (CTA 0).
// Scalar gate: g = sigmoid(logit + b_g), gt = bf16(g t).  The pages' per-rank
// gate: u = relu(W1 t + b1), gamma = sigmoid(W2 u + b2), gt = bf16(alpha gamma t),
// reported gate = mean of gamma (summed in rank order); the idle ring holds u
// and gamma.  Padded tokens get zero rows.
template <int MT>
__device__ __noinline__ void d3_build_gate(const D3Args& a, uint8_t* sm, uint8_t* ring) {
  const D3Smem SL = d3_smem(MT, a.nslot, a.slot, a.CS, a.own_cap, a.r);
  const float* ts = reinterpret_cast<const float*>(sm + SL.ts);
  __nv_bfloat16* gts = reinterpret_cast<__nv_bfloat16*>(sm + SL.gts);
  float* gv = reinterpret_cast<float*>(sm + SL.gv);
  const int tid = threadIdx.x, gs = a.r + 8;
  if (a.gate_kind == 0) {
    if (tid < MT) gv[tid] = tid < a.M ? sigmoidf_(ts[MT * a.r + tid] + a.b_g) : 0.f;
    __syncthreads();
    const int half = a.r / 2;
    for (int idx = tid; idx < MT * half; idx += D3_THREADS) {
      const int m = idx / half, j = 2 * (idx - m * half);
      const float g = gv[m];
      *reinterpret_cast<uint32_t*>(gts + m * gs + j) =
          m < a.M ? pack_bf16x2(g * ts[m * a.r + j], g * ts[m * a.r + j + 1]) : 0u;
    }
  } else {
    const int h = a.gate_h, r = a.r;
    float* hid = reinterpret_cast<float*>(ring);  // [MT][32]
    float* gam = hid + MT * 32;                   // [MT][r]
    for (int idx = tid; idx < a.M * h; idx += D3_THREADS) {
      const int m = idx / h, i = idx - m * h;
      const float4* w1 = reinterpret_cast<const float4*>(a.gw1 + (size_t)i * r);
      const float4* tv = reinterpret_cast<const float4*>(ts + m * r);
      float z0 = 0.f, z1 = 0.f, z2 = 0.f, z3 = 0.f;
      for (int j4 = 0; j4 < r / 4; ++j4) {
        const float4 wv = __ldg(w1 + j4), xv = tv[j4];
        z0 = fmaf(wv.x, xv.x, z0);
        z1 = fmaf(wv.y, xv.y, z1);
        z2 = fmaf(wv.z, xv.z, z2);
        z3 = fmaf(wv.w, xv.w, z3);
      }
      hid[m * 32 + i] = fmaxf((z0 + z1) + (z2 + z3) + __ldg(a.gb1 + i), 0.f);
    }
    __syncthreads();
    for (int idx = tid; idx < MT * r; idx += D3_THREADS) {
      const int m = idx / r, j = idx - m * r;
      float gam_v = 0.f;
      if (m < a.M) {
        const float4* w2 = reinterpret_cast<const float4*>(a.gw2 + (size_t)j * h);
        const float4* uv = reinterpret_cast<const float4*>(hid + m * 32);
        float z0 = 0.f, z1 = 0.f, z2 = 0.f, z3 = 0.f;
        for (int i4 = 0; i4 < h / 4; ++i4) {
          const float4 wv = __ldg(w2 + i4), xv = uv[i4];
          z0 = fmaf(wv.x, xv.x, z0);
          z1 = fmaf(wv.y, xv.y, z1);
          z2 = fmaf(wv.z, xv.z, z2);
          z3 = fmaf(wv.w, xv.w, z3);
        }
        gam_v = sigmoidf_(__ldg(a.gb2 + j) + ((z0 + z1) + (z2 + z3)));
      }
      gam[m * r + j] = gam_v;
      gts[m * gs + j] = __float2bfloat16_rn(m < a.M ? a.alpha * gam_v * ts[m * r + j] : 0.f);
    }
    __syncthreads();
    if (tid < MT) {
      float sgm = 0.f;
      for (int j = 0; j < r; ++j) sgm += gam[tid * r + j];
      gv[tid] = tid < a.M ? sgm / (float)r : 0.f;
    }
  }
  __syncthreads();
  if (blockIdx.x == 0 && tid < 32) {
    const int lane = tid;
    const bool valid = lane < a.M;
    const float g = lane < MT ? gv[lane] : 0.f;
    if (a.gate_out && valid) a.gate_out[lane] = g;
    const unsigned below = __ballot_sync(0xffffffffu, valid && g < a.tau);
    if (a.mask_count && lane == 0) *a.mask_count = __popc(below);
  }
}

// The owned weight strips: warp k % 9 finishes the k-th one -- the ranks'
// partials added in rank order, + gt . B', scaled, rounded to bf16 and stored
// with 16-byte stores (added to y in place in EC-only mode).
template <int MT, bool GROUP>
__device__ __noinline__ void d3_finish_strips(const D3Args& a, uint8_t* sm, int q, int n_ec, int w_lo, int n_own,
                                              volatile int* abortp) {
  constexpr int NT = MT / 8;
  constexpr unsigned FULL = 0xffffffffu;
  const D3Smem SL = d3_smem(MT, a.nslot, a.slot, a.CS, a.own_cap, a.r);
  const float4* park = reinterpret_cast<const float4*>(sm + SL.park);
  const float4* recv = reinterpret_cast<const float4*>(sm + SL.recv);
  const __nv_bfloat16* bps = reinterpret_cast<const __nv_bfloat16*>(sm + SL.bps);
  const __half* scs = reinterpret_cast<const __half*>(sm + SL.scs);
  const __nv_bfloat16* gts = reinterpret_cast<const __nv_bfloat16*>(sm + SL.gts);
  uint64_t* recvbar = reinterpret_cast<uint64_t*>(sm + SL.bars) + 2 * a.nslot + 2 * D3_NB;
  uint64_t* epibar = recvbar + a.own_cap;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, rho = lane >> 2, c = lane & 3;
  const bool has_ec = a.ES > 0;
  const int first_w = (n_ec - q + a.CS - 1) / a.CS;  // first owned index o with o * CS + q >= n_ec
  bool ok = true;
  for (int o = first_w + warp; o < n_own && ok; o += D3_NW + 1) {
    const int i = o * a.CS + q;
    const int p = w_lo + (i - n_ec);
    ok = __all_sync(FULL, d3_wait(epibar, 0, abortp, a.hdr));
    float tot[NT][4];
    if (a.ec_only) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) tot[nt][0] = tot[nt][1] = tot[nt][2] = tot[nt][3] = 0.f;
    } else {
      if (a.CS > 1) ok = ok && __all_sync(FULL, d3_wait(&recvbar[o], 0, abortp, a.hdr));
      if (!ok) break;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const float4 v0 = park[(o * NT + nt) * 32 + lane];
        float4 v = v0;
        if (a.CS > 1) {
          const float4 v1 = recv[(o * NT + nt) * 32 + lane];
          const float4 lo = q == 0 ? v0 : v1, hi = q == 0 ? v1 : v0;  // rank 0's partial first
          v = make_float4(lo.x + hi.x, lo.y + hi.y, lo.z + hi.z, lo.w + hi.w);
        }
        tot[nt][0] = v.x;
        tot[nt][1] = v.y;
        tot[nt][2] = v.z;
        tot[nt][3] = v.w;
      }
    }
    if (!ok) break;
    if (has_ec) d3_ecterm_r<MT>(bps + (size_t)o * 16 * a.r, gts, a.r, lane, tot);
    float s0 = 1.f, s1 = 1.f;
    if (!GROUP) {
      s0 = __half2float(scs[o * 16 + rho]);
      s1 = __half2float(scs[o * 16 + rho + 8]);
    }
    __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(sm + SL.stage) + warp * MT * 16;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int t0 = nt * 8 + 2 * c;
      stage[t0 * 16 + rho] = __float2bfloat16_rn(s0 * tot[nt][0]);
      stage[(t0 + 1) * 16 + rho] = __float2bfloat16_rn(s0 * tot[nt][1]);
      stage[t0 * 16 + rho + 8] = __float2bfloat16_rn(s1 * tot[nt][2]);
      stage[(t0 + 1) * 16 + rho + 8] = __float2bfloat16_rn(s1 * tot[nt][3]);
    }
    __syncwarp();
    const int m = lane >> 1, hh = lane & 1;
    if (m < a.M) {
      uint4 v = *reinterpret_cast<const uint4*>(stage + m * 16 + 8 * hh);
      uint4* dst = reinterpret_cast<uint4*>(a.y + (size_t)m * a.N + 16 * p + 8 * hh);
      if (a.ec_only) {
        // y holds the EC-disabled GEMM result: add the EC term in fp32, round once more
        const uint4 old = *dst;
        const uint32_t* ov = reinterpret_cast<const uint32_t*>(&old);
        uint32_t* nv = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 a2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(ov + e));
          const float2 b2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(nv + e));
          nv[e] = pack_bf16x2(a2.x + b2.x, a2.y + b2.y);
        }
      }
      *dst = v;
    }
    __syncwarp();
  }
}

template <int MT, int CH, bool GROUP>
__global__ void __launch_bounds__(D3_THREADS, 2)
    decode3_kernel(const __grid_constant__ D3Args a, const __grid_constant__ CUtensorMap tm_w,
                   const __grid_constant__ CUtensorMap tm_agt, const __grid_constant__ CUtensorMap tm_gate,
                   const __grid_constant__ CUtensorMap tm_bp, const __grid_constant__ CUtensorMap tm_gs) {
  constexpr int NT = MT / 8;
  constexpr unsigned FULL = 0xffffffffu;
  extern __shared__ uint8_t smem_raw[];
  __shared__ int s_abort;
  __shared__ int s_issued;  // ring units issued so far (read only after an abort)
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const D3Smem SL = d3_smem(MT, a.nslot, a.slot, a.CS, a.own_cap, a.r);
  uint8_t* ring = sm + SL.ring;
  float4* red = reinterpret_cast<float4*>(sm + SL.red);
  float4* park = reinterpret_cast<float4*>(sm + SL.park);
  float4* recv = reinterpret_cast<float4*>(sm + SL.recv);
  __nv_bfloat16* bps = reinterpret_cast<__nv_bfloat16*>(sm + SL.bps);
  __half* scs = reinterpret_cast<__half*>(sm + SL.scs);
  float* ts = reinterpret_cast<float*>(sm + SL.ts);
  __nv_bfloat16* gts = reinterpret_cast<__nv_bfloat16*>(sm + SL.gts);
  float* gv = reinterpret_cast<float*>(sm + SL.gv);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + SL.bars);
  uint64_t* empty = full + a.nslot;
  uint64_t* redfull = empty + a.nslot;
  uint64_t* redempty = redfull + D3_NB;
  uint64_t* recvbar = redempty + D3_NB;
  uint64_t* epibar = recvbar + a.own_cap;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rho = lane >> 2, c = lane & 3;
  const int q = a.CS > 1 ? (int)cluster_rank() : 0;
  const short4 ct = a.cl_tab[blockIdx.x / a.CS];
  const int ec_item = ct.x, w_lo = ct.y, n_w = ct.z;
  const int n_ec = ec_item >= 0 ? 1 : 0;
  const int n_items = n_ec + n_w;
  const bool has_ec = a.ES > 0;
  const int n_ecu = ec_item < 0 ? 0 : (ec_item < a.ES ? CH : 1);  // ring units of the EC item
  const int U = n_ecu + (a.ec_only ? 0 : n_w);
  const int n_own = n_items > q ? (n_items - q + a.CS - 1) / a.CS : 0;  // items i = o * CS + q
  const uint32_t wbytes = (uint32_t)a.KTC * 512u + (GROUP ? (uint32_t)a.KTC * 16u : 0u);
  volatile int* abortp = &s_abort;

  // ring unit u into slot `slot`
  auto issue = [&](int slot, int u) {
    uint64_t* bar = &full[slot];
    const uint32_t dst = smem_u32(ring + (size_t)slot * a.slot);
    if (u < n_ecu) {
      if (ec_item < a.ES) {
        // tile u of every warp's slice of the A^T strip
        mbar_arrive_tx(bar, D3_NW * 2048);
#pragma unroll
        for (int wi = 0; wi < D3_NW; ++wi)
          tma_load_2d(dst + wi * 2048, &tm_agt, bar, (q * a.KTC + wi * CH + u) * 64, 16 * ec_item);
      } else {
        // the gate row over every warp's slice
        mbar_arrive_tx(bar, D3_NW * CH * 128);
#pragma unroll
        for (int wi = 0; wi < D3_NW; ++wi)
          tma_load_2d(dst + wi * CH * 128, &tm_gate, bar, (q * a.KTC + wi * CH) * 64, a.r);
      }
    } else {
      const int p = w_lo + (u - n_ecu);
      mbar_arrive_tx(bar, wbytes);
      tma_load_3d(dst, &tm_w, bar, 0, q * a.KTC, p);
      if (GROUP) tma_load_2d(dst + a.KTC * 512, &tm_gs, bar, 16 * p, q * a.KTC / 2);
    }
  };

  if (warp == 0) {
    for (int s = lane; s < a.nslot; s += 32) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], D3_NW);
    }
    if (lane < D3_NB) {
      mbar_init(&redfull[lane], D3_NW);
      mbar_init(&redempty[lane], 1);
    }
    for (int o = lane; o < a.own_cap; o += 32) mbar_init(&recvbar[o], 1);
    if (lane == 0) {
      mbar_init(epibar, 1);
      s_abort = 0;
      s_issued = U < a.nslot ? U : a.nslot;
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    __syncwarp();
    if (a.CS > 1) {
      // the other rank's partials of the items this CTA finishes arrive by st.async
      for (int o = lane; o < n_own; o += 32) {
        const int i = o * a.CS + q;
        if (!(a.ec_only && i >= n_ec)) mbar_arrive_tx(&recvbar[o], NT * 512);
      }
    }
    // epilogue operands of the owned weight strips: B' rows and per-channel scales
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
    // nothing in the ring depends on the previous kernel: fill it now
    const int first = U < a.nslot ? U : a.nslot;
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
  // the next kernel in the stream may start (and fill its own ring) now
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // x, y and the workspace may belong to the previous kernel in the stream
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int tag = *reinterpret_cast<volatile int*>(&a.hdr->d2_epoch) + 1;
  if (!has_ec && blockIdx.x == 0 && warp == 1) {
    if (a.gate_out && lane < a.M) a.gate_out[lane] = 0.f;
    if (a.mask_count && lane == 0) *a.mask_count = a.M;
  }

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    const int first = U < a.nslot ? U : a.nslot;
    int slot = first % a.nslot;
    uint32_t round = first / a.nslot;
    bool ok = true;
    for (int u = first; u < U; ++u) {
      ok = __all_sync(FULL, d3_wait_sleep(&empty[slot], (round & 1) ^ 1, abortp, a.hdr));
      if (!ok) break;
      if (lane == 0) {
        issue(slot, u);
        s_issued = u + 1;
      }
      __syncwarp();
      if (++slot == a.nslot) {
        slot = 0;
        ++round;
      }
    }
    if (a.CS > 1) asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
    if (ok && has_ec) {
      // every EC item's flag, then the published rows of the live tokens
      const int ne = a.ES + a.gate_item;
      const long long t0 = clock64();
      uint32_t ns = 64;
      while (true) {
        bool ready = true;
        for (int e = 0; e < ne; ++e) ready = ready && ld_acquire_gpu(&a.hdr->d3_flag[e]) == tag + a.tag_skew;
        if (__all_sync(FULL, ready)) break;
        int stop = 0;
        if (lane == 0) {
          if (*abortp) {
            stop = 1;
          } else if (clock64() - t0 > a.pub_wait) {
            report_status(a.hdr, SPEAR_ERR_TIMEOUT);
            *abortp = 1;
            stop = 1;
          }
        }
        if (__shfl_sync(FULL, stop, 0)) {
          ok = false;
          break;
        }
        __nanosleep(ns);
        ns = ns < 512 ? ns * 2 : 512;
      }
      if (ok) {
        // t rows: [ES][MT][16] -> ts [m][r]; gate logits: row 0 of item ES -> ts[MT * r + m]
        constexpr int MAXV = 8 * MT * 16 / 4 / 32;  // float4 per lane for r = 128
        const int nv = a.ES * a.M * 4;              // float4 of t for the live tokens
        float4 v[MAXV];
#pragma unroll
        for (int j = 0; j < MAXV; ++j) {
          const int idx = j * 32 + lane;
          if (idx < nv) {
            const int e = idx / (a.M * 4), rem = idx - e * a.M * 4;
            v[j] = __ldcg(reinterpret_cast<const float4*>(a.tf + (size_t)e * MT * 16) + rem);
          }
        }
        float gl = 0.f;
        if (a.gate_item && lane < a.M) gl = __ldcg(a.tf + (size_t)a.ES * MT * 16 + lane * 16);
#pragma unroll
        for (int j = 0; j < MAXV; ++j) {
          const int idx = j * 32 + lane;
          if (idx < nv) {
            const int e = idx / (a.M * 4), rem = idx - e * a.M * 4;
            const int m = rem >> 2, r0 = (rem & 3) * 4;
            *reinterpret_cast<float4*>(ts + m * a.r + 16 * e + r0) = v[j];
          }
        }
        if (lane < a.M) ts[MT * a.r + lane] = gl;
      }
    }
  } else {
    // ---------------------------------------------------------------- consumers
    const int w = warp - 1;
    // activations of this warp's k slice as B fragments: word i of xf[t][nt]
    // = x[nt*8 + rho][64 (kt0 + t) + 16c + 2i .. + 1]
    uint32_t xf[CH][NT][8];
    const int kt0 = q * a.KTC + w * CH;
#pragma unroll
    for (int t = 0; t < CH; ++t)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int m = nt * 8 + rho;
        uint4 v0 = make_uint4(0u, 0u, 0u, 0u), v1 = v0;
        if (m < a.M) {
          const uint4* src = reinterpret_cast<const uint4*>(a.x + (size_t)m * a.K + (size_t)(kt0 + t) * 64 + 16 * c);
          v0 = __ldcg(src);
          v1 = __ldcg(src + 1);
        }
        xf[t][nt][0] = v0.x; xf[t][nt][1] = v0.y; xf[t][nt][2] = v0.z; xf[t][nt][3] = v0.w;
        xf[t][nt][4] = v1.x; xf[t][nt][5] = v1.y; xf[t][nt][6] = v1.z; xf[t][nt][7] = v1.w;
      }
    if (a.CS > 1) asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
    // per-channel codes enter the MMAs as 136 + q: remove 136 * sum(x) of the
    // slice per token (accumulator columns 2c and 2c + 1 of each n8 tile)
    float xsA[NT], xsB[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      xsA[nt] = xsB[nt] = 0.f;
      if (!GROUP) {
        float sx = 0.f;
#pragma unroll
        for (int t = 0; t < CH; ++t)
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xf[t][nt][i]));
            sx += f.x + f.y;
          }
        sx += __shfl_xor_sync(FULL, sx, 1);
        sx += __shfl_xor_sync(FULL, sx, 2);
        xsA[nt] = 136.f * __shfl_sync(FULL, sx, 8 * c);
        xsB[nt] = 136.f * __shfl_sync(FULL, sx, 8 * c + 4);
      }
    }

    bool ok = true;
    int u = 0;  // ring unit counter, in the producer's order
    // this warp's partial of item j into buffer j % NB (free once item j - NB
    // is reduced), then its turn at reducing item j - 1
    auto finish_item = [&](int j, const float (&acc)[NT][4]) {
      const int b = j % D3_NB, k = j / D3_NB;
      if (!__all_sync(FULL, d3_wait(&redempty[b], (k & 1) ^ 1, abortp, a.hdr))) {
        ok = false;
        return;
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        red[((b * D3_NW + w) * NT + nt) * 32 + lane] = make_float4(acc[nt][0], acc[nt][1], acc[nt][2], acc[nt][3]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&redfull[b]);
      if (j >= 1 && (j - 1) % D3_NW == w)
        ok = d3_reduce<MT>(a, sm, j - 1, q, n_ec, ec_item, tag, abortp, lane);
    };

    if (n_ec > 0) {
      // the EC item (at most one per cluster, first): an A^T strip or the gate row
      float acc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
      if (ec_item < a.ES) {
#pragma unroll
        for (int t = 0; t < CH; ++t) {
          const int slot = u % a.nslot;
          ok = ok && __all_sync(FULL, d3_wait(&full[slot], (u / a.nslot) & 1, abortp, a.hdr));
          if (ok) d3_ec_tile<NT>(ring + (size_t)slot * a.slot + w * 2048, xf[t], lane, acc);
          __syncwarp();
          if (lane == 0) mbar_arrive_relaxed(&empty[slot]);
          ++u;
        }
      } else {
        const int slot = u % a.nslot;
        ok = ok && __all_sync(FULL, d3_wait(&full[slot], (u / a.nslot) & 1, abortp, a.hdr));
        if (ok) {
#pragma unroll
          for (int t = 0; t < CH; ++t)
            d3_gate_tile<NT>(ring + (size_t)slot * a.slot + w * CH * 128 + t * 128, xf[t], lane, acc);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_relaxed(&empty[slot]);
        ++u;
      }
      if (ok) finish_item(0, acc);
    }
    // weight strips: the hot loop
    const int n_part = a.ec_only ? n_ec : n_items;  // items with partials
    int slot = u % a.nslot;
    uint32_t phase = (u / a.nslot) & 1;
    for (int j = n_ec; j < n_part && ok; ++j) {
      ok = __all_sync(FULL, d3_wait(&full[slot], phase, abortp, a.hdr));
      if (!ok) break;
      float acc[NT][4];
      d3_w_item<MT, CH, GROUP>(ring + (size_t)slot * a.slot, a.KTC, w, lane, xf, xsA, xsB, acc);
      __syncwarp();
      if (lane == 0) mbar_arrive_relaxed(&empty[slot]);
      if (++slot == a.nslot) {
        slot = 0;
        phase ^= 1u;
      }
      finish_item(j, acc);
    }
    if (ok && n_part > 0 && (n_part - 1) % D3_NW == w)
      ok = d3_reduce<MT>(a, sm, n_part - 1, q, n_ec, ec_item, tag, abortp, lane);
  }

  // ------------------------------------------------------------------ end phase
  __syncthreads();
  // Read once by every thread between two barriers: nothing writes the flag
  // before the gate block's last barrier, so the branch below is uniform.
  const bool live = !*abortp;
  if (has_ec && live) d3_build_gate<MT>(a, sm, ring);
  if (live) d3_finish_strips<MT, GROUP>(a, sm, q, n_ec, w_lo, n_own, abortp);
  if (warp == 0) {
    // no copy may still write into this CTA's shared memory when it exits: the
    // last nslot units issued (each slot holds one outstanding phase at most)
    // and the epilogue operands (already complete unless a role gave up early)
    const int issued = *abortp ? s_issued : U;
    for (int u2 = issued > a.nslot ? issued - a.nslot : 0; u2 < issued; ++u2)
      d3_drain(&full[u2 % a.nslot], (u2 / a.nslot) & 1);
    d3_drain(epibar, 0);
  }
  if (has_ec && threadIdx.x == 0 && live && !*abortp) {
    // every CTA has read this launch's rows; the last one advances the epoch
    if (atomicAdd(&a.hdr->gt_obs, 1) == a.G - 1) {
      a.hdr->gt_obs = 0;
      a.hdr->d2_epoch = tag;
    }
  }
  // no CTA of the cluster leaves while st.async writes into it may be in flight
  if (a.CS > 1) asm volatile("barrier.cluster.arrive.relaxed;\n\tbarrier.cluster.wait;" ::: "memory");
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
struct D3Plan {
  int MT, CH, CS, NC, KTC, ES, gate_item, nslot, slot, own_cap;
  size_t smem;
  const char* why;  // non-null: this kernel cannot run the shape
  std::vector<short4> cl_tab;
};

// CTAs per SM of one launch: 1 (the next launch's CTA fits beside it and
// fills its ring meanwhile) or 2 (two CTAs of the same launch).
static int d3_ctas_per_sm() {
  static int v = [] {
    const char* e = getenv("SPEAR_DECODE_CTAS_PER_SM");
    const int n = e ? atoi(e) : 1;
    return n == 2 ? 2 : 1;
  }();
  return v;
}

static D3Plan make_d3_plan(int MT, int K, int N, int r, int group, int gate_kind, int sms, int nc_cap) {
  D3Plan p = {};
  p.MT = MT;
  p.why = nullptr;
  const int KT = K / 64;
  if (KT % 8) {
    p.why = "K must be a multiple of 512";
    return p;
  }
  p.CS = KT / 8 <= 4 ? 1 : 2;
  if ((KT / p.CS) % 8 || KT / p.CS / 8 > 4) {
    p.why = "K above 4096 (or not a multiple of 1024 above 2048)";
    return p;
  }
  p.KTC = KT / p.CS;
  p.CH = p.KTC / 8;
  p.ES = r / 16;
  p.gate_item = r > 0 && gate_kind == SPEAR_GATE_SCALAR ? 1 : 0;
  const int n_ec = p.ES + p.gate_item;
  const int NS = N / 16;
  int NC = d3_ctas_per_sm() * sms / p.CS;
  NC = std::min(NC, nc_cap);
  NC = std::min(NC, NS + n_ec);
  NC = std::min(NC, D3_MAXCL);
  if (NC < n_ec) {
    p.why = "too few clusters for the EC items";
    return p;
  }
  p.NC = NC;
  // balance streamed bytes per k-tile: weight strip 512 B, A^T strip 2 KB, gate row 128 B
  const long long cw = 4, ce = 16, cg = 1;
  const long long C = cw * NS + ce * p.ES + cg * p.gate_item;
  p.cl_tab.resize(NC);
  int own = 1, w0 = 0;
  long long cum = 0;
  for (int c = 0; c < NC; ++c) {
    const int e = c < n_ec ? c : -1;
    const long long ec_cost = e < 0 ? 0 : (e < p.ES ? ce : cg);
    int nw;
    if (c == NC - 1) {
      nw = NS - w0;
    } else {
      const long long target = C * (c + 1) / NC;
      nw = (int)std::max<long long>(0, (target - cum - ec_cost + cw / 2) / cw);
      nw = std::min(nw, NS - w0);
    }
    p.cl_tab[c] = make_short4((short)e, (short)w0, (short)nw, 0);
    cum += ec_cost + cw * nw;
    w0 += nw;
    own = std::max(own, ((e >= 0 ? 1 : 0) + nw + p.CS - 1) / p.CS);
  }
  p.own_cap = own;
  if (own > D3_MAXOWN) {
    p.why = "too many strips per CTA for the decode kernel";
    return p;
  }
  p.slot = 16384 + (group ? 1024 : 0);
  const size_t cap = 112 * 1024;
  const D3Smem s0 = d3_smem(MT, 0, p.slot, p.CS, own, r);
  p.nslot = (int)std::min<size_t>(8, (cap - std::min<size_t>(s0.total + 16, cap)) / (p.slot + 16));
  if (p.nslot < 3) {
    p.why = "shared memory too small for the decode kernel's ring";
    return p;
  }
  p.smem = d3_smem(MT, p.nslot, p.slot, p.CS, own, r).total;
  return p;
}

template <int MT, int CH, bool GROUP>
static cudaError_t d3_attrs(size_t smem) {
  static std::mutex mu;
  static size_t opted = 0;
  std::lock_guard<std::mutex> lk(mu);
  if (smem <= opted) return cudaSuccess;
  cudaError_t e =
      cudaFuncSetAttribute(decode3_kernel<MT, CH, GROUP>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(decode3_kernel<MT, CH, GROUP>, cudaFuncAttributePreferredSharedMemoryCarveout,
                           (int)cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  opted = smem;
  return cudaSuccess;
}

// Clusters of the (MT, CH) instance resident at once with `smem` bytes per CTA.
template <int MT, int CH>
static int d3_max_clusters_t(int CS, size_t smem) {
  if (d3_attrs<MT, CH, false>(smem) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  if (CS == 1) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode3_kernel<MT, CH, false>, D3_THREADS, smem) !=
        cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    return per_sm * device_sm_count();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CS);
  cfg.blockDim = dim3(D3_THREADS);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, decode3_kernel<MT, CH, false>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

static int d3_max_clusters(int MT, int CH, int CS, size_t smem) {
  switch (MT * 10 + CH) {
    case 81: return d3_max_clusters_t<8, 1>(CS, smem);
    case 82: return d3_max_clusters_t<8, 2>(CS, smem);
    case 83: return d3_max_clusters_t<8, 3>(CS, smem);
    case 84: return d3_max_clusters_t<8, 4>(CS, smem);
    case 161: return d3_max_clusters_t<16, 1>(CS, smem);
    case 162: return d3_max_clusters_t<16, 2>(CS, smem);
    case 163: return d3_max_clusters_t<16, 3>(CS, smem);
    default: return d3_max_clusters_t<16, 4>(CS, smem);
  }
}

// The plan for a shape, its clusters capped at what is resident at once.
static const D3Plan& d3_plan(int MT, int K, int N, int r, int group, int gate_kind, int sms) {
  static std::mutex mu;
  static std::map<std::tuple<int, int, int, int, int, int, int, int, int>, D3Plan> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  const auto key = std::make_tuple(dev, MT, K, N, r, group, gate_kind, sms, d3_ctas_per_sm());
  std::lock_guard<std::mutex> lk(mu);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  D3Plan p = make_d3_plan(MT, K, N, r, group, gate_kind, sms, 1 << 30);
  for (int iter = 0; !p.why; ++iter) {
    const int mc = d3_max_clusters(MT, p.CH, p.CS, p.smem);
    if (mc <= 0) {
      p.why = "cluster occupancy query failed for the decode kernel";
    } else if (p.NC > mc) {
      if (iter == 3)
        p.why = "the decode kernel's clusters do not fit on the device at once";
      else
        p = make_d3_plan(MT, K, N, r, group, gate_kind, sms, mc);
    } else {
      break;
    }
  }
  return cache.emplace(key, std::move(p)).first->second;
}

const char* decode3_unsupported(int M, int K, int N, int r, int group, int gate_kind, int gate_h) {
  (void)gate_h;
  if (M < 1 || M > 16) return "the decode kernel needs 1 <= M <= 16";
  return d3_plan(M <= 8 ? 8 : 16, K, N, r, group, r > 0 ? gate_kind : 0, device_sm_count()).why;
}

template <int MT, int CH, bool GROUP>
static int d3_launch_t(const D3Args& a, const CUtensorMap* maps, size_t smem, int grid, cudaStream_t st) {
  cudaError_t e = d3_attrs<MT, CH, GROUP>(smem);
  if (e != cudaSuccess) return set_cuda_error("cudaFuncSetAttribute(decode)", e);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(D3_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[3];
  int na = 0;
  // programmatic dependent launch: this grid may start while the previous
  // kernel in the stream runs; it waits for it before touching x, y, ws
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  if (a.CS > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = a.CS;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
    attr[na].id = cudaLaunchAttributeClusterSchedulingPolicyPreference;
    attr[na].val.clusterSchedulingPolicyPreference = cudaClusterSchedulingPolicySpread;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  e = cudaLaunchKernelEx(&cfg, decode3_kernel<MT, CH, GROUP>, a, maps[0], maps[1], maps[2], maps[3], maps[4]);
  if (e != cudaSuccess) return set_cuda_error("decode launch", e);
  return SPEAR_OK;
}

template <int MT, int CH>
static int d3_dispatch_g(bool group, const D3Args& a, const CUtensorMap* maps, size_t smem, int grid,
                         cudaStream_t st) {
  return group ? d3_launch_t<MT, CH, true>(a, maps, smem, grid, st)
               : d3_launch_t<MT, CH, false>(a, maps, smem, grid, st);
}

template <int MT>
static int d3_dispatch_c(int ch, bool group, const D3Args& a, const CUtensorMap* maps, size_t smem, int grid,
                         cudaStream_t st) {
  switch (ch) {
    case 1: return d3_dispatch_g<MT, 1>(group, a, maps, smem, grid, st);
    case 2: return d3_dispatch_g<MT, 2>(group, a, maps, smem, grid, st);
    case 3: return d3_dispatch_g<MT, 3>(group, a, maps, smem, grid, st);
    default: return d3_dispatch_g<MT, 4>(group, a, maps, smem, grid, st);
  }
}

size_t decode3_tf_bytes() { return (size_t)D3_MAXE * 16 * 16 * sizeof(float); }

int launch_decode3(const LayerView& Lv, const __nv_bfloat16* x, int M, __nv_bfloat16* y, WsHeader* hdr, void* tf,
                   float* gate_out, int* mask_count, bool ec_only, cudaStream_t st) {
  if (M < 1 || M > 16) return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "decode path needs 1 <= M <= 16 (M=%d)", M);
  const int MT = M <= 8 ? 8 : 16;
  const int gk = Lv.r > 0 ? Lv.gate_kind : 0;
  const D3Plan& p = d3_plan(MT, Lv.K, Lv.N, Lv.r, Lv.group, gk, device_sm_count());
  if (p.why) return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "decode path: %s", p.why);
  if (ec_only && Lv.r == 0) return set_error(SPEAR_ERR_INVALID_ARG, "EC-only launch without an EC");
  D3Args a = {};
  a.scales = Lv.scales;
  a.x = x;
  a.y = y;
  a.gate_out = gate_out;
  a.mask_count = mask_count;
  a.hdr = hdr;
  a.tf = static_cast<float*>(tf);
  a.gw1 = Lv.gw1;
  a.gb1 = Lv.gb1;
  a.gw2 = Lv.gw2;
  a.gb2 = Lv.gb2;
  a.M = M;
  a.K = Lv.K;
  a.N = Lv.N;
  a.r = Lv.r;
  a.b_g = Lv.b_g;
  a.tau = Lv.tau;
  a.alpha = Lv.alpha;
  a.CS = p.CS;
  a.G = p.NC * p.CS;
  a.KTC = p.KTC;
  a.ES = Lv.r > 0 ? p.ES : 0;
  a.gate_item = Lv.r > 0 ? p.gate_item : 0;
  a.nslot = p.nslot;
  a.slot = p.slot;
  a.own_cap = p.own_cap;
  a.ec_only = ec_only ? 1 : 0;
  a.gate_kind = gk;
  a.gate_h = Lv.gate_h;
  const TestFault tf_ = test_fault();
  a.tag_skew = tf_.kernel == 1 ? 1 : 0;
  a.pub_wait = tf_.kernel == 1 ? tf_.cycles : kWaitCycles;
  for (int c = 0; c < p.NC; ++c) a.cl_tab[c] = p.cl_tab[c];
  CUtensorMap maps[5];
  memset(maps, 0, sizeof(maps));
  bool ok = tmap_packed_box(&maps[0], Lv.w, Lv.K, Lv.N, p.KTC, 1);
  if (ok && a.ES > 0) {
    ok = tmap_2d_bf16(&maps[1], Lv.agt, Lv.K, Lv.r + 1, 64, 16);
    if (ok) ok = tmap_2d_bf16(&maps[2], Lv.agt, Lv.K, Lv.r + 1, 64 * p.CH, 1, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (ok) ok = tmap_2d_bf16(&maps[3], Lv.bpt, Lv.r, Lv.N, Lv.r, 16, CU_TENSOR_MAP_SWIZZLE_NONE);
  }
  if (ok && Lv.group) ok = tmap_2d_f16(&maps[4], Lv.scales, Lv.N, Lv.K / 128, 16, p.KTC / 2);
  if (!ok) return set_error(SPEAR_ERR_CUDA, "cuTensorMapEncodeTiled failed (decode)");
  const int grid = p.NC * p.CS;
  return MT == 8 ? d3_dispatch_c<8>(p.CH, Lv.group != 0, a, maps, p.smem, grid, st)
                 : d3_dispatch_c<16>(p.CH, Lv.group != 0, a, maps, p.smem, grid, st);
}

}  // namespace spear
