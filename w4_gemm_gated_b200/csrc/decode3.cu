// Decode path (1 <= M <= 16) on sm_100a: W4 GEMV with the gated EC fused.
//
// SPEAR fuses the whole EC computation into the low-bit GEMM for the
// memory-bound decode phase (gist.science technical summary, section 2.2 A,
// decode at M = 1: one kernel, no inter-kernel launch on the critical path).
//
// One CTA per SM, 16 warps, each holding the activations of a 1/16 slice of K
// in registers (mma.sync B fragments) for the whole launch.  A CTA owns a few
// items, balanced over the SMs by the bytes they stream:
//   - at most one EC item, first: a 16-row strip of A^T, or the gate row w_g
//     (scalar gate), read from [A^T ; w_g];
//   - then 16-channel weight strips, each one unit of all of K.
// Every unit of the CTA is requested by TMA before the grid-dependency wait
// (nothing here depends on the previous kernel in the stream) into its own
// place in shared memory with its own barrier, so the weights stream while
// the previous kernel finishes, and nothing is reused or refilled.
//
// Per item each warp computes the partial of its K slice and writes it over
// the tiles it has just consumed; no warp waits for another inside the loop.
// The EC item is reduced (warp order) by the last warp to finish it, which
// publishes its rows t = x . A (or the gate logit x . w_g) for the live tokens
// to the workspace and raises the item's flag; one warp watches the flags
// between its items and fetches t as soon as every EC item is out.  At the
// end every warp builds g and gt = bf16(g t) (or the pages' per-rank gate),
// then warp j % 16 adds the 16 partials of strip j in warp order and stores
// y = bf16(s (acc + gt . B')) with 16-byte stores.
//
// Every wait is bounded; a timeout is reported in the workspace status word
// and every role falls through to the end, waiting there for the copies it
// issued (no early exit while copies into the CTA may be in flight).
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

constexpr int D3_NW = 16;                // warps, all of them consumers
constexpr int D3_THREADS = D3_NW * 32;
constexpr int D3_MAXCTA = 160;           // CTAs described in the kernel parameters
constexpr int D3_MAXU = 12;              // units of one CTA
constexpr int D3_MAXE = 9;               // EC items: 8 strips of A^T (r <= 128) + the gate row
constexpr int D3_ECU = D3_NW * 2048;     // an A^T-strip unit: one 64-wide k-tile of each warp's slice
constexpr size_t D3_SMEM_MAX = 232448;   // opt-in shared memory per CTA

struct D3Args {
  const __half* scales;
  const uint8_t* w;         // packed weights (spear_w4_pack layout)
  const __nv_bfloat16* x;
  __nv_bfloat16* y;
  float* gate_out;
  int* mask_count;
  WsHeader* hdr;
  float* tf;                // [D3_MAXE][MT][16] fp32: published EC rows (t, then the gate logit in row 0)
  const float *gw1, *gb1, *gw2, *gb2;
  const uint8_t* gate_row;   // row r of [A^T ; w_g]: w_g over all of K, bf16 (the gate item's one unit)
  int M, K, N, r;
  float b_g, tau, alpha;
  int G;                    // CTAs
  int ES;                   // strips of A^T (r / 16); 0 with the EC off
  int gate_item;            // 1: the gate row w_g is an EC item (scalar gate)
  int ec_only;              // 1: no weights; y += EC term in place (unfused path)
  int gate_kind, gate_h;
  int wunit;                // bytes of a weight unit: K/64 tiles of 512 B (+ group scales)
  int ubytes;               // unit space of the fullest CTA
  int own_cap;              // weight strips of the fullest CTA
  int tag_skew;             // test injection: publication flags are awaited at tag + skew (0 normally)
  long long pub_wait;       // bound of that wait (SM cycles)
  int dcheck_force;         // test hook: the y-store check fails (device-check build)
  const uint8_t* pf[3];     // the next call's buffers to warm in L2 (prefetch_next hint)
  unsigned long long pf_bytes[3];
  short4 tab[D3_MAXCTA];    // per CTA: EC item (-1 none), first weight strip, weight strips, 0
};

// Shared-memory carve-up (same on host and device).
struct D3Smem {
  uint32_t units, bps, scs, ts, gts, gpart, gv, rg, gp, stage, bars, total;
};
__host__ __device__ __forceinline__ uint32_t d3_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }
// rank-gate parameters W1 [h][r], W2 [r][h], b1 [h], b2 [r] fp32, staged at kernel start
__host__ __device__ __forceinline__ uint32_t d3_gp_bytes(int r, int h) { return (uint32_t)(2 * h * r + h + r) * 4; }
__host__ __device__ __forceinline__ D3Smem d3_smem(int MT, int ubytes, int own_cap, int r, int gate_kind, int gate_h) {
  D3Smem s;
  uint32_t off = 0;
  s.units = off;  // the CTA's units, each at a 1024-byte boundary
  off += d3_up(ubytes, 1024);
  s.bps = off;  // B' rows of the CTA's strips [own][16][r] bf16
  off += d3_up(own_cap * 32 * r, 128);
  s.scs = off;  // per-channel scales of its strips [own][16] fp16
  off += d3_up(own_cap * 32, 128);
  s.ts = off;  // t [MT][r] fp32, then the gate logits [MT]
  off += r > 0 ? d3_up((MT * r + MT) * 4, 16) : 0;
  s.gts = off;  // gt [MT][r + 8] bf16
  off += r > 0 ? d3_up(MT * (r + 8) * 2, 16) : 0;
  s.gpart = off;  // the warps' partial gate logits [16][MT] fp32
  off += D3_NW * MT * 4;
  s.gv = off;  // per-token gate g [MT] fp32
  off += 64;
  s.rg = off;  // rank gate: hidden [MT][32] and gamma [MT][r] fp32
  off += gate_kind == 1 ? d3_up(MT * (32 + r) * 4, 16) : 0;
  s.gp = off;  // rank gate: its parameters (16-byte multiples: h in {8, 16, 32}, r a multiple of 16)
  off += gate_kind == 1 ? d3_gp_bytes(r, gate_h) : 0;
  s.stage = off;  // per warp [MT tokens][16 channels] bf16
  off += D3_NW * MT * 32;
  s.bars = off;  // unit barriers, partials complete, epilogue operands, fetched t, gt ready
  off += (2 * D3_MAXU + 3) * 8;
  s.total = off + 1024;  // base alignment slack
  return s;
}
// Offset of unit u: the EC item's units first (n_ecu of ecu bytes), then weight units.
__host__ __device__ __forceinline__ uint32_t d3_unit_off(int u, int n_ecu, int ecu, int wunit) {
  return u < n_ecu ? (uint32_t)u * ecu : (uint32_t)n_ecu * ecu + (uint32_t)(u - n_ecu) * wunit;
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

// The same with the scalar gate, gt formed by the warp itself from t and the
// gate logit in shared memory (ts [MT][r], logits at ts[MT r + m]): the words
// it would have read from gt, bf16(g t) with g = sigmoid(logit + b_g), zero
// for padded tokens, in the same arithmetic as the gt builder.
template <int MT, int S, int NCH>
__device__ __forceinline__ void d3_ecterm_scalar(const __nv_bfloat16* bp, const float* ts, int M, float b_g, int r,
                                                 int lane, float (&acc)[MT / 8][4]) {
  constexpr int NT = MT / 8;
  const int rho = lane >> 2, c = lane & 3;
  float g[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int m = nt * 8 + rho;
    g[nt] = m < M ? sigmoidf_(ts[MT * r + m] + b_g) : 0.f;
  }
#pragma unroll
  for (int ch = 0; ch < NCH; ++ch) {
    uint32_t b0[8], b1[8], gw[NT][8];
    d3_lds_words<S>(bp + rho * r + 64 * ch + 4 * S * c, b0);
    d3_lds_words<S>(bp + (rho + 8) * r + 64 * ch + 4 * S * c, b1);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int m = nt * 8 + rho;
      const float2* tv = reinterpret_cast<const float2*>(ts + m * r + 64 * ch + 4 * S * c);
#pragma unroll
      for (int i = 0; i < 2 * S; ++i) {
        const float2 t2 = tv[i];
        gw[nt][i] = m < M ? pack_bf16x2(g[nt] * t2.x, g[nt] * t2.y) : 0u;
      }
    }
#pragma unroll
    for (int s2 = 0; s2 < S; ++s2) {
      const uint32_t af[4] = {b0[2 * s2], b1[2 * s2], b0[2 * s2 + 1], b1[2 * s2 + 1]};
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(acc[nt], af, gw[nt][2 * s2], gw[nt][2 * s2 + 1]);
    }
  }
}

template <int MT>
__device__ __forceinline__ void d3_ecterm_scalar_r(const __nv_bfloat16* bp, const float* ts, int M, float b_g, int r,
                                                   int lane, float (&acc)[MT / 8][4]) {
  if (r == 16)
    d3_ecterm_scalar<MT, 1, 1>(bp, ts, M, b_g, r, lane, acc);
  else if (r == 32)
    d3_ecterm_scalar<MT, 2, 1>(bp, ts, M, b_g, r, lane, acc);
  else if (r == 64)
    d3_ecterm_scalar<MT, 4, 1>(bp, ts, M, b_g, r, lane, acc);
  else
    d3_ecterm_scalar<MT, 4, 2>(bp, ts, M, b_g, r, lane, acc);
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

__device__ __forceinline__ uint32_t atom_add_acqrel_cta(int* p, int v) {
  uint32_t old;
  asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(smem_u32(p)), "r"(v) : "memory");
  return old;
}

// Gate and gt for the live tokens (every thread of the CTA; t and the gate
// logits are in shared memory), then the reported gate and mask count (CTA 0).
// Scalar gate: g = sigmoid(logit + b_g), gt = bf16(g t).  The pages' per-rank
// gate: u = relu(W1 t + b1), gamma = sigmoid(W2 u + b2), gt = bf16(alpha gamma t),
// reported gate = mean of gamma (a fixed lane-strided then shuffle-tree
// order).  Padded tokens get zero rows.
//
// What the gate builder reads of the launch's arguments, passed by value: an
// out-of-line callee reading the kernel's parameter block through a reference
// paid microseconds of load latency before its first instruction of work.
struct D3Gate {
  float* gate_out;
  int* mask_count;
  WsHeader* hdr;
  const float *gw1, *gb1, *gw2, *gb2;
  int M, r, gate_kind, gate_h, ubytes, own_cap;
  float b_g, alpha, tau;
};
__device__ __forceinline__ D3Gate d3_gate_args(const D3Args& a) {
  D3Gate g;
  g.gate_out = a.gate_out;
  g.mask_count = a.mask_count;
  g.hdr = a.hdr;
  g.gw1 = a.gw1;
  g.gb1 = a.gb1;
  g.gw2 = a.gw2;
  g.gb2 = a.gb2;
  g.M = a.M;
  g.r = a.r;
  g.gate_kind = a.gate_kind;
  g.gate_h = a.gate_h;
  g.ubytes = a.ubytes;
  g.own_cap = a.own_cap;
  g.b_g = a.b_g;
  g.alpha = a.alpha;
  g.tau = a.tau;
  return g;
}

template <int MT>
__device__ __noinline__ void d3_build_gate(const D3Gate a, uint8_t* sm, volatile int* abortp) {
  const D3Smem SL = d3_smem(MT, a.ubytes, a.own_cap, a.r, a.gate_kind, a.gate_h);
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
    float* hid = reinterpret_cast<float*>(sm + SL.rg);  // [MT][32]
    float* gam = hid + MT * 32;                         // [MT][r]
    // the parameters, staged in shared memory at kernel start (long landed:
    // the wait returns at once; a failed wait only leaves this CTA's gate
    // unused, the strips' own waits then stop)
    const float* gp = reinterpret_cast<const float*>(sm + SL.gp);
    const float* W1 = gp;
    const float* W2 = gp + h * r;
    const float* B1 = gp + 2 * h * r;
    const float* B2 = B1 + h;
    d3_wait(reinterpret_cast<uint64_t*>(sm + SL.bars) + 2 * D3_MAXU, 0, abortp, a.hdr);
    // u = relu(W1 t + b1): a team of tpi threads (a power of two, as many as
    // the block holds) per (token, hidden) item, each over j = sub, sub + tpi,
    // ... started at an item-dependent offset so that a warp's W1 and t reads
    // fall in different banks, then a fixed shuffle tree over the team
    {
      const int items = a.M * h;
      int tpi = 32;
      while (tpi > 1 && (tpi * items > D3_THREADS || r % tpi)) tpi >>= 1;
      for (int base = 0; base < items * tpi; base += D3_THREADS) {
        const int idx = base + tid, item = idx / tpi, sub = idx - item * tpi;
        float z = 0.f;
        if (item < items) {
          const int m = item / h, i = item - m * h;
          const float* w1 = W1 + i * r;
          const float* tv = ts + m * r;
          // j = sub + tpi (i + k) mod r for k = 0, 1, ...: every j = sub mod tpi
          // once (tpi divides r), from an item-dependent start, wrapped by a
          // subtraction rather than a division; two alternating sums
          const int n = r / tpi;
          int j = (i * tpi) % r + sub;
          float z0 = 0.f, z1 = 0.f;
          for (int k = 0; k < n; k += 2) {
            z0 = fmaf(w1[j], tv[j], z0);
            j += tpi;
            if (j >= r) j -= r;
            if (k + 1 < n) {
              z1 = fmaf(w1[j], tv[j], z1);
              j += tpi;
              if (j >= r) j -= r;
            }
          }
          z = z0 + z1;
        }
        for (int o = tpi >> 1; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
        if (item < items && sub == 0) {
          const int m = item / h, i = item - m * h;
          hid[m * 32 + i] = fmaxf(z + B1[i], 0.f);
        }
      }
    }
    __syncthreads();
    // gamma = sigmoid(W2 u + b2), gt = bf16(alpha gamma t): one thread per
    // (token, rank) item, its W2 row and u read from an item-dependent offset
    for (int idx = tid; idx < MT * r; idx += D3_THREADS) {
      const int m = idx / r, j = idx - m * r;
      float gam_v = 0.f;
      if (m < a.M) {
        const float* w2 = W2 + j * h;
        const float* uv = hid + m * 32;
        float z0 = 0.f, z1 = 0.f;
        for (int k = 0; k < h; k += 2) {
          const int i0 = (k + j) & (h - 1), i1 = (k + 1 + j) & (h - 1);
          z0 = fmaf(w2[i0], uv[i0], z0);
          z1 = fmaf(w2[i1], uv[i1], z1);
        }
        gam_v = sigmoidf_(B2[j] + (z0 + z1));
      }
      gam[m * r + j] = gam_v;
      gts[m * gs + j] = __float2bfloat16_rn(m < a.M ? a.alpha * gam_v * ts[m * r + j] : 0.f);
    }
    __syncthreads();
    // g = mean of gamma: warp m sums token m's r values (lane-strided, then a
    // fixed shuffle tree)
    {
      const int warp = tid >> 5, lane = tid & 31;
      if (warp < MT) {
        float sgm = 0.f;
        for (int j = lane; j < r; j += 32) sgm += gam[warp * r + j];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sgm += __shfl_xor_sync(0xffffffffu, sgm, o);
        if (lane == 0) gv[warp] = warp < a.M ? sgm / (float)r : 0.f;
      }
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

// Weight strip j of this CTA, by one warp: the 16 warp partials (left over
// each warp's own tiles of the strip's unit) added in warp order, + gt . B',
// scaled, rounded to bf16 and stored with 16-byte stores (added to y in
// place in EC-only mode, where the strip has no weight partials).
template <int MT, bool GROUP>
__device__ __noinline__ void d3_finish_strip(const D3Args& a, uint8_t* sm, int j, int p, const uint8_t* ubase, int CH,
                                             int lane, int warp) {
  constexpr int NT = MT / 8;
  const D3Smem SL = d3_smem(MT, a.ubytes, a.own_cap, a.r, a.gate_kind, a.gate_h);
  const __nv_bfloat16* bps = reinterpret_cast<const __nv_bfloat16*>(sm + SL.bps);
  const __half* scs = reinterpret_cast<const __half*>(sm + SL.scs);
  const __nv_bfloat16* gts = reinterpret_cast<const __nv_bfloat16*>(sm + SL.gts);
  const int rho = lane >> 2, c = lane & 3;
  float tot[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) tot[nt][0] = tot[nt][1] = tot[nt][2] = tot[nt][3] = 0.f;
  if (!a.ec_only) {
#pragma unroll 4
    for (int w2 = 0; w2 < D3_NW; ++w2)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const float4 v = *reinterpret_cast<const float4*>(ubase + w2 * CH * 512 + nt * 512 + lane * 16);
        tot[nt][0] += v.x;
        tot[nt][1] += v.y;
        tot[nt][2] += v.z;
        tot[nt][3] += v.w;
      }
  }
  if (a.ES > 0) {
    if (a.gate_kind == 0)
      d3_ecterm_scalar_r<MT>(bps + (size_t)j * 16 * a.r, reinterpret_cast<const float*>(sm + SL.ts), a.M, a.b_g, a.r,
                             lane, tot);
    else
      d3_ecterm_r<MT>(bps + (size_t)j * 16 * a.r, gts, a.r, lane, tot);
  }
  float s0 = 1.f, s1 = 1.f;
  if (!GROUP) {
    s0 = __half2float(scs[j * 16 + rho]);
    s1 = __half2float(scs[j * 16 + rho + 8]);
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
  if (m < a.M && SPEAR_DCHECK(16 * p + 16 <= a.N && !a.dcheck_force, a.hdr)) {
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

// Whether every EC item of this launch is published (each lane checks every
// flag itself, with acquire ordering for its own later reads of the rows).
// Every EC item's flag at this launch's tag?  Lane e reads flag e (all in
// flight together, one round trip), the warp votes, and once all are set each
// lane's acquire fence orders the rows read after it.
__device__ __forceinline__ bool d3_flags_ready(const D3Args& a, int tag) {
  const int ne = a.ES + a.gate_item;  // <= D3_MAXE <= 32
  bool mine = true;
  if ((int)(threadIdx.x & 31) < ne) {
    int v;
    asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(&a.hdr->d3_flag[threadIdx.x & 31]) : "memory");
    mine = v == tag + a.tag_skew;
  }
  const bool all = __all_sync(0xffffffffu, mine);
  if (all) asm volatile("fence.acq_rel.gpu;" ::: "memory");
  __syncwarp();
  return all;
}

// The published rows of the live tokens into shared memory by cp.async, one
// warp: t rows [ES][MT][16] -> ts [m][r] (16-byte chunks), gate logits (row 0
// of item ES) -> ts[MT r + m]; completion counted on `bar` (32 arrivals).
template <int MT>
__device__ __forceinline__ void d3_fetch_t(const D3Args& a, float* ts, uint64_t* bar, int lane) {
  const int nv = a.ES * a.M * 4;
  for (int idx = lane; idx < nv; idx += 32) {
    const int e = idx / (a.M * 4), rem = idx - e * a.M * 4;
    const int m = rem >> 2, r0 = (rem & 3) * 4;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(ts + m * a.r + 16 * e + r0)),
                 "l"(a.tf + (size_t)e * MT * 16 + rem * 4)
                 : "memory");
  }
  if (a.gate_item && lane < a.M)
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(ts + MT * a.r + lane)),
                 "l"(a.tf + (size_t)a.ES * MT * 16 + lane * 16)
                 : "memory");
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

template <int MT, int CH, bool GROUP>
__global__ void __launch_bounds__(D3_THREADS, 1)
    decode3_kernel(const __grid_constant__ D3Args a, const __grid_constant__ CUtensorMap tm_w,
                   const __grid_constant__ CUtensorMap tm_agt, const __grid_constant__ CUtensorMap tm_gate,
                   const __grid_constant__ CUtensorMap tm_bp, const __grid_constant__ CUtensorMap tm_gs) {
  constexpr int NT = MT / 8;
  constexpr unsigned FULL = 0xffffffffu;
  constexpr int KT = 16 * CH;  // k-tiles of all of K
  extern __shared__ uint8_t smem_raw[];
  __shared__ int s_abort, s_eccnt, s_fetched;
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const D3Smem SL = d3_smem(MT, a.ubytes, a.own_cap, a.r, a.gate_kind, a.gate_h);
  uint8_t* units = sm + SL.units;
  __nv_bfloat16* bps = reinterpret_cast<__nv_bfloat16*>(sm + SL.bps);
  __half* scs = reinterpret_cast<__half*>(sm + SL.scs);
  float* ts = reinterpret_cast<float*>(sm + SL.ts);
  float* gpart = reinterpret_cast<float*>(sm + SL.gpart);
  uint64_t* ubar = reinterpret_cast<uint64_t*>(sm + SL.bars);
  uint64_t* pbar = ubar + D3_MAXU;  // every warp's partial of unit u written (16 arrivals)
  uint64_t* epibar = pbar + D3_MAXU;
  uint64_t* tsbar = epibar + 1;
  uint64_t* gtbar = tsbar + 1;      // gt built (scalar gate)
  __nv_bfloat16* gts = reinterpret_cast<__nv_bfloat16*>(sm + SL.gts);
  float* gv = reinterpret_cast<float*>(sm + SL.gv);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rho = lane >> 2, c = lane & 3;
  const short4 ct = a.tab[blockIdx.x];
  const int ec_item = ct.x, w_lo = ct.y, n_w = ct.z;
  const bool has_ec = a.ES > 0;
  const int n_ecu = ec_item < 0 ? 0 : (ec_item < a.ES ? CH : 1);  // units of the EC item
  const int ecu = ec_item < a.ES ? D3_ECU : CH * D3_NW * 128;    // bytes of one of them
  const int U = n_ecu + (a.ec_only ? 0 : n_w);
  volatile int* abortp = &s_abort;
  auto ubase = [&](int u) { return units + d3_unit_off(u, n_ecu, ecu, a.wunit); };

  if (warp == 0) {
    for (int u = lane; u < U; u += 32) {
      mbar_init(&ubar[u], 1);
      mbar_init(&pbar[u], D3_NW);
    }
    if (lane == 0) {
      mbar_init(epibar, 1);
      mbar_init(tsbar, 32);
      mbar_init(gtbar, 1);
      s_abort = 0;
      s_eccnt = 0;
      s_fetched = 0;
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    __syncwarp();
    // epilogue operands of the CTA's strips: B' rows and per-channel scales
    // (and the rank gate's parameters, which every CTA's gate builder reads)
    const uint32_t gp_bytes = has_ec && a.gate_kind == 1 ? d3_gp_bytes(a.r, a.gate_h) : 0u;
    const uint32_t epi_bytes = (uint32_t)n_w * ((has_ec ? 32u * a.r : 0u) + (GROUP ? 0u : 32u)) + gp_bytes;
    if (lane == 0) {
      if (epi_bytes)
        mbar_arrive_tx(epibar, epi_bytes);
      else
        mbar_arrive(epibar);
    }
    __syncwarp();
    if (gp_bytes && lane < 4) {
      const int h = a.gate_h, r = a.r;
      float* gp = reinterpret_cast<float*>(sm + SL.gp);
      const float* src = lane == 0 ? a.gw1 : lane == 1 ? a.gw2 : lane == 2 ? a.gb1 : a.gb2;
      const int off = lane == 0 ? 0 : lane == 1 ? h * r : lane == 2 ? 2 * h * r : 2 * h * r + h;
      const int n = lane < 2 ? h * r : lane == 2 ? h : r;
      bulk_g2s(gp + off, src, (uint32_t)n * 4, epibar);
    }
    for (int j = lane; j < n_w; j += 32) {
      const int p = w_lo + j;
      if (has_ec) tma_load_2d(smem_u32(bps + (size_t)j * 16 * a.r), &tm_bp, epibar, 0, 16 * p);
      if (!GROUP) bulk_g2s(scs + j * 16, a.scales + 16 * p, 32, epibar);
    }
    // every unit: nothing here depends on the previous kernel in the stream.
    // The EC item's units go first: the rows it publishes are on every CTA's
    // critical path.  An A^T unit (k-tile u of every warp's slice of a
    // 16-row strip) is one 32 KB box of a 3-D map [slice][row][k]; the gate
    // row is one contiguous run (TMA instructions cost the issuing thread tens
    // of ns each, so 16 small boxes per unit delayed the EC item).
    for (int u = lane; u < n_ecu; u += 32) {
      uint64_t* bar = &ubar[u];
      if (ec_item < a.ES) {
        mbar_arrive_tx(bar, D3_ECU);
        tma_load_3d(smem_u32(ubase(u)), &tm_agt, bar, u * 64, 16 * ec_item, 0);
      } else {
        mbar_arrive_tx(bar, D3_NW * CH * 128);
        bulk_g2s(ubase(u), a.gate_row, D3_NW * CH * 128, bar);
      }
    }
    // A weight unit (strip p, all of K) is one contiguous run of the packed
    // array: it goes as 1-D bulk copies of 8 KB issued from several lanes
    // (measured much faster per SM than one large tensor box).
    constexpr int PIECE = 8192, NPIECE = KT * 512 / PIECE;
    for (int u = n_ecu + lane; u < U; u += 32) mbar_arrive_tx(&ubar[u], a.wunit);
    __syncwarp();
    for (int i = lane; i < (U - n_ecu) * NPIECE; i += 32) {
      const int u = n_ecu + i / NPIECE, k = i - (i / NPIECE) * NPIECE;
      const int p = w_lo + (u - n_ecu);
      bulk_g2s(ubase(u) + k * PIECE, a.w + ((size_t)p * KT * 512 + (size_t)k * PIECE), PIECE, &ubar[u]);
      if (GROUP && k == 0) tma_load_2d(smem_u32(ubase(u)) + KT * 512, &tm_gs, &ubar[u], 16 * p, 0);
    }
  }
  if (warp == 1) {
    // the next call's layer into L2 (hint): this CTA's 1/G slice of each buffer,
    // in 16 KB pieces, 16-byte aligned
    for (int i = 0; i < 3; ++i) {
      const unsigned long long n = a.pf_bytes[i];
      if (!n) continue;
      const unsigned long long beg = (n * blockIdx.x / a.G) & ~15ull, end = (n * (blockIdx.x + 1) / a.G) & ~15ull;
      for (unsigned long long off = beg + (unsigned long long)lane * 16384; off < end; off += 32ull * 16384) {
        const unsigned long long len = end - off < 16384 ? end - off : 16384;
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a.pf[i] + off), "r"((uint32_t)len)
                     : "memory");
      }
    }
  }
  __syncthreads();
  // the next kernel in the stream may start its own requests as SMs free up
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // x, y and the workspace may belong to the previous kernel in the stream
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (!has_ec && blockIdx.x == 0 && warp == 1) {
    if (a.gate_out && lane < a.M) a.gate_out[lane] = 0.f;
    if (a.mask_count && lane == 0) *a.mask_count = a.M;
  }

  // activations of this warp's k slice as B fragments: word i of xf[t][nt]
  // = x[nt*8 + rho][64 (w CH + t) + 16c + 2i .. + 1]; requested before the
  // launch tag, whose read then overlaps them
  uint32_t xf[CH][NT][8];
#pragma unroll
  for (int t = 0; t < CH; ++t)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int m = nt * 8 + rho;
      uint4 v0 = make_uint4(0u, 0u, 0u, 0u), v1 = v0;
      if (m < a.M) {
        const uint4* src = reinterpret_cast<const uint4*>(a.x + (size_t)m * a.K + (size_t)(warp * CH + t) * 64 + 16 * c);
        v0 = __ldcg(src);
        v1 = __ldcg(src + 1);
      }
      xf[t][nt][0] = v0.x; xf[t][nt][1] = v0.y; xf[t][nt][2] = v0.z; xf[t][nt][3] = v0.w;
      xf[t][nt][4] = v1.x; xf[t][nt][5] = v1.y; xf[t][nt][6] = v1.z; xf[t][nt][7] = v1.w;
    }
  const int tag = *reinterpret_cast<volatile int*>(&a.hdr->d2_epoch) + 1;
  // every warp has its tag before any warp of this CTA can count the CTA as
  // done with this launch's rows (which lets the epoch advance)
  __syncthreads();
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
  // one warp watches the flags between its items and fetches t (CTAs without
  // strips need no t, except CTA 0, which reports the gates)
  const bool needs_t = has_ec && (n_w > 0 || blockIdx.x == 0);
  const bool fetcher = needs_t && warp == D3_NW - 1;
  if (ec_item >= 0) {
    // the EC item: this warp's partial, then the last warp to finish it adds
    // the 16 partials (warp order) and publishes the rows of the live tokens
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
    if (ec_item < a.ES) {
#pragma unroll
      for (int t = 0; t < CH; ++t) {
        ok = ok && __all_sync(FULL, d3_wait(&ubar[t], 0, abortp, a.hdr));
        if (ok) d3_ec_tile<NT>(ubase(t) + warp * 2048, xf[t], lane, acc);
      }
      // over this warp's own (consumed) tile of unit 0
      __syncwarp();
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        *reinterpret_cast<float4*>(ubase(0) + warp * 2048 + nt * 512 + lane * 16) =
            make_float4(acc[nt][0], acc[nt][1], acc[nt][2], acc[nt][3]);
    } else {
      ok = ok && __all_sync(FULL, d3_wait(&ubar[0], 0, abortp, a.hdr));
      if (ok) {
#pragma unroll
        for (int t = 0; t < CH; ++t) d3_gate_tile<NT>(ubase(0) + warp * CH * 128 + t * 128, xf[t], lane, acc);
      }
      // row 0 only: lanes 0..3 hold tokens nt*8 + 2c and + 1
      if (rho == 0) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          gpart[warp * MT + nt * 8 + 2 * c] = acc[nt][0];
          gpart[warp * MT + nt * 8 + 2 * c + 1] = acc[nt][1];
        }
      }
    }
    __syncwarp();
    int last = 0;
    if (lane == 0) last = atom_add_acqrel_cta(&s_eccnt, 1) == D3_NW - 1 ? 1 : 0;
    last = __shfl_sync(FULL, last, 0);
    if (last && ok && SPEAR_DCHECK(ec_item < D3_MAXE, a.hdr)) {
      float* dst = a.tf + (size_t)ec_item * MT * 16;
      if (ec_item < a.ES) {
        float tot[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) tot[nt][0] = tot[nt][1] = tot[nt][2] = tot[nt][3] = 0.f;
        for (int w2 = 0; w2 < D3_NW; ++w2)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const float4 v = *reinterpret_cast<const float4*>(ubase(0) + w2 * 2048 + nt * 512 + lane * 16);
            tot[nt][0] += v.x;
            tot[nt][1] += v.y;
            tot[nt][2] += v.z;
            tot[nt][3] += v.w;
          }
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
      } else if (lane < a.M) {
        float g = 0.f;
        for (int w2 = 0; w2 < D3_NW; ++w2) g += gpart[w2 * MT + lane];
        dst[lane * 16] = g;
      }
      // the warp barrier orders every lane's rows before lane 0's release
      __syncwarp();
      if (lane == 0) st_release_gpu(&a.hdr->d3_flag[ec_item], tag);
    }
  }
  // weight strips: every warp's partial over its own consumed tiles
  if (!a.ec_only) {
    for (int j = 0; j < n_w && ok; ++j) {
      const int u = n_ecu + j;
      ok = __all_sync(FULL, d3_wait(&ubar[u], 0, abortp, a.hdr));
      if (!ok) break;
      float acc[NT][4];
      uint8_t* base = ubase(u);
      d3_w_item<MT, CH, GROUP>(base, KT, warp, lane, xf, xsA, xsB, acc);
      __syncwarp();  // every lane's reads of this warp's tiles are done
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        *reinterpret_cast<float4*>(base + warp * CH * 512 + nt * 512 + lane * 16) =
            make_float4(acc[nt][0], acc[nt][1], acc[nt][2], acc[nt][3]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&pbar[u]);
      if (fetcher && !s_fetched && d3_flags_ready(a, tag)) {
        d3_fetch_t<MT>(a, ts, tsbar, lane);
        if (lane == 0) s_fetched = 1;
        __syncwarp();
      }
    }
  }
  if (fetcher && ok && !s_fetched) {
    // the rest of the flags (bounded), then the rows
    const long long t0 = clock64();
    uint32_t ns = 32;
    while (!d3_flags_ready(a, tag)) {
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
      ns = ns < 256 ? ns * 2 : 256;
    }
    if (ok) {
      d3_fetch_t<MT>(a, ts, tsbar, lane);
      if (lane == 0) s_fetched = 1;
      __syncwarp();
    }
  }
  if (fetcher && s_fetched) ok = __all_sync(FULL, d3_wait(tsbar, 0, abortp, a.hdr));
  if (fetcher && ok && a.gate_kind == 0 && blockIdx.x == 0) {
    // scalar gate, CTA 0 only, which reports the gates: g = sigmoid(logit +
    // b_g) and gt = bf16(g t) for the live tokens (zero rows for the padded
    // ones).  The strip warps form their own gt words from t once it has
    // landed (they wait on tsbar), so no CTA waits for this warp.
    const int gs = a.r + 8, half = a.r / 2;
    if (lane < MT) gv[lane] = lane < a.M ? sigmoidf_(ts[MT * a.r + lane] + a.b_g) : 0.f;
    __syncwarp();
    for (int idx = lane; idx < MT * half; idx += 32) {
      const int m = idx / half, j = 2 * (idx - m * half);
      const float g = gv[m];
      *reinterpret_cast<uint32_t*>(gts + m * gs + j) =
          m < a.M ? pack_bf16x2(g * ts[m * a.r + j], g * ts[m * a.r + j + 1]) : 0u;
    }
    if (blockIdx.x == 0) {
      const bool valid = lane < a.M;
      const float g = lane < MT ? gv[lane] : 0.f;
      if (a.gate_out && valid) a.gate_out[lane] = g;
      const unsigned below = __ballot_sync(FULL, valid && g < a.tau);
      if (a.mask_count && lane == 0) *a.mask_count = __popc(below);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(gtbar);
  }

  // ------------------------------------------------------------------ end phase
  bool live = true;
  if (has_ec && a.gate_kind == 1) {
    // the pages' per-rank gate: built by the whole CTA (its MLP is the bulk of it)
    __syncthreads();
    // Read once by every thread between two barriers: nothing writes the flag
    // before the gate block's last barrier, so the branch below is uniform.
    live = !*abortp;
    if (needs_t && live) d3_build_gate<MT>(d3_gate_args(a), sm, abortp);
  }
  if (live) {
    // strip j by warp j % 16, as soon as its 16 partials (and gt) are ready
    bool eok = n_w > warp ? __all_sync(FULL, d3_wait(epibar, 0, abortp, a.hdr)) : false;
    for (int j = warp; j < n_w && eok; j += D3_NW) {
      if (!a.ec_only) eok = __all_sync(FULL, d3_wait(&pbar[n_ecu + j], 0, abortp, a.hdr));
      if (eok && has_ec && a.gate_kind == 0) eok = __all_sync(FULL, d3_wait(tsbar, 0, abortp, a.hdr));
      if (eok) d3_finish_strip<MT, GROUP>(a, sm, j, w_lo + j, ubase(n_ecu + j), CH, lane, warp);
    }
  }
  // every CTA reads this launch's rows at most once; the last one to be done
  // with them advances the epoch (CTAs that never read them count as well)
  const bool t_done = needs_t ? (fetcher && ok && s_fetched) : (warp == 0);
  if (has_ec && t_done && lane == 0 && !*abortp) {
    if (atomicAdd(&a.hdr->gt_obs, 1) == a.G - 1) {
      a.hdr->gt_obs = 0;
      a.hdr->d2_epoch = tag;
    }
  }
  if (warp == 0) {
    // no copy may still write into this CTA's shared memory when it exits
    // (all complete already unless a role gave up early)
    for (int u = 0; u < U; ++u) d3_drain(&ubar[u], 0);
    d3_drain(epibar, 0);
    if (s_fetched) d3_drain(tsbar, 0);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
struct D3Plan {
  int MT, CH, G, ES, gate_item, wunit, ubytes, own_cap;
  size_t smem;
  const char* why;  // non-null: this kernel cannot run the shape
  std::vector<short4> tab;
};

static D3Plan make_d3_plan(int MT, int K, int N, int r, int group, int gate_kind, int gate_h, int sms) {
  D3Plan p = {};
  p.MT = MT;
  p.why = nullptr;
  const int KT = K / 64;
  if (KT % D3_NW || KT / D3_NW > 4 || KT / D3_NW < MT / 8) {
    p.why = "K must be 1024, 2048, 3072 or 4096 (2048 or more at M > 8)";
    return p;
  }
  p.CH = KT / D3_NW;
  p.ES = r / 16;
  p.gate_item = r > 0 && gate_kind == SPEAR_GATE_SCALAR ? 1 : 0;
  const int n_ec = p.ES + p.gate_item;
  const int NS = N / 16;
  p.wunit = KT * 512 + (group ? KT * 16 : 0);
  int G = std::min(sms, NS + n_ec);
  G = std::min(G, D3_MAXCTA);
  if (G < n_ec) {
    p.why = "too few SMs for the EC items";
    return p;
  }
  p.G = G;
  // balance streamed bytes: weight strip KT * 512, A^T strip 4x that, gate row 1/4
  const long long cw = 4, ce = 16, cg = 1;
  const long long C = cw * NS + ce * p.ES + cg * p.gate_item;
  p.tab.resize(G);
  int w0 = 0, own = 1, ub = 0;
  long long cum = 0;
  for (int c = 0; c < G; ++c) {
    const int e = c < n_ec ? c : -1;
    const long long ec_cost = e < 0 ? 0 : (e < p.ES ? ce : cg);
    int nw;
    if (c == G - 1) {
      nw = NS - w0;
    } else {
      const long long target = C * (c + 1) / G;
      nw = (int)std::max<long long>(0, (target - cum - ec_cost + cw / 2) / cw);
      nw = std::min(nw, NS - w0);
    }
    p.tab[c] = make_short4((short)e, (short)w0, (short)nw, 0);
    cum += ec_cost + cw * nw;
    w0 += nw;
    own = std::max(own, nw);
    const int n_ecu = e < 0 ? 0 : (e < p.ES ? p.CH : 1);
    const int ecu = e < p.ES ? D3_ECU : p.CH * D3_NW * 128;
    if (n_ecu + nw > D3_MAXU) {
      p.why = "too many units per CTA for the decode kernel";
      return p;
    }
    ub = std::max(ub, (int)d3_unit_off(n_ecu + nw, n_ecu, ecu, p.wunit));
  }
  p.own_cap = own;
  p.ubytes = ub;
  p.smem = d3_smem(MT, ub, own, r, gate_kind, gate_h).total;
  if (p.smem > D3_SMEM_MAX) p.why = "a CTA's share does not fit in shared memory";
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
  opted = smem;
  return cudaSuccess;
}

// The plan for a shape (cached per device).
static const D3Plan& d3_plan(int MT, int K, int N, int r, int group, int gate_kind, int gate_h, int sms) {
  static std::mutex mu;
  static std::map<std::tuple<int, int, int, int, int, int, int, int, int>, D3Plan> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  if (gate_kind != 1) gate_h = 0;
  const auto key = std::make_tuple(dev, MT, K, N, r, group, gate_kind, gate_h, sms);
  std::lock_guard<std::mutex> lk(mu);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  return cache.emplace(key, make_d3_plan(MT, K, N, r, group, gate_kind, gate_h, sms)).first->second;
}

const char* decode3_unsupported(int M, int K, int N, int r, int group, int gate_kind, int gate_h) {
  if (M < 1 || M > 16) return "the decode kernel needs 1 <= M <= 16";
  return d3_plan(M <= 8 ? 8 : 16, K, N, r, group, r > 0 ? gate_kind : 0, gate_h, device_sm_count()).why;
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
  cudaLaunchAttribute attr[1];
  // programmatic dependent launch: this grid's CTAs may start (and request
  // their weights) while the previous kernel in the stream finishes; they
  // wait for it before touching x, y and the workspace
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
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

// [A^T ; w_g] ((r + 1) rows of K bf16) as a 3-D array [warp slice][row][k in
// the slice]: box (64 k, 16 rows, 16 slices) = k-tile u of every warp's slice
// of one 16-row strip, landing as [slice][row][64 k] with the 128-byte swizzle
// of the per-slice 2 KB tiles the EC item reads.
static bool d3_tmap_agt(CUtensorMap* m, const void* agt, int K, int r, int CH) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)CH * 64, (cuuint64_t)r + 1, (cuuint64_t)D3_NW};
  const cuuint64_t strides[2] = {(cuuint64_t)K * 2, (cuuint64_t)CH * 128};
  const cuuint32_t box[3] = {64, 16, D3_NW};
  const cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(agt), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t decode3_tf_bytes() { return (size_t)D3_MAXE * 16 * 16 * sizeof(float); }

int launch_decode3(const LayerView& Lv, const __nv_bfloat16* x, int M, __nv_bfloat16* y, WsHeader* hdr, void* tf,
                   float* gate_out, int* mask_count, bool ec_only, cudaStream_t st) {
  if (M < 1 || M > 16) return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "decode path needs 1 <= M <= 16 (M=%d)", M);
  const int MT = M <= 8 ? 8 : 16;
  const int gk = Lv.r > 0 ? Lv.gate_kind : 0;
  const D3Plan& p = d3_plan(MT, Lv.K, Lv.N, Lv.r, Lv.group, gk, Lv.gate_h, device_sm_count());
  if (p.why) return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "decode path: %s", p.why);
  if (ec_only && Lv.r == 0) return set_error(SPEAR_ERR_INVALID_ARG, "EC-only launch without an EC");
  if (MT == 8 && p.CH < 1) return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "decode path: K too small");
  D3Args a = {};
  a.scales = Lv.scales;
  a.w = Lv.w;
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
  a.G = p.G;
  a.ES = Lv.r > 0 ? p.ES : 0;
  a.gate_item = Lv.r > 0 ? p.gate_item : 0;
  a.ec_only = ec_only ? 1 : 0;
  a.gate_kind = gk;
  a.gate_h = Lv.gate_h;
  a.wunit = p.wunit;
  a.ubytes = p.ubytes;
  a.own_cap = p.own_cap;
  const TestFault tf_ = test_fault();
  a.tag_skew = tf_.kernel == 1 ? 1 : 0;
  a.pub_wait = tf_.kernel == 1 ? tf_.cycles : kWaitCycles;
  a.dcheck_force = test_force_check() == 1;
  for (int i = 0; i < 3; ++i) {
    a.pf[i] = static_cast<const uint8_t*>(Lv.pf[i]);
    a.pf_bytes[i] = Lv.pf_bytes[i];
  }
  for (int c = 0; c < p.G; ++c) a.tab[c] = p.tab[c];
  CUtensorMap maps[5];
  memset(maps, 0, sizeof(maps));
  const int KT = Lv.K / 64;
  bool ok = tmap_packed_box(&maps[0], Lv.w, Lv.K, Lv.N, KT, 1);
  if (ok && a.ES > 0) {
    ok = d3_tmap_agt(&maps[1], Lv.agt, Lv.K, Lv.r, p.CH);
    if (ok) ok = tmap_2d_bf16(&maps[3], Lv.bpt, Lv.r, Lv.N, Lv.r, 16, CU_TENSOR_MAP_SWIZZLE_NONE);
    a.gate_row = reinterpret_cast<const uint8_t*>(Lv.agt) + (size_t)Lv.r * Lv.K * 2;
  }
  if (ok && Lv.group) ok = tmap_2d_f16(&maps[4], Lv.scales, Lv.N, Lv.K / 128, 16, KT / 2);
  if (!ok) return set_error(SPEAR_ERR_CUDA, "cuTensorMapEncodeTiled failed (decode)");
  return MT == 8 ? d3_dispatch_c<8>(p.CH, Lv.group != 0, a, maps, p.smem, p.G, st)
                 : d3_dispatch_c<16>(p.CH, Lv.group != 0, a, maps, p.smem, p.G, st);
}

}  // namespace spear
