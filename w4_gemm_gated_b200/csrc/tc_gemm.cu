// Tensor-core path (M > 16): persistent tcgen05 W4A16 GEMM with the gated EC
// fused into the same kernel.
//
// SPEAR fuses the EC work into the low-bit GEMM (gist.science technical
// summary, section 2.2 A and B: the post-EC computation folded into the
// GEMM epilogue).  On sm_100a this kernel does, per 128-token x 256-channel
// output tile:
//   * a TMA producer warp streams the x tile (128 x 64 bf16, 128-byte
//     swizzle) and the packed int4 tile (256 channels x 64 k, 8 KB: sixteen
//     512-byte tiles of the packed layout, one 3-D tensor-map box);
//   * eight dequant warps turn the int4 tile into bf16 in shared memory, in
//     the UMMA canonical K-major 128-byte-swizzled layout (exact small
//     integers for per-channel scales; s * q rounded once for group scales);
//   * one MMA warp issues tcgen05.mma (kind::f16, M=128, N=256, K=16) into a
//     double-buffered fp32 accumulator in tensor memory;
//   * four epilogue warps read the accumulator with tcgen05.ld, apply the
//     per-channel scale and store bf16 y.
// The EC: the first tiles of the schedule are "projection tiles"
// [t | logit] = x . [A | w_g] (N = r+16 columns through the same pipeline);
// their epilogue applies the gate, writes gt = g * t (bf16) and raises an
// epoch-tagged flag per 128-token block.  Every output tile then runs
// ceil(r/64) extra K-steps, gt (128 x r) times (B')^T (256 x r), into the
// same accumulator (B' = B / s_n is folded once per layer, so s_n applies
// to the sum), so the EC costs neither a second kernel nor a pass over y.
//
// Schedules (a CTA per SM): with enough tiles, a persistent loop over whole
// tiles; while the tiles fill at most half the SMs, each tile's K split into
// S = 2, 4 or 8 parts whose fp32 partials each part sums for a 256/S-channel
// share; in between, stream-K, each SM an equal run of the tiles' k-steps,
// a tile finished by the CTA that holds its first k-steps (unit_info).
//
// Every wait on an mbarrier or a flag is bounded; on expiry the kernel
// records SPEAR_ERR_TIMEOUT and all roles leave their loops.
#include <cuda.h>

#include <map>
#include <mutex>
#include <tuple>

#include "common.cuh"
#include "kernels.h"
#include "tma.cuh"

namespace spear {

constexpr int TC_BM = 128;  // rows of one MMA (and of one TMEM accumulator)
constexpr int TC_BN = 256;
constexpr int TC_BK = 64;
// Tiles are BMT = 128 or 256 tokens (template): a 256-token tile runs two
// M = 128 MMAs per k-step into two accumulators, so each dequantised weight
// tile and each ring round trip feed twice the tensor-core work.
// Ring stages: as many as fit the 227 KB of shared memory (one stage is reused
// every TMA + dequant + MMA round trip): 4 at BMT = 128 (3 with the rank gate's
// parameters), 3 at BMT = 256.
constexpr int TC_STAGES = 4;
constexpr int TC_PREFETCH = 8;  // k-steps of L2 prefetch ahead of the TMA loads
constexpr int TC_THREADS = 14 * 32;  // producer, mma, 4 epilogue, 8 dequant warps
constexpr int TC_X_BYTES = TC_BM * TC_BK * 2;      // 16 KB: x rows of one MMA
constexpr int TC_B_BYTES = TC_BN * TC_BK * 2;      // 32 KB
constexpr int TC_P_BYTES = TC_BN * TC_BK / 2;      // 8 KB
__host__ __device__ constexpr int tc_stage_bytes(int bmt) { return bmt * TC_BK * 2 + TC_B_BYTES + TC_P_BYTES; }
__host__ __device__ constexpr int tc_smem(int nst, int bmt) {
  return nst * tc_stage_bytes(bmt) + 1024 /* barriers */ + 1024 /* alignment */;
}
constexpr int TC_SMEM = tc_smem(TC_STAGES, 128);
// rank-gate parameters (W1 [h][r], W2 [r][h], b1 [h], b2 [r], fp32) after the barriers
__host__ __device__ constexpr int tc_gpar_bytes(int h, int r) { return (2 * h * r + h + r) * 4; }
constexpr int tc_max3(int a, int b, int c) { return a > b ? (a > c ? a : c) : (b > c ? b : c); }
constexpr int TC_SMEM_MAX = 227 * 1024;  // the device's per-block limit
static_assert(tc_max3(TC_SMEM, tc_smem(TC_STAGES - 1, 128) + tc_gpar_bytes(32, 128), tc_smem(3, 256)) <= TC_SMEM_MAX,
              "tensor-core kernel shared memory");

struct TcArgs {
  const __half* scales;
  __nv_bfloat16* y;
  float* gate_out;
  int* mask_count;
  WsHeader* hdr;
  int* mflags;        // [4 * Mb * BMT / 128]: epoch + 1 once an epilogue warp's 32 gt rows are out
  __nv_bfloat16* gt;  // [Mb * BMT][r]
  int M, K, N, r, group;
  float b_g, tau;
  int Mb, Nb;       // BMT-token blocks, 256-channel blocks
  int with_ec;      // projection tiles + EC k-steps
  int NE;           // projection tile width: 16 * ceil((r + 1) / 16)
  int ec_steps;     // ceil(r / 64)
  int gate_kind, gate_h;  // 0: scalar gate; 1: per-rank gamma(t) with bottleneck h
  const float *gw1, *gb1, *gw2, *gb2;
  float alpha;
  int nst;                // ring stages
  int tag_skew;           // test injection: projection flags are awaited at epoch + 1 + skew (0 normally)
  long long pub_wait;     // bound of that wait (SM cycles)
  int S;                  // K parts per tile (1: none); CTA b takes part b % S of tiles b / S, + grid / S, ...
  float* kpart;           // [tiles * S][4 warps][64][32 lanes][4] fp32 partial accumulators (S > 1)
  int* kflags;            // [tiles * S][4 * NH]: epoch + 1 once an epilogue warp's partial rows are out
  int kpart_slots;        // 128 x 256 fp32 partial slots in the workspace (device-check build)
  int kflag_cap;          // K-part flags in the workspace (device-check build)
  int dcheck_force;       // test hook: the y-store check fails (device-check build)
  int sk;                 // 1: stream-K schedule (each CTA an equal run of the tiles' k-steps)
  long long sk_T;         // stream-K: k-steps of all tiles (tiles x K / 64)
};

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// SW128 K-major UMMA shared-memory descriptor (8-row groups 1024 bytes apart).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)1 << 16;            // leading byte offset (16 B; unused with 128-byte swizzle)
  d |= (uint64_t)(1024 >> 4) << 32;  // stride byte offset: next 8-row group
  d |= (uint64_t)1 << 46;            // descriptor version for sm_100
  d |= (uint64_t)2 << 61;            // 128-byte swizzle
  return d;
}

// kind::f16 instruction descriptor: bf16 x bf16 -> fp32, both K-major.
__host__ __device__ constexpr uint32_t make_idesc(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,"
      "%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
      "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
      "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15]))
      : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}


// ---------------------------------------------------------------------------
// schedule shared by all roles
// ---------------------------------------------------------------------------
struct TileInfo {
  int tile;    // projection tiles first, then output tiles
  int kind;    // 0 = projection tile, 1 = output tile
  int mb, nb;
  int k0, nk;  // this CTA's k-steps of the tile: k0 .. k0 + nk - 1
  int steps;   // k-steps here: its part, then the EC steps where this CTA finishes the tile
  int role;    // 0 whole tile; 1 K part `part` of S (column shares); 2 stream-K part sent to the
               // tile's owner; 3 stream-K owner (the tile's first k-steps) of `part` parts
  int part;
};

// The units of work of this CTA, in the order every role takes them:
//  - persistent (S == 1, no stream-K): tiles c, c + G, c + 2 G, ..., whole;
//  - K parts (S > 1): one unit, K part c % S of tile c / S;
//  - stream-K: the CTA's share [c T / G, (c + 1) T / G) of the T = tiles x K/64
//    k-steps, tile by tile in order.  A tile begun in an earlier CTA is a part
//    sent to that CTA (the tile's owner); a tile begun here is owned here and
//    takes the parts of the CTAs that finish it.  A sent part is always the
//    CTA's first unit and an owned tile with parts its last, so no wait cycles.
__device__ __forceinline__ long long sk_lo(const TcArgs& a, int c) { return (long long)c * a.sk_T / gridDim.x; }

__device__ __forceinline__ int unit_count(const TcArgs& a, int ntiles) {
  const int c = (int)blockIdx.x, G = (int)gridDim.x;
  if (a.sk) {
    const long long KT = a.K / TC_BK, lo = sk_lo(a, c), hi = sk_lo(a, c + 1);
    return hi > lo ? (int)((hi - 1) / KT - lo / KT) + 1 : 0;
  }
  if (a.S > 1) return 1;
  return c < ntiles ? (ntiles - 1 - c) / G + 1 : 0;
}

__device__ __forceinline__ TileInfo unit_info(const TcArgs& a, int u) {
  TileInfo t;
  const int KT = a.K / TC_BK;
  const int nproj = a.with_ec ? a.Mb : 0;
  const int c = (int)blockIdx.x, G = (int)gridDim.x;
  t.role = 0;
  t.part = 0;
  if (a.sk) {
    const long long lo = sk_lo(a, c), hi = sk_lo(a, c + 1);
    t.tile = (int)(lo / KT) + u;
    const long long t0 = (long long)t.tile * KT;
    const long long s0 = lo > t0 ? lo : t0, s1 = hi < t0 + KT ? hi : t0 + KT;
    t.k0 = (int)(s0 - t0);
    t.nk = (int)(s1 - s0);
    if (t.k0 > 0) {
      t.role = 2;
    } else {
      int np = 1;  // this CTA and the next ones that start inside the tile
      while (c + np < G && sk_lo(a, c + np) < t0 + KT) ++np;
      t.role = 3;
      t.part = np;
    }
  } else if (a.S > 1) {
    t.tile = c / a.S;
    t.role = 1;
    t.part = c % a.S;
    t.nk = KT / a.S;
    t.k0 = t.part * t.nk;
  } else {
    t.tile = c + u * G;
    t.k0 = 0;
    t.nk = KT;
  }
  const bool finishes = t.role == 0 || t.role == 3 || (t.role == 1 && t.part == a.S - 1);
  if (t.tile < nproj) {
    t.kind = 0;
    t.mb = t.tile;
    t.nb = 0;
    t.steps = t.nk;
  } else {
    const int i = t.tile - nproj;
    t.kind = 1;
    t.mb = i / a.Nb;
    t.nb = i % a.Nb;
    t.steps = t.nk + (a.with_ec && finishes ? a.ec_steps : 0);
  }
  return t;
}

// int4 tile (16 strips of 512 B) -> bf16 [256 rows][64 k] in the SW128 K-major layout.
template <bool GROUP>
__device__ __forceinline__ void dequant_tile(const uint8_t* psrc, uint8_t* bdst, int dt, const TcArgs& a, int nb,
                                             int kt) {
#pragma unroll
  for (int it = 0; it < 2; ++it) {
    const int chunk = dt + it * 256;          // 512 chunks of 16 bytes
    const int strip = chunk >> 5, L = chunk & 31;
    const int rho = L >> 2, c = L & 3;
    const uint4 w = *reinterpret_cast<const uint4*>(psrc + chunk * 16);
    const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
    uint32_t o[4][4];  // o[s][pi]
#pragma unroll
    for (int s = 0; s < 4; ++s) int4x8_to_bf16x8(wv[s], o[s]);
    const int n0 = strip * 16 + rho;  // row within the 256-row tile
    const int n1 = n0 + 8;
    if (GROUP) {
      // bf16(s * q), rounded once: q * s = q * s_hi + q * s_lo with s_hi = bf16(s)
      const int g = kt / 2;
      const float s0 = __half2float(a.scales[(size_t)g * a.N + nb * TC_BN + n0]);
      const float s1 = __half2float(a.scales[(size_t)g * a.N + nb * TC_BN + n1]);
      const __nv_bfloat16 h0 = __float2bfloat16_rn(s0), h1 = __float2bfloat16_rn(s1);
      const __nv_bfloat162 hi0 = __halves2bfloat162(h0, h0), hi1 = __halves2bfloat162(h1, h1);
      const __nv_bfloat16 l0 = __float2bfloat16_rn(s0 - __bfloat162float(h0));
      const __nv_bfloat16 l1 = __float2bfloat16_rn(s1 - __bfloat162float(h1));
      const __nv_bfloat162 lo0 = __halves2bfloat162(l0, l0), lo1 = __halves2bfloat162(l1, l1);
#pragma unroll
      for (int s = 0; s < 4; ++s) {
#pragma unroll
        for (int pi = 0; pi < 4; ++pi) {
          const bool row1 = pi & 1;
          __nv_bfloat162 q = *reinterpret_cast<__nv_bfloat162*>(&o[s][pi]);
          const __nv_bfloat162 p = __hmul2(q, row1 ? lo1 : lo0);
          q = __hfma2(q, row1 ? hi1 : hi0, p);
          o[s][pi] = *reinterpret_cast<uint32_t*>(&q);
        }
      }
    }
    // row n0: k 16c + 4s + {0,1} = o[s][0], {2,3} = o[s][2];  row n1: o[s][1], o[s][3]
    const int ch0 = 2 * c, ch1 = 2 * c + 1;  // 16-byte chunks of the 128-byte row
    uint8_t* r0 = bdst + (n0 >> 3) * 1024 + (n0 & 7) * 128;
    uint8_t* r1 = bdst + (n1 >> 3) * 1024 + (n1 & 7) * 128;
    *reinterpret_cast<uint4*>(r0 + ((ch0 ^ (n0 & 7)) << 4)) = make_uint4(o[0][0], o[0][2], o[1][0], o[1][2]);
    *reinterpret_cast<uint4*>(r0 + ((ch1 ^ (n0 & 7)) << 4)) = make_uint4(o[2][0], o[2][2], o[3][0], o[3][2]);
    *reinterpret_cast<uint4*>(r1 + ((ch0 ^ (n1 & 7)) << 4)) = make_uint4(o[0][1], o[0][3], o[1][1], o[1][3]);
    *reinterpret_cast<uint4*>(r1 + ((ch1 ^ (n1 & 7)) << 4)) = make_uint4(o[2][1], o[2][3], o[3][1], o[3][3]);
  }
}

// Wait, bounded and without reporting, for asynchronous work already issued
// against this CTA's shared memory or TMEM (before the CTA frees them).
__device__ __forceinline__ void tc_drain(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > kWaitCycles) break;
}

template <bool GROUP, int BMT>
__global__ void __launch_bounds__(TC_THREADS, 1)
    tc_kernel(const __grid_constant__ TcArgs a, const __grid_constant__ CUtensorMap tm_x,
              const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_agt,
              const __grid_constant__ CUtensorMap tm_bpt, const __grid_constant__ CUtensorMap tm_gt) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, derived from the shared array itself so that the
  // compiler keeps every access in the shared window (ld/st.shared)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  constexpr int NH = BMT / TC_BM;          // accumulators (M = 128 MMAs) per tile
  constexpr int NBA = NH == 1 ? 2 : 1;      // accumulator buffers (TMEM holds 512 columns)
  constexpr int XB = BMT * TC_BK * 2;       // x bytes of a stage
  uint8_t* xs = smem;                                        // [NST][XB]
  const int NST = a.nst;
  uint8_t* bs = smem + NST * XB;                             // [NST][32 KB]
  uint8_t* ps = bs + NST * TC_B_BYTES;                       // [NST][8 KB]
  uint64_t* bars = reinterpret_cast<uint64_t*>(ps + NST * TC_P_BYTES);
  uint64_t* full = bars;                     // TMA loads of a stage landed
  uint64_t* ready = bars + NST;              // B operand of a stage ready (dequant warps)
  uint64_t* empty = bars + 2 * NST;          // MMAs of a stage done
  uint64_t* acc_full = bars + 3 * NST;       // [2]
  uint64_t* acc_empty = acc_full + 2;        // [2]
  uint32_t* tmem_base_holder = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_holder + 1);
  float* gpar = reinterpret_cast<float*>(ps + NST * TC_P_BYTES + 1024);
  // the output tile's 256 per-channel scales (epilogue warps), in the barrier block's second half
  __half* esc = reinterpret_cast<__half*>(ps + NST * TC_P_BYTES + 512);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int epoch = *reinterpret_cast<volatile int*>(&a.hdr->epoch);
  const int ntiles = (a.with_ec ? a.Mb : 0) + a.Mb * a.Nb;
  const int nunits = unit_count(a, ntiles);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&ready[s], 8);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < NBA; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_base_holder)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_base_holder;
  if (!a.with_ec && blockIdx.x == 0) {
    // EC disabled: every gate is 0, below any positive threshold
    if (a.gate_out)
      for (int m = threadIdx.x; m < a.M; m += blockDim.x) a.gate_out[m] = 0.f;
    if (a.mask_count && threadIdx.x == 0) *a.mask_count = a.M;
  }

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int issued = 0;  // stages whose loads went out
      bool ok = true;
      for (int u = 0; u < nunits && ok; ++u) {
        const TileInfo ti = unit_info(a, u);
        for (int k = 0; k < ti.steps && ok; ++k) {
          ok = mbar_wait(&empty[s], ph ^ 1, abort_flag, a.hdr);
          if (!ok) break;
          uint8_t* xd = xs + s * XB;
          uint8_t* bd = bs + s * TC_B_BYTES;
          uint8_t* pd = ps + s * TC_P_BYTES;
          if (ti.kind == 0) {
            mbar_arrive_tx(&full[s], XB + a.NE * 128);
            tma_load_2d(smem_u32(xd), &tm_x, &full[s], (ti.k0 + k) * TC_BK, ti.mb * BMT);
            tma_load_2d(smem_u32(bd), &tm_agt, &full[s], (ti.k0 + k) * TC_BK, 0);
          } else if (k < ti.nk) {
            const int kg = ti.k0 + k;
            mbar_arrive_tx(&full[s], XB + TC_P_BYTES);
            tma_load_2d(smem_u32(xd), &tm_x, &full[s], kg * TC_BK, ti.mb * BMT);
            tma_load_3d(smem_u32(pd), &tm_w, &full[s], 0, kg, ti.nb * (TC_BN / 16));
            // then warm L2 a few k-steps ahead (each TMA instruction costs this
            // thread tens of ns, so the step's own loads go out first), so the
            // shallow shared-memory ring does not see the full HBM latency on
            // every stage
            if (k + TC_PREFETCH < ti.nk) {
              tma_prefetch_2d(&tm_x, (kg + TC_PREFETCH) * TC_BK, ti.mb * BMT);
              tma_prefetch_3d(&tm_w, 0, kg + TC_PREFETCH, ti.nb * (TC_BN / 16));
            } else {
              // the tile's tail: warm its EC operands (L2 is coherent, so gt may
              // be warmed before the projection is published) and the first
              // k-steps of this CTA's next tile
              const int j = k + TC_PREFETCH - ti.nk;
              if (j == 0 && ti.steps > ti.nk)
                for (int e = 0; e < a.ec_steps; ++e) {
                  tma_prefetch_2d(&tm_bpt, e * TC_BK, ti.nb * TC_BN);
                  tma_prefetch_2d(&tm_gt, e * TC_BK, ti.mb * BMT);
                }
              if (u + 1 < nunits) {
                const TileInfo tn = unit_info(a, u + 1);
                if (tn.kind == 1 && j < tn.nk) {
                  tma_prefetch_2d(&tm_x, (tn.k0 + j) * TC_BK, tn.mb * BMT);
                  tma_prefetch_3d(&tm_w, 0, tn.k0 + j, tn.nb * (TC_BN / 16));
                }
              }
            }
            // the CTA's first tile: once the ring's first loads are out, warm the
            // steps after them that the per-step warm-up above does not reach
            // (later tiles had theirs warmed during the previous tile's tail)
            if (u == 0 && k == min(NST, ti.nk) - 1)
              for (int pk = NST; pk < TC_PREFETCH && pk < ti.nk; ++pk) {
                tma_prefetch_2d(&tm_x, (ti.k0 + pk) * TC_BK, ti.mb * BMT);
                tma_prefetch_3d(&tm_w, 0, ti.k0 + pk, ti.nb * (TC_BN / 16));
              }
          } else {
            const int e = k - ti.nk;
            // B' does not depend on the projection: its load goes out first
            mbar_arrive_tx(&full[s], XB + TC_B_BYTES);
            tma_load_2d(smem_u32(bd), &tm_bpt, &full[s], e * TC_BK, ti.nb * TC_BN);
            if (e == 0) {
              // gated projection of this token block must be published (all
              // its flags polled together)
              ok = wait_flags_eq(&a.mflags[4 * NH * ti.mb], 4 * NH, epoch + 1 + a.tag_skew, a.hdr, a.pub_wait);
              if (!ok) *abort_flag = 1;
              asm volatile("fence.proxy.async.global;" ::: "memory");
            }
            // (issued even after a failed wait, so that the stage's barrier
            // completes and is drained below; nobody reads it then)
            tma_load_2d(smem_u32(xd), &tm_gt, &full[s], e * TC_BK, ti.mb * BMT);
          }
          ++issued;
          if (++s == NST) {
            s = 0;
            ph ^= 1;
          }
        }
      }
      // Before the CTA exits, no load may still write its shared memory: wait
      // for the last NST stages issued (a stage has one outstanding phase at
      // most).  Without an abort they have all been consumed already.
      for (int j = 0; j < NST && j < issued; ++j) {
        if (--s < 0) {
          s = NST - 1;
          ph ^= 1;
        }
        tc_drain(&full[s], ph);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int buf = 0;
      uint32_t aph[2] = {0, 0};
      int last_s = -1;      // stage (and its phase) of the last commit
      uint32_t last_ph = 0;
      bool ok = true;
      for (int u = 0; u < nunits && ok; ++u) {
        const TileInfo ti = unit_info(a, u);
        ok = mbar_wait(&acc_empty[buf], aph[buf] ^ 1, abort_flag, a.hdr);
        if (!ok) break;
        tc_fence_after();
        const uint32_t idesc = ti.kind == 0 ? make_idesc(TC_BM, a.NE) : make_idesc(TC_BM, TC_BN);
        for (int k = 0; k < ti.steps && ok; ++k) {
          ok = mbar_wait(&ready[s], ph, abort_flag, a.hdr);
          if (!ok) break;
          tc_fence_after();
          const uint64_t bd = sw128_desc(smem_u32(bs + s * TC_B_BYTES));
#pragma unroll
          for (int h = 0; h < NH; ++h) {
            // rows 128 h .. 128 h + 127 of the x tile (8-row groups 1024 B apart)
            const uint64_t ad = sw128_desc(smem_u32(xs + s * XB + h * TC_X_BYTES));
            const uint32_t d = tmem_base + (uint32_t)(buf * NH + h) * 256;
#pragma unroll
            for (int kk = 0; kk < TC_BK / 16; ++kk)
              umma(d, ad + 2 * kk, bd + 2 * kk, idesc, (k > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&empty[s]);
          last_s = s;
          last_ph = ph;
          if (++s == NST) {
            s = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&acc_full[buf]);
        aph[buf] ^= 1;
        buf = buf + 1 == NBA ? 0 : buf + 1;
      }
      // the MMAs read shared memory and write TMEM asynchronously: wait for the
      // last commit (it tracks every earlier MMA) before TMEM is freed
      if (last_s >= 0) tc_drain(&empty[last_s], last_ph);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter of this warp
    if (a.gate_kind == 1) {
      // rank-gate parameters into shared memory (the 4 epilogue warps; every
      // array has a multiple of 4 floats and is 16-byte aligned)
      const int h = a.gate_h, r = a.r, et = threadIdx.x - 64;
      auto stage4 = [&](const float* src, float* dst, int n) {
        for (int i = et; i < n / 4; i += 128)
          reinterpret_cast<float4*>(dst)[i] = __ldg(reinterpret_cast<const float4*>(src) + i);
      };
      stage4(a.gw1, gpar, h * r);
      stage4(a.gw2, gpar + h * r, r * h);
      stage4(a.gb1, gpar + 2 * h * r, h);
      stage4(a.gb2, gpar + 2 * h * r + h, r);
      asm volatile("bar.sync 1, 128;" ::: "memory");
    }
    const float* W1 = gpar;
    const float* W2 = gpar + a.gate_h * a.r;
    const float* B1 = gpar + 2 * a.gate_h * a.r;
    const float* B2 = B1 + a.gate_h;
    int buf = 0;
    uint32_t aph[2] = {0, 0};
    bool ok = true;
    for (int u = 0; u < nunits && ok; ++u) {
      const TileInfo ti = unit_info(a, u);
      const int tile = ti.tile;
      ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[buf], aph[buf], abort_flag, a.hdr));
      if (!ok) break;
      tc_fence_after();
      if (!GROUP && ti.kind == 1) {
        // the tile's scales into shared memory once (the previous tile's
        // readers are done: every epilogue warp passed the first barrier)
        asm volatile("bar.sync 1, 128;" ::: "memory");
        const int et = threadIdx.x - 64;
        reinterpret_cast<uint32_t*>(esc)[et] =
            __ldg(reinterpret_cast<const uint32_t*>(a.scales + ti.nb * TC_BN) + et);
        asm volatile("bar.sync 1, 128;" ::: "memory");
      }
#pragma unroll 1
      for (int h = 0; h < NH; ++h) {
      const int row = q * 32 + lane;
      const int m = ti.mb * BMT + h * TC_BM + row;
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * NH + h) * 256;
      // K parts (S > 1): every part puts its accumulator in the workspace and
      // raises its flag; then each part sums, in part order, its share of the
      // tile (a projection tile whole on part 0, 256 / S output channels per
      // part) back into its own accumulator, and the code below stores that
      // share.  A warp's partial is [column / 4][lane][4] fp32 (a store of 4
      // columns is 512 contiguous bytes, a run of columns one contiguous
      // block), read back with one bulk copy per part and chunk of columns
      // into the ring, which is idle once the accumulator is complete (a CTA
      // holds one tile when S > 1).  A warp whose 32 rows are all past M skips
      // the exchange on every part alike.
      int lo = 0, hi = TC_BN;
      bool run_gate = true, sent = false;
      if (BMT == 128 && ti.role == 1) {
        const int part = ti.part;
        // (device-check build: this tile's partial slots and flags lie in the workspace)
        const bool kp_ok =
            SPEAR_DCHECK((tile + 1) * a.S <= a.kpart_slots && (tile + 1) * a.S * 4 * NH <= a.kflag_cap, a.hdr);
        const bool rows = ti.mb * BMT + h * TC_BM + q * 32 < a.M && kp_ok;
        const int ncol = ti.kind == 0 ? a.NE : TC_BN;
        constexpr int QF = TC_BN * 32;  // floats of one warp's partial
        const float* qbase = a.kpart + ((size_t)tile * a.S * 4 * NH + 4 * h + q) * QF;
        int* kflag = a.kflags + (tile * a.S) * 4 * NH + 4 * h + q;
        if (rows) {
          float4* pdst = reinterpret_cast<float4*>(const_cast<float*>(qbase) + (size_t)part * 4 * NH * QF);
          for (int c0 = 0; c0 < ncol; c0 += 16) {
            float v[16];
            tmem_ld16(taddr + c0, v);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              pdst[(c0 / 4 + i) * 32 + lane] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
          }
          // the warp barrier orders every lane's stores before lane 0's release
          __syncwarp();
          if (lane == 0) st_release_gpu(kflag + part * 4 * NH, epoch + 1);
        }
        lo = ti.kind == 0 ? 0 : part * (TC_BN / a.S);
        hi = !rows ? lo : ti.kind == 0 ? (part == 0 ? a.NE : 0) : lo + TC_BN / a.S;
        run_gate = part == 0;
        if (hi > lo) {
          // this warp's share of the ring (split among the warps that hold
          // rows, warps 0 .. nw - 1): NB buffers of S x CC columns, then NB
          // mbarriers.  CC columns per chunk: the whole share when it fits.
          const int nw = min(4, (a.M - ti.mb * BMT - h * TC_BM + 31) / 32);
          const int XW = (NST * tc_stage_bytes(BMT) / nw) & ~1023;
          uint8_t* xw = smem + q * XW;
          uint64_t* xbar = reinterpret_cast<uint64_t*>(xw + XW - 128);
          int CC = hi - lo;
          while (a.S * CC * 128 > XW - 128) CC = (CC / 2 + 15) & ~15;
          const int CB = a.S * CC * 128;  // bytes of one buffer
          const int nch = (hi - lo + CC - 1) / CC;
          const int NB = min(min(nch, (XW - 128) / CB), 16);
          if (lane == 0) {
            for (int b = 0; b < NB; ++b) mbar_init(&xbar[b], 1);
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
          }
          // lane p watches part p's flag: one round trip per poll for all parts
          const bool fok = lane >= a.S || wait_flag_eq(kflag + lane * 4 * NH, epoch + 1, a.hdr);
          if (!__all_sync(0xffffffffu, fok)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          auto issue = [&](int ch) {  // lane 0: columns lo + CC ch .. of every part
            const int b = ch % NB, c0 = lo + ch * CC, nb = (min(hi, c0 + CC) - c0) * 128;
            mbar_arrive_tx(&xbar[b], a.S * nb);
            for (int p = 0; p < a.S; ++p)
              bulk_g2s(xw + b * CB + p * CC * 128, qbase + (size_t)p * 4 * NH * QF + c0 * 32, nb, &xbar[b]);
          };
          // the polling lanes' acquires, the warp barrier, then lane 0's bulk
          // copies (async proxy) read the partials
          __syncwarp();
          if (lane == 0) {
            asm volatile("fence.proxy.async.global;" ::: "memory");
            for (int ch = 0; ch < NB; ++ch) issue(ch);
          }
          int ch = 0;
          for (; ch < nch; ++ch) {
            const int b = ch % NB, c0 = lo + ch * CC, c1 = min(hi, c0 + CC);
            if (!__all_sync(0xffffffffu, mbar_wait(&xbar[b], (ch / NB) & 1, abort_flag, a.hdr))) break;
            for (int g = c0; g < c1; g += 16) {
              float sum[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) sum[i] = 0.f;
              for (int p = 0; p < a.S; ++p) {
                const float4* src = reinterpret_cast<const float4*>(xw + b * CB + p * CC * 128 + (g - c0) * 128) + lane;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  const float4 v = src[32 * i];
                  sum[4 * i] += v.x;
                  sum[4 * i + 1] += v.y;
                  sum[4 * i + 2] += v.z;
                  sum[4 * i + 3] += v.w;
                }
              }
              tmem_st16(taddr + g, sum);
            }
            __syncwarp();
            if (lane == 0 && ch + NB < nch) {
              asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
              issue(ch + NB);
            }
          }
          asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
          if (ch < nch) {
            // gave up: let the copies in flight land before the ring is released
            if (lane == 0)
              for (int c = ch; c < nch && c < ch + NB; ++c) tc_drain(&xbar[c % NB], (c / NB) & 1);
            __syncwarp();
            ok = false;
            break;
          }
        }
      }
      // stream-K: a sent part puts its accumulator in the workspace slot of this
      // CTA ([column/4][lane][4] per warp, as above) and raises its flag; the
      // owner waits for the parts of the CTAs after it, reads them with one
      // bulk copy per part and chunk into the ring (idle: an owned tile with
      // parts is the CTA's last unit), and adds them in k order to its own
      // accumulator, on which the epilogue below then runs.
      if (BMT == 128 && (ti.role == 2 || (ti.role == 3 && ti.part > 1))) {
        constexpr int QF = TC_BN * 32;
        const bool rows = ti.mb * BMT + h * TC_BM + q * 32 < a.M &&
                          SPEAR_DCHECK((int)gridDim.x <= a.kpart_slots && (int)gridDim.x * 4 * NH <= a.kflag_cap,
                                       a.hdr);
        const int ncol = ti.kind == 0 ? a.NE : TC_BN;
        auto slot = [&](int cta) { return a.kpart + ((size_t)cta * 4 * NH + 4 * h + q) * QF; };
        auto sflag = [&](int cta) { return a.kflags + cta * 4 * NH + 4 * h + q; };
        if (ti.role == 2) {
          sent = true;
          if (rows) {
            float4* pdst = reinterpret_cast<float4*>(slot((int)blockIdx.x));
            for (int c0 = 0; c0 < ncol; c0 += 16) {
              float v[16];
              tmem_ld16(taddr + c0, v);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                pdst[(c0 / 4 + i) * 32 + lane] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            }
            // the warp barrier orders every lane's stores before lane 0's release
            __syncwarp();
            if (lane == 0) st_release_gpu(sflag((int)blockIdx.x), epoch + 1);
          }
        } else if (rows) {
          const int nother = ti.part - 1;  // parts of CTAs blockIdx.x + 1 .. + nother
          const int nw = min(4, (a.M - ti.mb * BMT - h * TC_BM + 31) / 32);
          const int XW = (NST * tc_stage_bytes(BMT) / nw) & ~1023;
          uint8_t* xw = smem + q * XW;
          uint64_t* xbar = reinterpret_cast<uint64_t*>(xw + XW - 128);
          int CC = ncol;
          while (nother * CC * 128 > XW - 128) CC = (CC / 2 + 15) & ~15;
          const int CB = nother * CC * 128;
          const int nch = (ncol + CC - 1) / CC;
          const int NB = min(min(nch, (XW - 128) / CB), 16);
          if (lane == 0) {
            for (int b = 0; b < NB; ++b) mbar_init(&xbar[b], 1);
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
          }
          const bool fok = lane >= nother || wait_flag_eq(sflag((int)blockIdx.x + 1 + lane), epoch + 1, a.hdr);
          if (!__all_sync(0xffffffffu, fok)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          auto issue = [&](int ch) {  // lane 0: columns CC ch .. of every other part
            const int b = ch % NB, c0 = ch * CC, nb = (min(ncol, c0 + CC) - c0) * 128;
            mbar_arrive_tx(&xbar[b], nother * nb);
            for (int pp = 0; pp < nother; ++pp)
              bulk_g2s(xw + b * CB + pp * CC * 128, slot((int)blockIdx.x + 1 + pp) + c0 * 32, nb, &xbar[b]);
          };
          __syncwarp();
          if (lane == 0) {
            asm volatile("fence.proxy.async.global;" ::: "memory");
            for (int ch = 0; ch < NB; ++ch) issue(ch);
          }
          int ch = 0;
          for (; ch < nch; ++ch) {
            const int b = ch % NB, c0 = ch * CC, c1 = min(ncol, c0 + CC);
            if (!__all_sync(0xffffffffu, mbar_wait(&xbar[b], (ch / NB) & 1, abort_flag, a.hdr))) break;
            for (int g = c0; g < c1; g += 16) {
              float sum[16];
              tmem_ld16(taddr + g, sum);  // this CTA's part comes first in k order
              for (int pp = 0; pp < nother; ++pp) {
                const float4* src = reinterpret_cast<const float4*>(xw + b * CB + pp * CC * 128 + (g - c0) * 128) + lane;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  const float4 v = src[32 * i];
                  sum[4 * i] += v.x;
                  sum[4 * i + 1] += v.y;
                  sum[4 * i + 2] += v.z;
                  sum[4 * i + 3] += v.w;
                }
              }
              tmem_st16(taddr + g, sum);
            }
            __syncwarp();
            if (lane == 0 && ch + NB < nch) {
              asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
              issue(ch + NB);
            }
          }
          asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
          if (ch < nch) {
            // gave up: let the copies in flight land before the ring is released
            if (lane == 0)
              for (int c = ch; c < nch && c < ch + NB; ++c) tc_drain(&xbar[c % NB], (c / NB) & 1);
            __syncwarp();
            ok = false;
            break;
          }
        }
      }
      if (sent) {
        // the tile's owner stores it
      } else if (ti.kind == 0 && !run_gate) {
        // another part runs this projection tile's gate
      } else if (ti.kind == 0) {
        // projection tile: columns 0..r-1 = t, column r = gate logit
        __nv_bfloat16* gdst = a.gt + (size_t)m * a.r;
        float g;
        if (a.gate_kind == 1) {
          // rank gate (summary section 2.1 A): u = relu(W1 t + b1),
          // gamma = sigmoid(W2 u + b2), gt = bf16(alpha gamma t); this
          // thread's token row, t read from TMEM twice
          float u[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) u[i] = i < a.gate_h ? B1[i] : 0.f;
          for (int c0 = 0; c0 < a.r; c0 += 16) {
            float tv[16];
            tmem_ld16(taddr + c0, tv);
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (i < a.gate_h) {
                const float4* w = reinterpret_cast<const float4*>(W1 + i * a.r + c0);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                  const float4 wv = w[q4];
                  u[i] = fmaf(wv.x, tv[4 * q4], u[i]);
                  u[i] = fmaf(wv.y, tv[4 * q4 + 1], u[i]);
                  u[i] = fmaf(wv.z, tv[4 * q4 + 2], u[i]);
                  u[i] = fmaf(wv.w, tv[4 * q4 + 3], u[i]);
                }
              }
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) u[i] = fmaxf(u[i], 0.f);
          float gsum = 0.f;
          for (int c0 = 0; c0 < a.r; c0 += 16) {
            float tv[16];
            tmem_ld16(taddr + c0, tv);
            float o[16];
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
              const int j = c0 + jj;
              float z = B2[j];
              const float4* w = reinterpret_cast<const float4*>(W2 + j * a.gate_h);
#pragma unroll
              for (int i4 = 0; i4 < 8; ++i4)
                if (4 * i4 < a.gate_h) {
                  const float4 wv = w[i4];
                  z = fmaf(wv.x, u[4 * i4], z);
                  z = fmaf(wv.y, u[4 * i4 + 1], z);
                  z = fmaf(wv.z, u[4 * i4 + 2], z);
                  z = fmaf(wv.w, u[4 * i4 + 3], z);
                }
              const float gam = sigmoidf_(z);
              gsum += gam;
              o[jj] = a.alpha * gam * tv[jj];
            }
            uint32_t pk[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) pk[i] = pack_bf16x2(o[2 * i], o[2 * i + 1]);
            uint4* d4 = reinterpret_cast<uint4*>(gdst + c0);
            d4[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            d4[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
          g = gsum / (float)a.r;  // the reported gate: mean of gamma
        } else {
          float lv[16];
          tmem_ld16(taddr + (a.r / 16) * 16, lv);
          g = sigmoidf_(lv[0] + a.b_g);
          for (int c0 = 0; c0 < a.r; c0 += 16) {
            float tv[16];
            tmem_ld16(taddr + c0, tv);
            uint32_t pk[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) pk[i] = pack_bf16x2(g * tv[2 * i], g * tv[2 * i + 1]);
            uint4* d4 = reinterpret_cast<uint4*>(gdst + c0);
            d4[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            d4[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
        }
        const bool valid = m < a.M;
        if (valid && a.gate_out) a.gate_out[m] = g;
        const unsigned below = __ballot_sync(0xffffffffu, valid && g < a.tau);
        if (lane == 0 && a.mask_count && below) atomicAdd(&a.hdr->ec_done, __popc(below));
        asm volatile("fence.proxy.async.global;" ::: "memory");
        tc_fence_before();
        // the warp barrier orders every lane's gt stores before lane 0's release
        __syncwarp();
        // one flag per epilogue warp (32 token rows), tagged with this launch's epoch
        if (lane == 0) st_release_gpu(&a.mflags[4 * NH * ti.mb + 4 * h + q], epoch + 1);
      } else {
        const int n0 = ti.nb * TC_BN;
#pragma unroll 1
        for (int c0 = lo; c0 < hi; c0 += 32) {
          float v[32];
          tmem_ld32(taddr + c0, v);
          if (!GROUP) {
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              const float2 sc = __half22float2(*reinterpret_cast<const __half2*>(esc + c0 + i));
              v[i] *= sc.x;
              v[i + 1] *= sc.y;
            }
          }
          if (m < a.M && SPEAR_DCHECK(n0 + c0 + 32 <= a.N && !a.dcheck_force, a.hdr)) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
            uint4* dst = reinterpret_cast<uint4*>(a.y + (size_t)m * a.N + n0 + c0);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          }
        }
        tc_fence_before();
      }
      }  // accumulator halves
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
      aph[buf] ^= 1;
      buf = buf + 1 == NBA ? 0 : buf + 1;
    }
  } else {
    // ------------------------------------------------------------ dequant
    const int dt = threadIdx.x - 6 * 32;  // 0..255
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int u = 0; u < nunits && ok; ++u) {
      const TileInfo ti = unit_info(a, u);
      for (int k = 0; k < ti.steps && ok; ++k) {
        ok = __all_sync(0xffffffffu, mbar_wait(&full[s], ph, abort_flag, a.hdr));
        if (!ok) break;
        if (ti.kind == 1 && k < ti.nk) {
          dequant_tile<GROUP>(ps + s * TC_P_BYTES, bs + s * TC_B_BYTES, dt, a, ti.nb, ti.k0 + k);
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&ready[s]);
        if (++s == NST) {
          s = 0;
          ph ^= 1;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(512));
  }
  if (threadIdx.x == 0) {
    __threadfence();
    const int prev = atomicAdd(&a.hdr->done_ctas, 1);
    if (prev == (int)gridDim.x - 1) {
      if (a.mask_count && a.with_ec) *a.mask_count = a.hdr->ec_done;
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
TcPlan plan_tc(int M, int K, int N, int r, int group, int sm_count) {
  (void)K;
  (void)r;
  (void)group;
  TcPlan p = {};
  p.m_blocks = (M + TC_BM - 1) / TC_BM;
  p.n_blocks = N / TC_BN;
  p.grid = sm_count;
  p.smem = TC_SMEM;
  return p;
}

template <bool GROUP, int BMT>
static int launch_tc_t(const TcPlan& p, const TcArgs& a, const CUtensorMap* maps, cudaStream_t st) {
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [&] {
    attr_err = cudaFuncSetAttribute(tc_kernel<GROUP, BMT>, cudaFuncAttributeMaxDynamicSharedMemorySize, TC_SMEM_MAX);
  });
  if (attr_err != cudaSuccess) return set_cuda_error("cudaFuncSetAttribute(tc)", attr_err);
  const int ntiles = (a.with_ec ? a.Mb : 0) + a.Mb * a.Nb;
  const int groups = ntiles < p.grid / a.S ? ntiles : p.grid / a.S;
  const int grid = a.sk ? p.grid : groups * a.S;
  const size_t smem = tc_smem(a.nst, BMT) + (a.gate_kind == 1 ? tc_gpar_bytes(a.gate_h, a.r) : 0);
  tc_kernel<GROUP, BMT><<<grid, TC_THREADS, smem, st>>>(a, maps[0], maps[1], maps[2], maps[3], maps[4]);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SPEAR_OK : set_cuda_error("tc kernel launch", e);
}

// Tile height: 256 tokens (twice the tensor-core work per dequantised tile
// and per ring round trip) once such tiles fill at least half the SMs, when
// the rank gate's parameters, if any, fit beside three stages; 128 otherwise,
// where K parts fill the SMs (at M = 512, N = 4096 the 34 tall tiles ran
// their whole K on 34 SMs, as slow as M = 2048).
static int tc_tile_rows(int M, const LayerView& L, bool with_ec, int sms) {
  if (M < 512) return 128;
  const int mb = (M + 255) / 256;
  const int tiles = (with_ec && L.r > 0 ? mb : 0) + mb * (L.N / TC_BN);
  if (2 * tiles < sms) return 128;
  const bool rank = with_ec && L.r > 0 && L.gate_kind == 1;
  return (!rank || tc_smem(3, 256) + tc_gpar_bytes(L.gate_h, L.r) <= TC_SMEM_MAX) ? 256 : 128;
}

int launch_tc(const TcPlan& p, const LayerView& L, const __nv_bfloat16* x, int M, __nv_bfloat16* y, bool with_ec,
              WsHeader* hdr, int* mflags, int* kflags, float* kpart, __nv_bfloat16* gt, float* gate_out,
              int* mask_count, cudaStream_t st) {
  if (L.N % TC_BN) return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "tensor-core path needs N %% 256 == 0 (N=%d)", L.N);
  const int bmt = tc_tile_rows(M, L, with_ec, p.grid);
  TcArgs a = {};
  a.scales = L.scales;
  a.y = y;
  a.gate_out = gate_out;
  a.mask_count = mask_count;
  a.hdr = hdr;
  a.mflags = mflags;
  a.gt = gt;
  a.M = M;
  a.K = L.K;
  a.N = L.N;
  a.r = with_ec ? L.r : 0;
  a.group = L.group;
  a.b_g = L.b_g;
  a.tau = L.tau;
  a.Mb = (M + bmt - 1) / bmt;
  a.Nb = p.n_blocks;
  a.with_ec = with_ec && L.r > 0;
  a.NE = 16 * ((a.r + 1 + 15) / 16);
  a.ec_steps = (a.r + TC_BK - 1) / TC_BK;
  a.gate_kind = a.with_ec ? L.gate_kind : 0;
  a.gate_h = L.gate_h;
  a.gw1 = L.gw1;
  a.gb1 = L.gb1;
  a.gw2 = L.gw2;
  a.gb2 = L.gb2;
  a.alpha = L.alpha;
  a.nst = bmt == 256 ? 3 : (a.gate_kind == 1 ? TC_STAGES - 1 : TC_STAGES);
  // K parts at mid M: while the tiles fill less than half the SMs, split each
  // tile's K in two more parts (up to 8, at least 8 k-steps per part); every
  // group of S CTAs then holds exactly one tile, all resident at once
  a.S = 1;
  a.kflags = kflags;
  a.kpart = kpart;
  if (bmt == 128 && kflags && kpart) {
    const int ntiles = (a.with_ec ? a.Mb : 0) + a.Mb * a.Nb;
    const int KT = L.K / TC_BK;
    while (a.S < 8 && ntiles * a.S * 2 <= p.grid && KT % (a.S * 2) == 0 && KT / (a.S * 2) >= 8) a.S *= 2;
    // stream-K where the tiles leave SMs idle but no K split was taken (more
    // than half as many tiles as SMs, or a K that the split cannot divide):
    // every SM takes an equal run of at least 8 of the tiles' k-steps
    const long long T = (long long)ntiles * KT;
    if (a.S == 1 && ntiles < p.grid && T / p.grid >= 8) {
      a.sk = 1;
      a.sk_T = T;
    }
  }
  const TestFault tf_ = test_fault();
  a.tag_skew = tf_.kernel == 2 ? 1 : 0;
  a.pub_wait = tf_.kernel == 2 ? tf_.cycles : kWaitCycles;
  a.kpart_slots = p.grid;  // the workspace holds one slot per SM
  a.kflag_cap = kKFlagCapacity;
  a.dcheck_force = test_force_check() == 2;
  CUtensorMap maps[5];
  memset(maps, 0, sizeof(maps));
  bool ok = tmap_2d_bf16(&maps[0], x, L.K, M, TC_BK, bmt) && tmap_packed_box(&maps[1], L.w, L.K, L.N, 1, TC_BN / 16);
  if (ok && a.with_ec) {
    ok = tmap_2d_bf16(&maps[2], L.agt, L.K, L.r + 1, TC_BK, a.NE) &&
         tmap_2d_bf16(&maps[3], L.bpt, L.r, L.N, TC_BK, TC_BN) &&
         tmap_2d_bf16(&maps[4], gt, L.r, (uint64_t)a.Mb * bmt, TC_BK, bmt);
  }
  if (!ok) return set_error(SPEAR_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  if (bmt == 256) return L.group ? launch_tc_t<true, 256>(p, a, maps, st) : launch_tc_t<false, 256>(p, a, maps, st);
  return L.group ? launch_tc_t<true, 128>(p, a, maps, st) : launch_tc_t<false, 128>(p, a, maps, st);
}

}  // namespace spear
