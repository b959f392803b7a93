// Shared device-side helpers of the sm_100a kernels: workspace header,
// status reporting, bounded waits, bf16 packing, int4 -> bf16 conversion,
// warp-level tensor-core MMA and cluster (DSMEM) primitives.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/spear.h"

namespace spear {

// ---------------------------------------------------------------------------
// Workspace header (first 256 bytes of every workspace).  All fields start at
// zero (spear_workspace_init) and every kernel leaves them in a state that the
// next launch on the same stream can use without re-initialisation.
// ---------------------------------------------------------------------------
struct WsHeader {
  int status;     // first device-side error code (SPEAR_ERR_*), sticky until read
  int epoch;      // launch counter, advanced by the last CTA of each launch
  int done_ctas;  // CTAs finished in the current launch
  int ec_done;    // EC row groups finalised in the current launch
  int ec_flag;    // == epoch + 1 once the gated EC projection of this launch is ready
  int d2_epoch;   // decode path: launches completed (tags its EC projection words)
  int gt_obs;     // decode path: CTAs that have read the complete EC projection
  int sf_done;    // semi-fused EC projection launch: CTAs finished
  int sf_count;   // semi-fused EC projection launch: tokens with g < tau
  int d3_flag[16];  // decode kernel: EC item e of the current launch published once == d2_epoch + 1
  int pad0[39];
};
static_assert(sizeof(WsHeader) <= 256, "header must fit in 256 bytes");
constexpr size_t kWsHeaderBytes = 256;

// Upper bound of a device-side wait (SM clock cycles).  Far above any
// legitimate wait in these kernels (microseconds), far below a hang.
constexpr long long kWaitCycles = 2000000000LL;  // ~1 s at 1.9 GHz

__device__ __forceinline__ void report_status(WsHeader* h, int code) {
  atomicCAS(&h->status, 0, code);
}

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release_gpu(int* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Device-side argument checks of the debug build (-DSPEAR_DEVICE_CHECKS): a
// failed check reports SPEAR_ERR_DEVICE_CHECK in the status word and the
// access it guards is skipped; nothing traps or faults.  In the normal build
// a check is `true` and its condition is not evaluated.
#ifdef SPEAR_DEVICE_CHECKS
__device__ __forceinline__ bool spear_dcheck(bool ok, WsHeader* h) {
  if (!ok) report_status(h, SPEAR_ERR_DEVICE_CHECK);
  return ok;
}
#define SPEAR_DCHECK(cond, hdr) ::spear::spear_dcheck((cond), (hdr))
#else
#define SPEAR_DCHECK(cond, hdr) true
#endif

// Spin until the n flags f[0..n) all equal want, their loads in flight
// together (one round trip per poll), then an acquire fence; false (and a
// status report) if the bound expires.
__device__ __forceinline__ bool wait_flags_eq(const int* f, int n, int want, WsHeader* h, long long limit) {
  const long long t0 = clock64();
  for (;;) {
    int v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (i < n) asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v[i]) : "l"(f + i) : "memory");
    bool all = true;
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (i < n) all = all && v[i] == want;
    if (all) break;
    if (clock64() - t0 > limit) {
      report_status(h, SPEAR_ERR_TIMEOUT);
      return false;
    }
    __nanosleep(32);
  }
  asm volatile("fence.acq_rel.gpu;" ::: "memory");
  return true;
}

// Spin until *p == want; false (and a status report) if the bound expires.
__device__ __forceinline__ bool wait_flag_eq(const int* p, int want, WsHeader* h, long long limit = kWaitCycles) {
  long long t0 = clock64();
  while (ld_acquire_gpu(p) != want) {
    if (clock64() - t0 > limit) {
      report_status(h, SPEAR_ERR_TIMEOUT);
      return false;
    }
    __nanosleep(64);
  }
  return true;
}

// ---------------------------------------------------------------------------
// bf16 helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// int4 (offset binary, 8 nibbles in one word) -> 4 bf16x2 registers.
// Register pi (pi = 0..3) holds (nibble pi, nibble pi + 4) as (low, high).
// Each nibble u is placed in the mantissa of bf16 128.0 (0x4300 | u = 128 + u,
// exact since the bf16 spacing at 128 is 1), then 136 is subtracted, giving
// q = u - 8 exactly.
__device__ __forceinline__ void int4x8_to_bf16x8(uint32_t w, uint32_t (&o)[4]) {
  const uint32_t magic = 0x43004300u;
  const __nv_bfloat162 bias = __floats2bfloat162_rn(136.0f, 136.0f);
#pragma unroll
  for (int pi = 0; pi < 4; ++pi) {
    uint32_t v;
    uint32_t sh = w >> (4 * pi);
    asm("lop3.b32 %0, %1, %2, %3, 0xea;" : "=r"(v) : "r"(sh), "r"(0x000F000Fu), "r"(magic));  // (a & b) | c
    __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&v);
    b = __hsub2(b, bias);
    o[pi] = *reinterpret_cast<uint32_t*>(&b);
  }
}

// ---------------------------------------------------------------------------
// Warp-level tensor-core MMA: D(16x8, fp32) += A(16x16, bf16) . B(16x8, bf16)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// 128-bit streaming load that bypasses L1 allocation (weights are read once).
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// ---------------------------------------------------------------------------
// Thread-block cluster / distributed shared memory
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

__device__ __forceinline__ float4 ld_dsmem_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ uint32_t atom_add_dsmem_acqrel(uint32_t addr, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.cluster.shared::cluster.add.u32 %0, [%1], %2;"
               : "=r"(old)
               : "r"(addr), "r"(v)
               : "memory");
  return old;
}

__device__ __forceinline__ void fence_acq_rel_cluster() {
  asm volatile("fence.acq_rel.cluster;" ::: "memory");
}

// Non-blocking test of an mbarrier phase (local shared memory).
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bulk copy global -> shared (16-byte aligned, size a multiple of 16), counted
// on an mbarrier of this CTA.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// 16 bytes into the shared memory of another CTA of the cluster; completion
// is counted (bytes) on an mbarrier of that CTA.  Both addresses come from mapa.
__device__ __forceinline__ void st_async_f4(uint32_t remote, float4 v, uint32_t remote_bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
                   remote),
               "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w), "r"(remote_bar)
               : "memory");
}

__device__ __forceinline__ float sigmoidf_(float z) { return 1.0f / (1.0f + expf(-z)); }

}  // namespace spear
