// Allocation-free variant of the decode-path layer call.
//
// Some callers cannot allocate device memory at the point where they run the
// layer: code that executes while another component owns the CUDA allocator
// (a serving engine's memory pool, where a stray cudaMalloc fragments or
// oversubscribes the pool), latency-critical token loops in which an
// allocation would synchronise the device, and plugin hosts that hand the
// library only input and output buffers.  For them this entry point keeps its
// scratch (launch header, EC projection, gated projection) in a file-scope
// device array instead of a caller-provided workspace.
//
// The array is shared by every call in the process on that device and keeps
// the last call's contents; each call first clears the part that must start
// at zero (the launch header).  Two calls whose executions overlap on the GPU
// (different streams, or the same array reached from several host threads
// without ordering) race on the array and give wrong results.
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace spear {

// Scratch capacity: header, then either the tagged EC projection words of the
// decode kernel ([9 EC strips][16 tokens][16 rows] x 8 bytes, r <= 128) or, for
// shapes only the cluster split-K kernel runs, its projection rows [16 tokens]
// [176 fp32] and gated projection [16][128 bf16].
constexpr size_t kNoAllocHeader = kWsHeaderBytes;
constexpr size_t kNoAllocEcp = 9 * 16 * 16 * 8;
constexpr size_t kNoAllocT = 16 * 176 * sizeof(float);
constexpr size_t kNoAllocGt = 16 * 128 * 2;
constexpr size_t kNoAllocBytes = 40960;
static_assert(kNoAllocHeader + kNoAllocT + kNoAllocGt <= kNoAllocBytes, "scratch layout exceeds its array");
static_assert(kNoAllocHeader + kNoAllocEcp <= kNoAllocBytes, "scratch layout exceeds its array");

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocBytes];

// Device address of the scratch array, looked up once per device (with that
// device current) and cached.
static int noalloc_scratch_ptr(uint8_t** out) {
  static std::mutex mu;
  static uint8_t* cache[64] = {nullptr};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return set_cuda_error("cudaGetDevice", e);
  if (dev < 0 || dev >= 64) return set_error(SPEAR_ERR_INVALID_ARG, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lk(mu);
  if (!cache[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return set_cuda_error("cudaGetSymbolAddress(scratch)", e);
    cache[dev] = static_cast<uint8_t*>(p);
  }
  *out = cache[dev];
  return SPEAR_OK;
}

}  // namespace spear

using namespace spear;

extern "C" int spear_linear_forward_decode_noalloc(const spear_layer* layer, const uint16_t* x, int M, uint16_t* y,
                                                   float* gate_out, int* mask_count, void* stream) {
  LayerView L;
  int rc = validate_layer(layer, &L);
  if (rc) return rc;
  if (M < 1 || M > 16)
    return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE,
                     "allocation-free call supports 1 <= M <= 16 (its scratch array holds 16 tokens); M=%d", M);
  if (!x || !y) return set_error(SPEAR_ERR_INVALID_ARG, "x and y must be non-NULL");
  if ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(y) & 15) ||
      (gate_out && (reinterpret_cast<uintptr_t>(gate_out) & 3)) ||
      (mask_count && (reinterpret_cast<uintptr_t>(mask_count) & 3)))
    return set_error(SPEAR_ERR_ALIGNMENT, "x and y must be 16-byte aligned");
  const bool v2 = decode2_unsupported(M, L.K, L.N, L.r, L.gate_kind, L.gate_h) == nullptr;
  if (!v2 && L.gate_kind)
    return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "decode path: the rank gate needs the main decode kernel");
  if (v2 && decode2_tt_bytes(L.r) > kNoAllocEcp)
    return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "EC projection scratch exceeds the allocation-free array");
  const DecodePlan p = v2 ? DecodePlan{} : plan_decode(M, L.K, L.N, L.r, L.group, device_sm_count());
  const char* why = v2 ? nullptr : check_decode_plan(p);
  if (why) return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "decode path: %s", why);
  uint8_t* scratch = nullptr;
  rc = noalloc_scratch_ptr(&scratch);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the launch header (epoch, arrival counters, flags) and the tagged EC
  // projection words (their tags are checked against the header's epoch) must
  // start at zero
  cudaError_t e = cudaMemsetAsync(scratch, 0, kNoAllocHeader + (v2 ? kNoAllocEcp : 0), st);
  if (e != cudaSuccess) return set_cuda_error("scratch header clear", e);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(scratch);
  if (v2)
    return launch_decode2(L, reinterpret_cast<const __nv_bfloat16*>(x), M, reinterpret_cast<__nv_bfloat16*>(y), hdr,
                          scratch + kNoAllocHeader, gate_out, mask_count, false, st);
  float* tbuf = reinterpret_cast<float*>(scratch + kNoAllocHeader);
  __nv_bfloat16* gt = reinterpret_cast<__nv_bfloat16*>(scratch + kNoAllocHeader + kNoAllocT);
  return launch_decode(p, L, reinterpret_cast<const __nv_bfloat16*>(x), M, reinterpret_cast<__nv_bfloat16*>(y), hdr,
                       tbuf, gt, gate_out, mask_count, false, st);
}
