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

#include "common.cuh"
#include "kernels.h"

namespace spear {

// Scratch capacity: header, then the EC rows of whichever decode kernel runs
// the shape: the published rows of the main kernel ([9 EC items][16 tokens]
// [16 rows] fp32), the tagged words of the earlier one (the same shape in
// 8-byte words, r <= 128), or, for shapes only the cluster split-K kernel
// runs, its projection rows [16 tokens][176 fp32] and gated projection
// [16][128 bf16].
constexpr size_t kNoAllocHeader = kWsHeaderBytes;
constexpr size_t kNoAllocEcp = 9 * 16 * 16 * 8;
constexpr size_t kNoAllocT = 16 * 176 * sizeof(float);
constexpr size_t kNoAllocGt = 16 * 128 * 2;
constexpr size_t kNoAllocBytes = 40960;
static_assert(kNoAllocHeader + kNoAllocT + kNoAllocGt <= kNoAllocBytes, "scratch layout exceeds its array");
static_assert(kNoAllocHeader + kNoAllocEcp <= kNoAllocBytes, "scratch layout exceeds its array");

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocBytes];

// Device address of the scratch array on the current device.  Looked up on
// every call (a cheap runtime query), so the address stays right after a
// cudaDeviceReset reloads the module.  The first lookup on a device may load
// the module (lazy loading), which must not happen inside a stream capture.
static int noalloc_scratch_ptr(uint8_t** out) {
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess) return set_cuda_error("cudaGetSymbolAddress(scratch)", e);
  *out = static_cast<uint8_t*>(p);
  return SPEAR_OK;
}

}  // namespace spear

using namespace spear;

extern "C" int spear_linear_forward_decode_noalloc(const spear_layer* layer, const uint16_t* x, int M, uint16_t* y,
                                                   float* gate_out, int* mask_count, void* stream) {
  TraceRange trace_("spear_linear_forward_decode_noalloc");
  LayerView L;
  int rc = validate_layer(layer, &L);
  if (rc) return rc;
  if (M < 1 || M > 16)
    return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE,
                     "allocation-free call supports 1 <= M <= 16 (its scratch array holds 16 tokens); M=%d", M);
  if (!x || !y) return set_error(SPEAR_ERR_INVALID_ARG, "x and y must be non-NULL");
  if ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(y) & 15))
    return set_error(SPEAR_ERR_ALIGNMENT, "x and y must be 16-byte aligned");
  if ((gate_out && (reinterpret_cast<uintptr_t>(gate_out) & 3)) ||
      (mask_count && (reinterpret_cast<uintptr_t>(mask_count) & 3)))
    return set_error(SPEAR_ERR_ALIGNMENT, "gate_out and mask_count must be 4-byte aligned");
  // the kernel that runs the shape: 3 (no serial reducer), 2, or 1 (cluster split-K)
  int kind = 1;
  if (!decode3_unsupported(M, L.K, L.N, L.r, L.group, L.gate_kind, L.gate_h))
    kind = 3;
  else if (!decode2_unsupported(M, L.K, L.N, L.r, L.gate_kind, L.gate_h))
    kind = 2;
  if (kind == 1 && L.r > 0 && L.gate_kind)
    return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "decode path: the rank gate needs the main decode kernels");
  if (kind == 3 && decode3_tf_bytes() > kNoAllocEcp)
    return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "EC projection scratch exceeds the allocation-free array");
  if (kind == 2 && decode2_tt_bytes(L.r) > kNoAllocEcp)
    return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "EC projection scratch exceeds the allocation-free array");
  const DecodePlan p = kind == 1 ? plan_decode(M, L.K, L.N, L.r, L.group, device_sm_count()) : DecodePlan{};
  const char* why = kind == 1 ? check_decode_plan(p) : nullptr;
  if (why) return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "decode path: %s", why);
  uint8_t* scratch = nullptr;
  rc = noalloc_scratch_ptr(&scratch);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The launch header (epoch, arrival counters, publication flags) and, for
  // the kernel that tags its EC words, those words must start at zero.  The
  // first int of the header, the device status word, is left alone: it keeps
  // the first device-side error until spear_read_status_noalloc reads it.
  const size_t clear = kNoAllocHeader + (kind == 2 ? kNoAllocEcp : 0) - sizeof(int);
  cudaError_t e = cudaMemsetAsync(scratch + sizeof(int), 0, clear, st);
  if (e != cudaSuccess) return set_cuda_error("scratch header clear", e);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(scratch);
  const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(x);
  __nv_bfloat16* yb = reinterpret_cast<__nv_bfloat16*>(y);
  if (kind == 3) return launch_decode3(L, xb, M, yb, hdr, scratch + kNoAllocHeader, gate_out, mask_count, false, st);
  if (kind == 2) return launch_decode2(L, xb, M, yb, hdr, scratch + kNoAllocHeader, gate_out, mask_count, false, st);
  float* tbuf = reinterpret_cast<float*>(scratch + kNoAllocHeader);
  __nv_bfloat16* gt = reinterpret_cast<__nv_bfloat16*>(scratch + kNoAllocHeader + kNoAllocT);
  return launch_decode(p, L, xb, M, yb, hdr, tbuf, gt, gate_out, mask_count, false, st);
}

extern "C" int spear_read_status_noalloc(int* device_status, void* stream) {
  TraceRange trace_("spear_read_status_noalloc");
  if (!device_status) return set_error(SPEAR_ERR_INVALID_ARG, "device_status is NULL");
  uint8_t* scratch = nullptr;
  int rc = noalloc_scratch_ptr(&scratch);
  if (rc) return rc;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return set_cuda_error("stream synchronize", e);
  int v = 0;
  e = cudaMemcpy(&v, scratch, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return set_cuda_error("status read", e);
  if (v) {
    const int zero = 0;
    e = cudaMemcpy(scratch, &zero, sizeof(int), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return set_cuda_error("status clear", e);
  }
  *device_status = v;
  return SPEAR_OK;
}
