// Internal interface between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace spear {

struct WsHeader;

// Record a CUDA failure as the thread's last error; returns SPEAR_ERR_CUDA.
int set_cuda_error(const char* what, cudaError_t e);
// Record a message as the thread's last error; returns `code`.
int set_error(int code, const char* fmt, ...);

// Failure injection for tests (spear_test_inject_timeout): the kernel whose
// publication wait is made unsatisfiable (0 none, 1 decode, 2 tensor core),
// and that wait's bound in SM cycles.
struct TestFault {
  int kernel;
  long long cycles;
};
TestFault test_fault();
// test hook: 1 forces the decode kernels' y-store check to fail, 2 the
// tensor-core kernel's (device-check build only; 0 = off)
int test_force_check();
// An NVTX range named for a C-ABI call, for the call's duration, when tracing
// is on (SPEAR_NVTX=1 in the environment, or spear_set_tracing(1)); nothing otherwise
struct TraceRange {
  bool on;
  explicit TraceRange(const char* name);
  ~TraceRange();
  TraceRange(const TraceRange&) = delete;
  TraceRange& operator=(const TraceRange&) = delete;
};
// K-part flags in the workspace: 4 per (tile, part, 128-row half), tiles x parts <= SMs
constexpr int kKFlagCapacity = 4 * 1024;

struct LayerView;
// Validate a public layer description (same checks as every layer call).
int validate_layer(const struct spear_layer* layer, LayerView* out);
// Multiprocessor count of the current device (cached).
int device_sm_count();

// A validated layer, with typed device pointers.
struct LayerView {
  int K, N, group, r;
  const uint8_t* w;
  const __half* scales;
  const __nv_bfloat16* agt;  // (r+1) x K, or null when r == 0
  const __nv_bfloat16* bpt;  // N x r, or null when r == 0
  float b_g, tau;
  // gate form: 0 scalar sigmoid(x.w_g + b_g); 1 per-rank gamma(t) = sigmoid(W2 relu(W1 t + b1) + b2)
  int gate_kind, gate_h;
  const float *gw1, *gb1, *gw2, *gb2;  // h x r, h, r x h, r (kind 1)
  float alpha;
  // the next call's layer, to be warmed in L2 (prefetch_next hint): packed
  // weights, [A^T ; w_g], B'^T (null / 0 bytes when absent)
  const void* pf[3];
  size_t pf_bytes[3];
};

// ---- decode path (decode.cu) ----
struct DecodePlan {
  int MT;       // token tile: 8 or 16
  int CS;       // cluster size = number of K parts
  int NC;       // clusters
  int kt_part;  // 64-wide k-tiles per K part
  int E2, P2;   // EC pairs, weight pairs
  int RT;       // row stride of the EC projection buffer (32 * E2)
  int ring;     // 4 KB shared-memory ring slots
  size_t smem;
};
DecodePlan plan_decode(int M, int K, int N, int r, int group, int sm_count);
// 0 if the plan respects the kernel's static limits, else a message.
const char* check_decode_plan(const DecodePlan& p);
int launch_decode(const DecodePlan& p, const LayerView& L, const __nv_bfloat16* x, int M, __nv_bfloat16* y,
                  WsHeader* hdr, float* ws_t, __nv_bfloat16* ws_gt, float* gate_out, int* mask_count, bool ec_only,
                  cudaStream_t st);

// ---- decode path for back-to-back launches (decode2.cu) ----
// null if the kernel can run (M, K, N, r), else the reason
const char* decode2_unsupported(int M, int K, int N, int r, int gate_kind, int gate_h);
// bytes of tagged EC projection words the kernel needs in the workspace
size_t decode2_tt_bytes(int r);
int launch_decode2(const LayerView& L, const __nv_bfloat16* x, int M, __nv_bfloat16* y, WsHeader* hdr, void* tt,
                   float* gate_out, int* mask_count, bool ec_only, cudaStream_t st);

// ---- decode path without a serial reducer (decode3.cu) ----
// null if the kernel can run (M, K, N, r, group, gate form), else the reason
const char* decode3_unsupported(int M, int K, int N, int r, int group, int gate_kind, int gate_h);
// bytes of published EC rows the kernel needs in the workspace (fits in decode2_tt_bytes(128))
size_t decode3_tf_bytes();
int launch_decode3(const LayerView& L, const __nv_bfloat16* x, int M, __nv_bfloat16* y, WsHeader* hdr, void* tf,
                   float* gate_out, int* mask_count, bool ec_only, cudaStream_t st);

// ---- standalone EC kernel (ec.cu): y += g * (x.A).B, in place ----
// Two launches: phase 1 writes gt, the gate outputs and the mask count
// (independent of y); phase 2 updates y, after phase 1 in stream order.
struct EcPlan {
  int ksplit;   // K parts of the projection
  int grid;     // CTAs at most
  int RT;       // row stride of projection partials
  size_t part_floats;  // floats of the partial buffer
};
EcPlan plan_ec(int M, int K, int N, int r, int sm_count);
int launch_ec(const EcPlan& p, const LayerView& L, const __nv_bfloat16* x, int M, __nv_bfloat16* y,
              WsHeader* hdr, float* part, int* tickets, __nv_bfloat16* gt, float* gate_out, int* mask_count,
              cudaStream_t st, int phase);

// ---- tensor-core path (tc_gemm.cu) ----
struct TcPlan {
  int grid;
  int m_blocks, n_blocks;
  size_t smem;
};
TcPlan plan_tc(int M, int K, int N, int r, int group, int sm_count);
int launch_tc(const TcPlan& p, const LayerView& L, const __nv_bfloat16* x, int M, __nv_bfloat16* y, bool with_ec,
              WsHeader* hdr, int* mflags, int* kflags, float* kpart, __nv_bfloat16* gt, float* gate_out,
              int* mask_count, cudaStream_t st);

// ---- packing kernels (pack.cu) ----
int launch_quantize(const float* W, int K, int N, int group, int8_t* q, __half* s, cudaStream_t st);
int launch_pack(const int8_t* q, int N, int K, uint8_t* packed, cudaStream_t st);
int launch_unpack(const uint8_t* packed, int N, int K, int8_t* q, cudaStream_t st);
int launch_prescale(const __nv_bfloat16* B, const __half* s, int r, int N, __nv_bfloat16* Bp, bool transpose,
                    cudaStream_t st);
int launch_agt(const __nv_bfloat16* A, const __nv_bfloat16* w_g, int K, int r, __nv_bfloat16* AgT,
               cudaStream_t st);
int launch_transpose_b(const __nv_bfloat16* B, int r, int N, __nv_bfloat16* BT, cudaStream_t st);

}  // namespace spear
