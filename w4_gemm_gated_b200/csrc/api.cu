// C ABI of the library (declared in include/spear.h): argument validation,
// workspace layout, the measured-time dispatch table and path selection.
#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdlib>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <tuple>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "kernels.h"

namespace spear {

static thread_local std::string g_last_error;

int set_error(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int set_cuda_error(const char* what, cudaError_t e) {
  return set_error(SPEAR_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static std::mutex g_fault_mu;
static TestFault g_fault = {0, 0};
std::atomic<int> g_force_check{0};

// tracing: -1 until the environment is read (SPEAR_NVTX=1 turns it on)
static std::atomic<int> g_trace{-1};
static bool tracing() {
  int v = g_trace.load();
  if (v < 0) {
    const char* e = std::getenv("SPEAR_NVTX");
    int expected = -1;
    g_trace.compare_exchange_strong(expected, (e && e[0] == '1') ? 1 : 0);
    v = g_trace.load();
  }
  return v > 0;
}
TraceRange::TraceRange(const char* name) : on(tracing()) {
  if (on) nvtxRangePushA(name);
}
TraceRange::~TraceRange() {
  if (on) nvtxRangePop();
}
void set_tracing(bool on) { g_trace.store(on ? 1 : 0); }
int test_force_check() { return g_force_check.load(); }

TestFault test_fault() {
  std::lock_guard<std::mutex> lk(g_fault_mu);
  return g_fault;
}

static int sm_count() {
  static std::mutex mu;
  static std::map<int, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    dev = -1;  // no usable device: size plans for a full B200
  }
  std::lock_guard<std::mutex> lk(mu);
  auto it = cache.find(dev);
  if (it != cache.end()) return it->second;
  int n = 0;
  if (dev < 0 || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = 148;
  }
  cache[dev] = n;
  return n;
}

static bool valid_r(int r) { return r == 0 || r == 16 || r == 32 || r == 64 || r == 128; }

static int check_kn(int K, int N) {
  if (K <= 0 || N <= 0 || K % 128 || N % 128)
    return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "K=%d N=%d: both must be positive multiples of 128", K, N);
  if ((long long)K * N > (1LL << 34)) return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "K*N too large");
  return SPEAR_OK;
}

static int check_layer(const spear_layer* l, LayerView* out) {
  if (!l) return set_error(SPEAR_ERR_INVALID_ARG, "layer is NULL");
  int rc = check_kn(l->K, l->N);
  if (rc) return rc;
  if (l->group != 0 && l->group != 128)
    return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "group=%d: must be 0 or 128", l->group);
  if (!valid_r(l->r)) return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "r=%d: must be 0, 16, 32, 64 or 128", l->r);
  if (!l->w_packed || !l->scales) return set_error(SPEAR_ERR_INVALID_ARG, "w_packed / scales is NULL");
  if (l->r > 0 && (!l->AgT || !l->BpT)) return set_error(SPEAR_ERR_INVALID_ARG, "r > 0 needs AgT and BpT");
  if (!aligned16(l->w_packed) || !aligned16(l->scales) || (l->r > 0 && (!aligned16(l->AgT) || !aligned16(l->BpT))))
    return set_error(SPEAR_ERR_ALIGNMENT, "layer device pointers must be 16-byte aligned");
  out->K = l->K;
  out->N = l->N;
  out->group = l->group;
  out->r = l->r;
  out->w = l->w_packed;
  out->scales = reinterpret_cast<const __half*>(l->scales);
  out->agt = l->r > 0 ? reinterpret_cast<const __nv_bfloat16*>(l->AgT) : nullptr;
  out->bpt = l->r > 0 ? reinterpret_cast<const __nv_bfloat16*>(l->BpT) : nullptr;
  out->b_g = l->b_g;
  out->tau = l->gate_tau > 0.f ? l->gate_tau : 0.1f;
  out->gate_kind = l->gate_kind;
  out->gate_h = 0;
  out->gw1 = out->gb1 = out->gw2 = out->gb2 = nullptr;
  out->alpha = 1.f;
  if (l->gate_kind != SPEAR_GATE_SCALAR && l->gate_kind != SPEAR_GATE_RANK_MLP)
    return set_error(SPEAR_ERR_INVALID_ARG, "gate_kind=%d: must be 0 (scalar) or 1 (rank MLP)", l->gate_kind);
  if (l->gate_kind == SPEAR_GATE_RANK_MLP) {
    if (l->r == 0) return set_error(SPEAR_ERR_INVALID_ARG, "the rank gate needs an EC (r > 0)");
    if (l->gate_hidden != 8 && l->gate_hidden != 16 && l->gate_hidden != 32)
      return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "gate_hidden=%d: must be 8, 16 or 32", l->gate_hidden);
    if (!l->gate_w1 || !l->gate_b1 || !l->gate_w2 || !l->gate_b2)
      return set_error(SPEAR_ERR_INVALID_ARG, "the rank gate needs gate_w1, gate_b1, gate_w2 and gate_b2");
    if (!aligned16(l->gate_w1) || !aligned16(l->gate_b1) || !aligned16(l->gate_w2) || !aligned16(l->gate_b2))
      return set_error(SPEAR_ERR_ALIGNMENT, "rank-gate parameters must be 16-byte aligned");
    out->gate_h = l->gate_hidden;
    out->gw1 = l->gate_w1;
    out->gb1 = l->gate_b1;
    out->gw2 = l->gate_w2;
    out->gb2 = l->gate_b2;
    out->alpha = l->gate_alpha;
  }
  for (int i = 0; i < 3; ++i) {
    out->pf[i] = nullptr;
    out->pf_bytes[i] = 0;
  }
  if (const spear_layer* nx = l->prefetch_next) {
    // the hint's buffers are only prefetched: validate what is read of them
    if (check_kn(nx->K, nx->N)) return set_error(SPEAR_ERR_INVALID_ARG, "prefetch_next: bad K=%d N=%d", nx->K, nx->N);
    if (!valid_r(nx->r)) return set_error(SPEAR_ERR_INVALID_ARG, "prefetch_next: bad r=%d", nx->r);
    if (!nx->w_packed || !aligned16(nx->w_packed) ||
        (nx->r > 0 && (!nx->AgT || !nx->BpT || !aligned16(nx->AgT) || !aligned16(nx->BpT))))
      return set_error(SPEAR_ERR_INVALID_ARG, "prefetch_next: NULL or unaligned device pointer");
    out->pf[0] = nx->w_packed;
    out->pf_bytes[0] = (size_t)nx->N * nx->K / 2;
    if (nx->r > 0) {
      out->pf[1] = nx->AgT;
      out->pf_bytes[1] = (size_t)(nx->r + 1) * nx->K * 2;
      out->pf[2] = nx->BpT;
      out->pf_bytes[2] = (size_t)nx->N * nx->r * 2;
    }
  }
  return SPEAR_OK;
}

int validate_layer(const spear_layer* layer, LayerView* out) { return check_layer(layer, out); }
int device_sm_count() { return sm_count(); }

// ---------------------------------------------------------------------------
// workspace layout
// ---------------------------------------------------------------------------
struct WsLayout {
  size_t hdr, tickets, tcflags, kflags, t, gt, part, kpart, total;
  int n_flags;
};

static size_t up256(size_t v) { return (v + 255) & ~(size_t)255; }

// Every region that carries state between launches (header, flags,
// tickets) sits at a fixed offset with capacity for the largest M, so one
// workspace can serve any M, path and layer in any order; only the stateless
// scratch after them (gated projection, K-split partials) grows with M.
static constexpr int kMaxM = 65536;
static constexpr int kFlagCap = kMaxM / 16 + 64;  // 16-token blocks (+ slack)
static constexpr int kKFlagCap = kKFlagCapacity;

static WsLayout ws_layout_uncached(const LayerView& L, int M_max) {
  WsLayout w = {};
  const int Mpad = ((M_max + 255) / 256) * 256;  // tensor-core tiles of up to 256 tokens
  const int RT = 32 * ((128 / 16 + 2) / 2) + 16;  // row stride for the largest rank
  w.n_flags = kFlagCap;
  size_t off = kWsHeaderBytes;
  w.hdr = 0;
  w.tickets = off;
  off = up256(off + sizeof(int) * kFlagCap);
  w.tcflags = off;
  off = up256(off + sizeof(int) * 4 * kFlagCap);
  w.kflags = off;
  off = up256(off + sizeof(int) * kKFlagCap);
  w.t = off;
  off = up256(off + sizeof(float) * std::max<size_t>(16 * (size_t)RT, decode2_tt_bytes(128) / sizeof(float)));
  w.gt = off;
  off = up256(off + 2 * (size_t)Mpad * (L.r > 0 ? L.r : 1));
  w.part = off;
  size_t part_floats = 0;
  if (L.r > 0) {
    // largest partial buffer over every M <= M_max (the K split shrinks as M grows)
    for (int M = 16; M <= M_max + 15; M += 16) {
      EcPlan p = plan_ec(std::min(M, M_max), L.K, L.N, L.r, sm_count());
      part_floats = std::max(part_floats, p.part_floats);
    }
  }
  off = up256(off + sizeof(float) * part_floats);
  // K-part partial accumulators of the tensor-core tiles (M > 16): tiles x
  // parts <= SMs, each 128 tokens x 256 channels fp32
  w.kpart = off;
  off = up256(off + (M_max > 16 ? (size_t)sm_count() * 128 * 256 * sizeof(float) : 0));
  w.total = off;
  return w;
}

static WsLayout ws_layout(const LayerView& L, int M_max) {
  static std::mutex mu;
  static std::map<std::tuple<int, int, int, int, int, int>, WsLayout> cache;
  const auto key = std::make_tuple(L.K, L.N, L.r, L.group, M_max, sm_count());
  {
    std::lock_guard<std::mutex> lk(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
  }
  const WsLayout w = ws_layout_uncached(L, M_max);
  std::lock_guard<std::mutex> lk(mu);
  if (cache.size() > 4096) cache.clear();
  cache[key] = w;
  return w;
}

// ---------------------------------------------------------------------------
// dispatch table
// ---------------------------------------------------------------------------
// K, N, r, group, gate kind, gate bottleneck width, M bucket: a scalar-gate and a
// rank-gate layer of the same shape run at different speeds, so they have
// separate entries (gate fields are 0 for the scalar gate and without an EC)
using DKey = std::tuple<int, int, int, int, int, int, int>;
static std::mutex g_dmu;
struct DEntry {
  int path;
  float us;  // measured time of that path at the bucket's M, < 0 if not measured
};
static std::map<DKey, DEntry> g_table;

static int m_bucket(int M) {
  int b = 1;
  while (b < M) b <<= 1;
  return b;
}

static DKey dkey(const LayerView& L, int M) {
  const int gk = L.r > 0 ? L.gate_kind : 0;
  return DKey(L.K, L.N, L.r, L.group, gk, gk ? L.gate_h : 0, m_bucket(M));
}

// The device a table is measured on: its name and multiprocessor count.
static std::string device_ident(int* sms_out) {
  int dev = 0;
  cudaDeviceProp prop;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaGetDeviceProperties(&prop, dev) != cudaSuccess) {
    cudaGetLastError();
    *sms_out = 0;
    return "no-device";
  }
  *sms_out = prop.multiProcessorCount;
  return prop.name;
}

static int default_path(const LayerView& L, int M) {
  (void)L;
  return M <= 16 ? SPEAR_PATH_DECODE : SPEAR_PATH_FUSED;
}

static int choose_path(const LayerView& L, int M) {
  {
    std::lock_guard<std::mutex> lk(g_dmu);
    auto it = g_table.find(dkey(L, M));
    if (it != g_table.end()) {
      const int p = it->second.path;
      if (!(p == SPEAR_PATH_DECODE && M > 16)) return p;
    }
  }
  return default_path(L, M);
}

// ---------------------------------------------------------------------------
// semi-fused prefill: a side stream per device and the fork / join events
// ---------------------------------------------------------------------------
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
static std::mutex g_side_mu;  // held from the fork to the join of one call

static int side_stream(SideStream** out) {
  static std::map<int, SideStream> streams;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return set_cuda_error("get device", e);
  SideStream& ss = streams[dev];
  if (!ss.s) {
    int lo = 0, hi = 0;
    cudaDeviceGetStreamPriorityRange(&lo, &hi);
    // the projection is short and lies on the DAG's critical path: its CTAs
    // go to the block scheduler ahead of the GEMM's tiles
    e = cudaStreamCreateWithPriority(&ss.s, cudaStreamNonBlocking, hi);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming);
    if (e != cudaSuccess) {
      ss = SideStream{};
      return set_cuda_error("side stream create", e);
    }
  }
  *out = &ss;
  return SPEAR_OK;
}

// ---------------------------------------------------------------------------
// forward
// ---------------------------------------------------------------------------
static int run_path(const LayerView& L, const __nv_bfloat16* x, int M, __nv_bfloat16* y, uint8_t* ws,
                    const WsLayout& wl, float* gate_out, int* mask_count, int path, cudaStream_t st) {
  WsHeader* hdr = reinterpret_cast<WsHeader*>(ws + wl.hdr);
  int* tickets = reinterpret_cast<int*>(ws + wl.tickets);
  int* tcflags = reinterpret_cast<int*>(ws + wl.tcflags);
  int* kflags = reinterpret_cast<int*>(ws + wl.kflags);
  float* kpart = wl.total > wl.kpart ? reinterpret_cast<float*>(ws + wl.kpart) : nullptr;
  float* tbuf = reinterpret_cast<float*>(ws + wl.t);
  __nv_bfloat16* gt = reinterpret_cast<__nv_bfloat16*>(ws + wl.gt);
  float* part = reinterpret_cast<float*>(ws + wl.part);
  const int sms = sm_count();
  // A decode-path launch (M <= 16) of layer LL: the kernel without a serial
  // reducer where it runs the shape, else the earlier decode kernel, else the
  // cluster split-K kernel (long or ragged K).
  auto decode_launch = [&](const LayerView& LL, float* go, int* mc, bool ec_only) -> int {
    if (!decode3_unsupported(M, LL.K, LL.N, LL.r, LL.group, LL.gate_kind, LL.gate_h))
      return launch_decode3(LL, x, M, y, hdr, tbuf, go, mc, ec_only, st);
    if (!decode2_unsupported(M, LL.K, LL.N, LL.r, LL.gate_kind, LL.gate_h))
      return launch_decode2(LL, x, M, y, hdr, tbuf, go, mc, ec_only, st);
    if (LL.r > 0 && LL.gate_kind)
      return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "decode path: the rank gate needs the main decode kernels (%s)",
                       decode2_unsupported(M, LL.K, LL.N, LL.r, LL.gate_kind, LL.gate_h));
    DecodePlan p = plan_decode(M, LL.K, LL.N, LL.r, LL.group, sms);
    const char* why = check_decode_plan(p);
    if (why) return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "decode path: %s", why);
    return launch_decode(p, LL, x, M, y, hdr, tbuf, gt, go, mc, ec_only, st);
  };
  LayerView L0 = L;  // the same layer with the EC disabled
  L0.r = 0;
  L0.agt = nullptr;
  L0.bpt = nullptr;
  L0.gate_kind = 0;
  if (path == SPEAR_PATH_DECODE) {
    if (M > 16) return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "decode path needs M <= 16 (M=%d)", M);
    return decode_launch(L, gate_out, mask_count, false);
  }
  if (path == SPEAR_PATH_UNFUSED) {
    int rc;
    if (M <= 16) {
      if (L.r > 0 && L.gate_kind && decode3_unsupported(M, L.K, L.N, L.r, L.group, L.gate_kind, L.gate_h) &&
          decode2_unsupported(M, L.K, L.N, L.r, L.gate_kind, L.gate_h))
        return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "unfused path at M <= 16: the rank gate needs the main decode kernels");
      rc = decode_launch(L0, L.r > 0 ? nullptr : gate_out, L.r > 0 ? nullptr : mask_count, false);
      if (rc || L.r == 0) return rc;
      // the separate EC launch: a decode kernel in EC-only mode, y += g (t . B) in place
      return decode_launch(L, gate_out, mask_count, true);
    }
    TcPlan p = plan_tc(M, L.K, L.N, 0, L.group, sms);
    rc = launch_tc(p, L0, x, M, y, false, hdr, tcflags, kflags, kpart, gt, L.r > 0 ? nullptr : gate_out,
                   L.r > 0 ? nullptr : mask_count, st);
    if (rc || L.r == 0) return rc;
    // the separate EC kernel: projection and gate, then the update of y
    EcPlan ep = plan_ec(M, L.K, L.N, L.r, sms);
    rc = launch_ec(ep, L, x, M, y, hdr, part, tickets, gt, gate_out, mask_count, st, 1);
    if (rc) return rc;
    return launch_ec(ep, L, x, M, y, hdr, part, tickets, gt, nullptr, nullptr, st, 2);
  }
  if (path == SPEAR_PATH_SEMIFUSED) {
    auto gemm = [&](float* go, int* mc) {
      if (M <= 16) return decode_launch(L0, go, mc, false);
      TcPlan p = plan_tc(M, L.K, L.N, 0, L.group, sms);
      return launch_tc(p, L0, x, M, y, false, hdr, tcflags, kflags, kpart, gt, go, mc, st);
    };
    if (L.r == 0) return gemm(gate_out, mask_count);
    const EcPlan ep = plan_ec(M, L.K, L.N, L.r, sms);
    std::lock_guard<std::mutex> lk(g_side_mu);
    SideStream* ss = nullptr;
    int rc = side_stream(&ss);
    if (rc) return rc;
    cudaError_t e = cudaEventRecord(ss->fork, st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(ss->s, ss->fork, 0);
    if (e != cudaSuccess) return set_cuda_error("semi-fused fork", e);
    rc = launch_ec(ep, L, x, M, y, hdr, part, tickets, gt, gate_out, mask_count, ss->s, 1);
    e = cudaEventRecord(ss->join, ss->s);
    // the GEMM goes on `st` after the fork only, so it runs beside the projection
    if (rc == SPEAR_OK && e == cudaSuccess) rc = gemm(nullptr, nullptr);
    // join on every return, so a capture of `st` never loses the side branch
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st, ss->join, 0);
    if (e != cudaSuccess) return set_cuda_error("semi-fused join", e);
    if (rc) return rc;
    return launch_ec(ep, L, x, M, y, hdr, part, tickets, gt, nullptr, nullptr, st, 2);
  }
  if (path == SPEAR_PATH_FUSED) {
    TcPlan p = plan_tc(M, L.K, L.N, L.r, L.group, sms);
    return launch_tc(p, L, x, M, y, L.r > 0, hdr, tcflags, kflags, kpart, gt, gate_out, mask_count, st);
  }
  return set_error(SPEAR_ERR_INVALID_ARG, "unknown path %d", path);
}

static int forward_impl(const spear_layer* layer, const uint16_t* x, int M, uint16_t* y, void* ws, size_t ws_bytes,
                        float* gate_out, int* mask_count, int path, void* stream) {
  LayerView L;
  int rc = check_layer(layer, &L);
  if (rc) return rc;
  if (M < 1 || M > 65536) return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "M=%d outside [1, 65536]", M);
  if (!x || !y || !ws) return set_error(SPEAR_ERR_INVALID_ARG, "x, y and ws must be non-NULL");
  if (!aligned16(x) || !aligned16(y) || !aligned16(ws) || (gate_out && ((uintptr_t)gate_out & 3)) ||
      (mask_count && ((uintptr_t)mask_count & 3)))
    return set_error(SPEAR_ERR_ALIGNMENT, "x, y, ws must be 16-byte aligned");
  if (path < SPEAR_PATH_AUTO || path > SPEAR_PATH_SEMIFUSED)
    return set_error(SPEAR_ERR_INVALID_ARG, "bad path %d", path);
  const WsLayout wl = ws_layout(L, M);
  if (ws_bytes < wl.total)
    return set_error(SPEAR_ERR_WORKSPACE, "workspace of %zu bytes, %zu needed for M=%d", ws_bytes, wl.total, M);
  if (path == SPEAR_PATH_AUTO) path = choose_path(L, M);
  if (path == SPEAR_PATH_DECODE && M > 16)
    return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "decode path needs M <= 16 (M=%d)", M);
  return run_path(L, reinterpret_cast<const __nv_bfloat16*>(x), M, reinterpret_cast<__nv_bfloat16*>(y),
                  static_cast<uint8_t*>(ws), wl, gate_out, mask_count, path, static_cast<cudaStream_t>(stream));
}

}  // namespace spear

using namespace spear;

extern "C" {

const char* spear_last_error(void) { return g_last_error.c_str(); }

const char* spear_status_string(int status) {
  switch (status) {
    case SPEAR_OK: return "SPEAR_OK";
    case SPEAR_ERR_INVALID_ARG: return "SPEAR_ERR_INVALID_ARG";
    case SPEAR_ERR_UNSUPPORTED_SHAPE: return "SPEAR_ERR_UNSUPPORTED_SHAPE";
    case SPEAR_ERR_ALIGNMENT: return "SPEAR_ERR_ALIGNMENT";
    case SPEAR_ERR_WORKSPACE: return "SPEAR_ERR_WORKSPACE";
    case SPEAR_ERR_CUDA: return "SPEAR_ERR_CUDA";
    case SPEAR_ERR_TIMEOUT: return "SPEAR_ERR_TIMEOUT";
    case SPEAR_ERR_DEVICE_CHECK: return "SPEAR_ERR_DEVICE_CHECK";
    default: return "SPEAR_ERR_UNKNOWN";
  }
}

int spear_version(void) { return 100; }

int spear_test_inject_timeout(int kernel, long long wait_cycles) {
  g_last_error.clear();
  if (kernel < 0 || kernel > 2) return set_error(SPEAR_ERR_INVALID_ARG, "kernel=%d: must be 0, 1 or 2", kernel);
  if (kernel != 0 && wait_cycles < 1) return set_error(SPEAR_ERR_INVALID_ARG, "wait_cycles must be >= 1");
  std::lock_guard<std::mutex> lk(g_fault_mu);
  g_fault = TestFault{kernel, kernel ? wait_cycles : 0};
  return SPEAR_OK;
}

int spear_test_force_device_check(int kernel) {
  g_last_error.clear();
  if (kernel < 0 || kernel > 2) return set_error(SPEAR_ERR_INVALID_ARG, "kernel=%d: must be 0, 1 or 2", kernel);
  g_force_check.store(kernel);
  return SPEAR_OK;
}

int spear_set_tracing(int on) {
  g_last_error.clear();
  set_tracing(on != 0);
  return SPEAR_OK;
}

int spear_tracing_enabled(void) { return tracing() ? 1 : 0; }

int spear_device_checks_enabled(void) {
#ifdef SPEAR_DEVICE_CHECKS
  return 1;
#else
  return 0;
#endif
}

size_t spear_w4_packed_bytes(int N, int K) {
  if (N <= 0 || K <= 0 || N % 16 || K % 64) return 0;
  return (size_t)N * K / 2;
}

size_t spear_scale_count(int N, int K, int group) {
  if (N <= 0 || K <= 0) return 0;
  if (group == 0) return (size_t)N;
  if (group == 128 && K % 128 == 0) return (size_t)(K / 128) * N;
  return 0;
}

int spear_w4_quantize(const float* W, int K, int N, int group, int8_t* q, uint16_t* scales, void* stream) {
  TraceRange trace_("spear_w4_quantize");
  g_last_error.clear();
  if (!W || !q || !scales) return set_error(SPEAR_ERR_INVALID_ARG, "NULL pointer");
  if (K <= 0 || N <= 0 || K % 32 || N % 32)
    return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "quantize needs K, N positive multiples of 32");
  if (group != 0 && !(group == 128 && K % 128 == 0))
    return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "group=%d with K=%d", group, K);
  if (!aligned16(W) || !aligned16(q) || !aligned16(scales)) return set_error(SPEAR_ERR_ALIGNMENT, "unaligned pointer");
  return launch_quantize(W, K, N, group, q, reinterpret_cast<__half*>(scales), static_cast<cudaStream_t>(stream));
}

int spear_w4_pack(const int8_t* q, int N, int K, uint8_t* packed, void* stream) {
  TraceRange trace_("spear_w4_pack");
  g_last_error.clear();
  if (!q || !packed) return set_error(SPEAR_ERR_INVALID_ARG, "NULL pointer");
  if (N <= 0 || K <= 0 || N % 16 || K % 64)
    return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "pack needs N %% 16 == 0 and K %% 64 == 0");
  if (!aligned16(q) || !aligned16(packed)) return set_error(SPEAR_ERR_ALIGNMENT, "unaligned pointer");
  return launch_pack(q, N, K, packed, static_cast<cudaStream_t>(stream));
}

int spear_w4_unpack(const uint8_t* packed, int N, int K, int8_t* q, void* stream) {
  TraceRange trace_("spear_w4_unpack");
  g_last_error.clear();
  if (!q || !packed) return set_error(SPEAR_ERR_INVALID_ARG, "NULL pointer");
  if (N <= 0 || K <= 0 || N % 16 || K % 64)
    return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "unpack needs N %% 16 == 0 and K %% 64 == 0");
  if (!aligned16(q) || !aligned16(packed)) return set_error(SPEAR_ERR_ALIGNMENT, "unaligned pointer");
  return launch_unpack(packed, N, K, q, static_cast<cudaStream_t>(stream));
}

int spear_ec_prescale_B(const uint16_t* B, const uint16_t* scales, int r, int N, uint16_t* Bp, void* stream) {
  TraceRange trace_("spear_ec_prescale_B");
  g_last_error.clear();
  if (!B || !scales || !Bp) return set_error(SPEAR_ERR_INVALID_ARG, "NULL pointer");
  if (r <= 0 || N <= 0) return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "r and N must be positive");
  if (!aligned16(B) || !aligned16(scales) || !aligned16(Bp)) return set_error(SPEAR_ERR_ALIGNMENT, "unaligned pointer");
  return launch_prescale(reinterpret_cast<const __nv_bfloat16*>(B), reinterpret_cast<const __half*>(scales), r, N,
                         reinterpret_cast<__nv_bfloat16*>(Bp), false, static_cast<cudaStream_t>(stream));
}

size_t spear_ec_agt_count(int K, int r) { return (K > 0 && r > 0) ? (size_t)(r + 1) * K : 0; }
size_t spear_ec_bpt_count(int N, int r) { return (N > 0 && r > 0) ? (size_t)N * r : 0; }

int spear_ec_pack(const uint16_t* A, const uint16_t* B, const uint16_t* w_g, const uint16_t* scales, int K, int N,
                  int r, int group, uint16_t* AgT, uint16_t* BpT, void* stream) {
  TraceRange trace_("spear_ec_pack");
  g_last_error.clear();
  if (!A || !B || !w_g || !AgT || !BpT || (group == 0 && !scales)) return set_error(SPEAR_ERR_INVALID_ARG, "NULL pointer");
  int rc = check_kn(K, N);
  if (rc) return rc;
  if (r <= 0 || !valid_r(r)) return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "r=%d", r);
  if (group != 0 && group != 128) return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "group=%d", group);
  if (!aligned16(A) || !aligned16(B) || !aligned16(w_g) || !aligned16(AgT) || !aligned16(BpT))
    return set_error(SPEAR_ERR_ALIGNMENT, "unaligned pointer");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  rc = launch_agt(reinterpret_cast<const __nv_bfloat16*>(A), reinterpret_cast<const __nv_bfloat16*>(w_g), K, r,
                  reinterpret_cast<__nv_bfloat16*>(AgT), st);
  if (rc) return rc;
  if (group == 0)
    return launch_prescale(reinterpret_cast<const __nv_bfloat16*>(B), reinterpret_cast<const __half*>(scales), r, N,
                           reinterpret_cast<__nv_bfloat16*>(BpT), true, st);
  return launch_transpose_b(reinterpret_cast<const __nv_bfloat16*>(B), r, N, reinterpret_cast<__nv_bfloat16*>(BpT), st);
}

size_t spear_workspace_bytes(const spear_layer* layer, int M_max) {
  LayerView L;
  if (check_layer(layer, &L) != SPEAR_OK || M_max < 1 || M_max > 65536) return 0;
  return ws_layout(L, M_max).total;
}

int spear_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  TraceRange trace_("spear_workspace_init");
  g_last_error.clear();
  if (!ws || ws_bytes < kWsHeaderBytes) return set_error(SPEAR_ERR_INVALID_ARG, "bad workspace");
  cudaError_t e = cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SPEAR_OK : set_cuda_error("workspace memset", e);
}

int spear_linear_forward(const spear_layer* layer, const uint16_t* x, int M, uint16_t* y, void* ws, size_t ws_bytes,
                         float* gate_out, int* mask_count, void* stream) {
  TraceRange trace_("spear_linear_forward");
  g_last_error.clear();
  return forward_impl(layer, x, M, y, ws, ws_bytes, gate_out, mask_count, SPEAR_PATH_AUTO, stream);
}

int spear_linear_forward_path(const spear_layer* layer, const uint16_t* x, int M, uint16_t* y, void* ws,
                              size_t ws_bytes, float* gate_out, int* mask_count, int path, void* stream) {
  TraceRange trace_("spear_linear_forward_path");
  g_last_error.clear();
  return forward_impl(layer, x, M, y, ws, ws_bytes, gate_out, mask_count, path, stream);
}

int spear_read_status(void* ws, int* device_status, void* stream) {
  TraceRange trace_("spear_read_status");
  g_last_error.clear();
  if (!ws || !device_status) return set_error(SPEAR_ERR_INVALID_ARG, "NULL pointer");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return set_cuda_error("stream synchronize", e);
  int v = 0;
  e = cudaMemcpy(&v, ws, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return set_cuda_error("status read", e);
  if (v) {
    const int zero = 0;
    e = cudaMemcpy(ws, &zero, sizeof(int), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return set_cuda_error("status clear", e);
  }
  *device_status = v;
  return SPEAR_OK;
}

int spear_dispatch_choice(const spear_layer* layer, int M) {
  LayerView L;
  if (check_layer(layer, &L) != SPEAR_OK || M < 1) return SPEAR_PATH_AUTO;
  return choose_path(L, M);
}

int spear_dispatch_set(int K, int N, int r, int group, int M, int path) {
  g_last_error.clear();
  if (path < SPEAR_PATH_DECODE || path > SPEAR_PATH_SEMIFUSED) return set_error(SPEAR_ERR_INVALID_ARG, "bad path");
  if (M < 1) return set_error(SPEAR_ERR_INVALID_ARG, "bad M");
  if (path == SPEAR_PATH_DECODE && M > 16) return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "decode path needs M <= 16");
  std::lock_guard<std::mutex> lk(g_dmu);
  g_table[DKey(K, N, r, group, 0, 0, m_bucket(M))] = DEntry{path, -1.f};
  return SPEAR_OK;
}

int spear_dispatch_set_layer(const spear_layer* layer, int M, int path, float us) {
  g_last_error.clear();
  LayerView L;
  int rc = check_layer(layer, &L);
  if (rc) return rc;
  if (path < SPEAR_PATH_DECODE || path > SPEAR_PATH_SEMIFUSED) return set_error(SPEAR_ERR_INVALID_ARG, "bad path");
  if (M < 1) return set_error(SPEAR_ERR_INVALID_ARG, "bad M");
  if (path == SPEAR_PATH_DECODE && M > 16) return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "decode path needs M <= 16");
  std::lock_guard<std::mutex> lk(g_dmu);
  g_table[dkey(L, M)] = DEntry{path, us >= 0.f ? us : -1.f};
  return SPEAR_OK;
}

int spear_dispatch_set_time(int K, int N, int r, int group, int M, int path, float us) {
  g_last_error.clear();
  if (!(us >= 0.f)) return set_error(SPEAR_ERR_INVALID_ARG, "time must be >= 0 us");
  const int rc = spear_dispatch_set(K, N, r, group, M, path);
  if (rc) return rc;
  std::lock_guard<std::mutex> lk(g_dmu);
  g_table[DKey(K, N, r, group, 0, 0, m_bucket(M))].us = us;
  return SPEAR_OK;
}

int spear_dispatch_time_us(const spear_layer* layer, int M, float* us) {
  g_last_error.clear();
  LayerView L;
  int rc = check_layer(layer, &L);
  if (rc) return rc;
  if (M < 1 || !us) return set_error(SPEAR_ERR_INVALID_ARG, "bad M or NULL output");
  std::lock_guard<std::mutex> lk(g_dmu);
  auto it = g_table.find(dkey(L, M));
  if (it == g_table.end() || it->second.us < 0.f)
    return set_error(SPEAR_ERR_INVALID_ARG, "no measured time for K=%d N=%d r=%d group=%d gate=%d at M bucket %d",
                     L.K, L.N, L.r, L.group, L.r > 0 ? L.gate_kind : 0, m_bucket(M));
  *us = it->second.us;
  return SPEAR_OK;
}

// SLO-constrained chunk size (SPEAR, gist.science technical summary, section
// 2.2 C: the scheduler picks the largest prefill chunk that meets the
// inter-token latency SLO, from precomputed kernel latency tables).  A step
// runs decode_tokens + chunk tokens through every layer; its predicted time is
// step_overhead_us plus the table time of each layer at the step's M bucket
// (the bucket rounds M up, so the prediction is the bucket's measured time).
int spear_slo_chunk(const spear_layer* const* layers, int n_layers, int decode_tokens, float slo_us,
                    float step_overhead_us, const int* chunks, int n_chunks, int* chunk_out, float* predicted_us) {
  g_last_error.clear();
  if (!layers || n_layers <= 0 || !chunks || n_chunks <= 0 || !chunk_out)
    return set_error(SPEAR_ERR_INVALID_ARG, "NULL or empty argument");
  if (decode_tokens < 0 || !(slo_us > 0.f) || !(step_overhead_us >= 0.f))
    return set_error(SPEAR_ERR_INVALID_ARG, "bad decode_tokens, SLO or overhead");
  std::vector<LayerView> Ls(n_layers);
  for (int l = 0; l < n_layers; ++l) {
    int rc = check_layer(layers[l], &Ls[l]);
    if (rc) return rc;
  }
  int best = 0;
  float best_t = -1.f;
  std::lock_guard<std::mutex> lk(g_dmu);
  for (int c = 0; c < n_chunks; ++c) {
    const int chunk = chunks[c];
    if (chunk < 0) return set_error(SPEAR_ERR_INVALID_ARG, "negative chunk size");
    const int M = decode_tokens + chunk;
    if (M < 1) continue;
    float t = step_overhead_us;
    for (int l = 0; l < n_layers; ++l) {
      const LayerView& L = Ls[l];
      auto it = g_table.find(dkey(L, M));
      if (it == g_table.end() || it->second.us < 0.f)
        return set_error(SPEAR_ERR_INVALID_ARG,
                         "layer %d (K=%d N=%d r=%d group=%d gate=%d) has no measured time at M bucket %d", l, L.K,
                         L.N, L.r, L.group, L.r > 0 ? L.gate_kind : 0, m_bucket(M));
      t += it->second.us;
    }
    if (t <= slo_us && chunk >= best) {
      if (chunk > best || best_t < 0.f) best_t = t;
      best = chunk;
    }
  }
  *chunk_out = best;
  if (predicted_us) *predicted_us = best_t;
  return SPEAR_OK;
}

void spear_dispatch_clear(void) {
  std::lock_guard<std::mutex> lk(g_dmu);
  g_table.clear();
}

int spear_dispatch_save(const char* path) {
  g_last_error.clear();
  if (!path) return set_error(SPEAR_ERR_INVALID_ARG, "NULL path");
  int sms = 0;
  const std::string dev = device_ident(&sms);
  FILE* f = fopen(path, "w");
  if (!f) return set_error(SPEAR_ERR_INVALID_ARG, "cannot open %s for writing", path);
  std::lock_guard<std::mutex> lk(g_dmu);
  fprintf(f, "# spear dispatch table v3 sms=%d device=%s\n", sms, dev.c_str());
  fprintf(f, "# K N r group gate_kind gate_hidden M_bucket path time_us (-1 = not measured)\n");
  for (const auto& kv : g_table)
    fprintf(f, "%d %d %d %d %d %d %d %d %.3f\n", std::get<0>(kv.first), std::get<1>(kv.first),
            std::get<2>(kv.first), std::get<3>(kv.first), std::get<4>(kv.first), std::get<5>(kv.first),
            std::get<6>(kv.first), kv.second.path, kv.second.us);
  fclose(f);
  return SPEAR_OK;
}

int spear_dispatch_load(const char* path) {
  g_last_error.clear();
  if (!path) return set_error(SPEAR_ERR_INVALID_ARG, "NULL path");
  FILE* f = fopen(path, "r");
  if (!f) return set_error(SPEAR_ERR_INVALID_ARG, "cannot open %s", path);
  std::map<DKey, DEntry> t;
  char line[512];
  int lineno = 0;
  bool v3 = false;
  while (fgets(line, sizeof(line), f)) {
    ++lineno;
    int fsms = 0;
    char fdev[400];
    if (sscanf(line, "# spear dispatch table v3 sms=%d device=%399[^\n]", &fsms, fdev) == 2) {
      // a table measured on another device (name or multiprocessor count) is refused
      int sms = 0;
      const std::string dev = device_ident(&sms);
      if (fsms != sms || dev != fdev) {
        fclose(f);
        return set_error(SPEAR_ERR_INVALID_ARG, "%s: table measured on \"%s\" (%d SMs), this device is \"%s\" (%d SMs)",
                         path, fdev, fsms, dev.c_str(), sms);
      }
      v3 = true;
      continue;
    }
    if (line[0] == '#' || line[0] == '\n') continue;
    int v[8];
    float us = -1.f;
    DKey key;
    int p = -1;
    if (v3) {
      // K N r group gate_kind gate_hidden M_bucket path [time_us]
      const int n = sscanf(line, "%d %d %d %d %d %d %d %d %f", &v[0], &v[1], &v[2], &v[3], &v[4], &v[5], &v[6],
                           &v[7], &us);
      if ((n == 8 || n == 9) && v[6] >= 1 && (v[4] == 0 || v[4] == 1)) {
        key = DKey(v[0], v[1], v[2], v[3], v[4], v[5], v[6]);
        p = v[7];
        if (n == 8) us = -1.f;
      }
    } else {
      // a table without a device line (the earlier format): scalar-gate
      // entries "K N r group M_bucket path [time_us]"
      const int n = sscanf(line, "%d %d %d %d %d %d %f", &v[0], &v[1], &v[2], &v[3], &v[4], &v[5], &us);
      if ((n == 6 || n == 7) && v[4] >= 1) {
        key = DKey(v[0], v[1], v[2], v[3], 0, 0, v[4]);
        p = v[5];
        if (n == 6) us = -1.f;
      }
    }
    if (p < SPEAR_PATH_DECODE || p > SPEAR_PATH_SEMIFUSED) {
      fclose(f);
      return set_error(SPEAR_ERR_INVALID_ARG, "%s:%d: malformed entry", path, lineno);
    }
    t[key] = DEntry{p, us};
  }
  fclose(f);
  std::lock_guard<std::mutex> lk(g_dmu);
  for (const auto& kv : t) g_table[kv.first] = kv.second;
  return SPEAR_OK;
}

int spear_dispatch_tune(const spear_layer* layer, const int* Ms, int nM, const uint16_t* x, uint16_t* y, void* ws,
                        size_t ws_bytes, void* flush, size_t flush_bytes, int reps, float* times_us, void* stream) {
  TraceRange trace_("spear_dispatch_tune");
  g_last_error.clear();
  LayerView L;
  int rc = check_layer(layer, &L);
  if (rc) return rc;
  if (!Ms || nM <= 0 || !x || !y || !ws) return set_error(SPEAR_ERR_INVALID_ARG, "NULL argument");
  if (reps < 1) reps = 1;
  int M_max = 0;
  for (int i = 0; i < nM; ++i) {
    if (Ms[i] < 1 || Ms[i] > 65536) return set_error(SPEAR_ERR_UNSUPPORTED_SHAPE, "bad M %d", Ms[i]);
    M_max = std::max(M_max, Ms[i]);
  }
  const WsLayout wl = ws_layout(L, M_max);
  if (ws_bytes < wl.total) return set_error(SPEAR_ERR_WORKSPACE, "workspace too small for M_max=%d", M_max);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaEvent_t e0, e1;
  if (cudaEventCreate(&e0) != cudaSuccess || cudaEventCreate(&e1) != cudaSuccess)
    return set_error(SPEAR_ERR_CUDA, "event create failed");
  int result = SPEAR_OK;
  for (int i = 0; i < nM && result == SPEAR_OK; ++i) {
    const int M = Ms[i];
    float best = 1e30f;
    int best_path = default_path(L, M);
    const int paths[4] = {SPEAR_PATH_DECODE, SPEAR_PATH_FUSED, SPEAR_PATH_UNFUSED, SPEAR_PATH_SEMIFUSED};
    for (int pi = 0; pi < 4; ++pi) {
      const int path = paths[pi];
      float med = -1.f;
      if (!(path == SPEAR_PATH_DECODE && M > 16)) {
        std::vector<float> ts;
        int prc = SPEAR_OK;
        for (int rep = 0; rep < reps + 2 && prc == SPEAR_OK; ++rep) {
          if (flush && flush_bytes) cudaMemsetAsync(flush, rep & 0xff, flush_bytes, st);
          cudaEventRecord(e0, st);
          prc = run_path(L, reinterpret_cast<const __nv_bfloat16*>(x), M, reinterpret_cast<__nv_bfloat16*>(y),
                         static_cast<uint8_t*>(ws), wl, nullptr, nullptr, path, st);
          cudaEventRecord(e1, st);
          if (prc == SPEAR_OK) {
            cudaError_t ce = cudaEventSynchronize(e1);
            if (ce != cudaSuccess) {
              result = set_cuda_error("tune", ce);
              break;
            }
            float ms = 0.f;
            cudaEventElapsedTime(&ms, e0, e1);
            if (rep >= 2) ts.push_back(ms * 1000.f);
          }
        }
        if (result) break;
        if (prc == SPEAR_OK && !ts.empty()) {
          std::sort(ts.begin(), ts.end());
          med = ts[ts.size() / 2];
          if (med < best) {
            best = med;
            best_path = path;
          }
        } else {
          g_last_error.clear();
        }
      }
      if (times_us) times_us[i * 4 + pi] = med;
    }
    if (result == SPEAR_OK) {
      std::lock_guard<std::mutex> lk(g_dmu);
      g_table[dkey(L, M)] = DEntry{best_path, best < 1e29f ? best : -1.f};
    }
  }
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  return result;
}

}  // extern "C"
