/*
 * spear.h -- C ABI of the B200 (sm_100a) W4A16 linear layer with a
 * per-token-gated low-rank Error Compensator (EC).
 *
 * The operation (SPEAR, gist.science technical summary, section 2.1 A
 * "Compensateurs d'erreurs adaptatifs a l'entree": an EC projects the input
 * into a low-rank space with A, gates it per token and projects back with B,
 * on top of the 4-bit weight; fugumt.com abstract of arXiv 2606.11244: ECs
 * "modulated by per-token gates" over W4 per-channel weights), in the
 * row-vector form implemented here, with a scalar gate per token by default:
 *
 *     g_m = sigmoid(x_m . w_g + b_g)
 *     y_m = x_m . dequant(W4) + g_m * ((x_m . A) . B)
 *
 * or, per layer, the pages' per-rank gate gamma(x_m . A) (spear_layer's
 * gate_kind, below).
 *
 *   x    M x K   bf16, row-major (token-major)
 *   W    K x N   logically; stored as N output channels x K int4 codes
 *   A    K x r   bf16,  B  r x N  bf16,  w_g  K  bf16,  b_g  float
 *   y    M x N   bf16, row-major
 *
 * Conventions for every call below:
 *   - bf16 and fp16 tensors are passed as uint16_t bit patterns.
 *   - "device" pointers must point to CUDA device memory of the current
 *     device; "host" pointers to ordinary host memory.  Device pointers must be
 *     16-byte aligned (SPEAR_ERR_ALIGNMENT otherwise).
 *   - stream is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls that launch work are asynchronous on that stream and return after
 *     enqueueing.
 *   - The caller owns every buffer.  No call allocates device memory.
 *   - Arguments are validated before anything is enqueued; on error nothing
 *     is launched and the call returns a nonzero SPEAR_* status, with a
 *     message available from spear_last_error() (per host thread).  No call
 *     aborts or exits the process.
 *   - Shapes: K and N multiples of 128; r in {0, 16, 32, 64, 128}; group 0
 *     (one fp16 scale per output channel) or 128 (one fp16 scale per 128
 *     consecutive k and output channel); 1 <= M <= 65536.  The tensor-core
 *     paths also need N % 256 == 0 and the decode path (M <= 16) K % 128 == 0
 *     (SPEAR_ERR_UNSUPPORTED_SHAPE otherwise).
 */
#ifndef SPEAR_H_
#define SPEAR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------- */
enum {
  SPEAR_OK = 0,
  SPEAR_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad enum   */
  SPEAR_ERR_UNSUPPORTED_SHAPE = 2, /* K/N/r/group/M outside the list above    */
  SPEAR_ERR_ALIGNMENT = 3,         /* a device pointer is not 16-byte aligned */
  SPEAR_ERR_WORKSPACE = 4,         /* workspace smaller than required          */
  SPEAR_ERR_CUDA = 5,              /* a CUDA runtime call or launch failed     */
  SPEAR_ERR_TIMEOUT = 6,           /* a device-side bounded wait expired       */
  SPEAR_ERR_DEVICE_CHECK = 7       /* a device-side argument check failed      */
};

/* Kernel paths (for spear_linear_forward_path and the dispatcher). */
enum {
  SPEAR_PATH_AUTO = 0,    /* dispatcher's choice                                   */
  SPEAR_PATH_DECODE = 1,  /* split-K GEMV kernel with the EC fused (M <= 16)       */
  SPEAR_PATH_FUSED = 2,   /* tcgen05 GEMM with the EC fused into the same kernel   */
  SPEAR_PATH_UNFUSED = 3, /* GEMM with the EC disabled, then a separate EC kernel  */
  SPEAR_PATH_SEMIFUSED = 4 /* SPEAR's prefill DAG (gist.science technical summary,
                            * section 2.2 A): the EC projection (g, g*t) on a
                            * second, high-priority stream concurrently with the
                            * EC-disabled GEMM on `stream`, then the in-place
                            * update g*(t.B) after both.  The fork and join are
                            * CUDA events, so capturing `stream` into a CUDA
                            * graph captures the two-branch DAG.  One side stream
                            * per device, shared by all callers: host enqueue of
                            * this path is serialised by a mutex. */
};

/* Message of the last failing call on this host thread ("" if none). */
const char* spear_last_error(void);
/* Static name of a status code. */
const char* spear_status_string(int status);
/* Library version, major*10000 + minor*100 + patch. */
int spear_version(void);

/* ---- sizes ---------------------------------------------------------------- */
/* Bytes of a packed N x K int4 weight: N*K/2 (0 on a bad shape). */
size_t spear_w4_packed_bytes(int N, int K);
/* Number of fp16 scales: N (group 0) or (K/128)*N (group 128); 0 on a bad shape. */
size_t spear_scale_count(int N, int K, int group);

/* ---- a-0: quantiser --------------------------------------------------------
 * Symmetric round-to-nearest int4 (SPEAR evaluates RTN per-channel W4
 * weights, gist.science technical summary, section 3.1).  For every output
 * channel n (and, for group 128, every block of 128 consecutive k):
 *     s = fp16_rne(max|w| / 7)   (fp32 arithmetic; saturated to 65504;
 *                                 s == 0 becomes 1.0 with all codes 0)
 *     q = clamp(rint_even(w / s), -7, 7)   (IEEE fp32 quotient)
 * W       device fp32, K x N row-major (W[k*N + n]).
 * q       device int8, N x K row-major (q[n*K + k]), written.
 * scales  device fp16 bits, [N] or [K/128][N], written.
 * Bit-exact and deterministic. */
int spear_w4_quantize(const float* W, int K, int N, int group, int8_t* q,
                      uint16_t* scales, void* stream);

/* ---- a-1: packed int4 weight layout -----------------------------------------
 * Packed int4 weight layout (the pages give none; this one is built so that
 * one 128-bit load per lane yields whole tensor-core operand fragments and a
 * 16-row x 64-k tile is one contiguous, 16-byte aligned 512-byte block):
 *   tile (p, t), p = n / 16, t = k / 64, occupies bytes
 *       [(p * (K/64) + t) * 512, +512);
 *   inside a tile, lane L = 0..31 owns bytes [16L, 16L+16) as four
 *   little-endian uint32 words w_s (s = 0..3) at byte 16L + 4s;
 *   with rho = L / 4 and c = L % 4, nibble slot i = 0..7 of w_s (bits
 *   4i..4i+3) holds the code of
 *       n = 16p + rho + 8*(i & 1)
 *       k = 64t + 16c + 4s + 2*((i & 3) >> 1) + (i >> 2)
 *   stored offset-binary: u = q + 8 (0..15).
 * Requires N % 16 == 0 and K % 64 == 0 (the layer calls need multiples of 128).
 * q       device int8 N x K (codes in [-8, 7]; other values are masked to 4 bits)
 * packed  device uint8 [N*K/2], written.  Bit-exact. */
int spear_w4_pack(const int8_t* q, int N, int K, uint8_t* packed, void* stream);
/* Inverse of spear_w4_pack: packed -> q (N x K int8 in [-8, 7]).  Bit-exact. */
int spear_w4_unpack(const uint8_t* packed, int N, int K, int8_t* q, void* stream);

/* ---- EC operands -------------------------------------------------------------
 * Per-channel fold: B'[j][n] = bf16_rne(fp32(B[j][n] / s[n])), so that a
 * kernel accumulates x.q and (g t).B' in one fp32 accumulator and applies s_n
 * once.  B, Bp: device bf16 r x N row-major; scales: device fp16 [N].
 * Bit-exact. */
int spear_ec_prescale_B(const uint16_t* B, const uint16_t* scales, int r, int N,
                        uint16_t* Bp, void* stream);

/* Elements of the two EC operand arrays: AgT (r+1) x K and BpT N x r. */
size_t spear_ec_agt_count(int K, int r);
size_t spear_ec_bpt_count(int N, int r);

/* EC operands in the kernels' layout (one-off per layer):
 *   AgT = [A^T ; w_g]          (r+1) x K bf16 row-major: the r projection rows
 *                               and the gate weight as one extra row;
 *   BpT = (B')^T (group 0) or B^T (group 128), N x r bf16 row-major.
 * A: device bf16 K x r; B: device bf16 r x N; w_g: device bf16 [K];
 * scales: the layer's fp16 scales (read only for group 0).  Bit-exact. */
int spear_ec_pack(const uint16_t* A, const uint16_t* B, const uint16_t* w_g,
                  const uint16_t* scales, int K, int N, int r, int group,
                  uint16_t* AgT, uint16_t* BpT, void* stream);

/* ---- the layer ----------------------------------------------------------------- */
typedef struct spear_layer {
  int K;                   /* input features  (multiple of 128)                  */
  int N;                   /* output features (multiple of 128)                  */
  int group;               /* 0 = per-channel scales, 128 = group-wise scales    */
  int r;                   /* EC rank; 0 disables the EC                         */
  const uint8_t* w_packed; /* device, spear_w4_pack layout, N*K/2 bytes           */
  const uint16_t* scales;  /* device fp16, spear_scale_count(N, K, group) values  */
  const uint16_t* AgT;     /* device bf16 (r+1) x K from spear_ec_pack (r > 0)    */
  const uint16_t* BpT;     /* device bf16 N x r from spear_ec_pack (r > 0)        */
  float b_g;               /* gate bias (scalar gate)                             */
  float gate_tau;          /* threshold of the gate-mask count; <= 0 means 0.1    */
  /* Gate form.  A zero-initialised tail keeps the scalar gate.
   * SPEAR_GATE_RANK_MLP is the pages' form (gist.science technical summary,
   * section 2.1 A: effective weight W + alpha B diag(gamma(A x)) A, gamma a
   * bottleneck MLP on the low-rank projection):
   *   t = x . A,  u = relu(W1 t + b1),  gamma = sigmoid(W2 u + b2),
   *   y = x . dequant(W4) + alpha * (t * gamma) . B,
   * with gt = bf16(alpha * gamma * t) feeding the up-projection.  The row of
   * w_g in AgT is then unused (pack it with w_g = 0); b_g is ignored.  The
   * per-token gate reported by gate_out (and compared with gate_tau) is the
   * mean of gamma over the r ranks.  Paths: the decode kernel (not its
   * fallback for K % 256 != 0 or very long K), the tensor-core kernel, and
   * the unfused / semi-fused EC kernel. */
  int gate_kind;           /* SPEAR_GATE_SCALAR (0) or SPEAR_GATE_RANK_MLP (1)    */
  int gate_hidden;         /* h, the bottleneck width of the rank gate: 8, 16, 32 */
  const float* gate_w1;    /* device fp32 h x r row-major (16-byte aligned)       */
  const float* gate_b1;    /* device fp32 [h]                                     */
  const float* gate_w2;    /* device fp32 r x h row-major                         */
  const float* gate_b2;    /* device fp32 [r]                                     */
  float gate_alpha;        /* alpha of the rank gate                              */
  /* Optional hint for calls that run layers back to back (a decoder's token
   * step): the layer the NEXT call on this stream will run, or NULL.  While
   * this call's decode-path kernel runs, it warms L2 with that layer's packed
   * weights and EC operands, so the next call's weight loads hit L2 while
   * DRAM keeps streaming.  A hint only: results are bitwise unchanged, and in
   * a chain of hinted calls every byte still leaves DRAM once per call.
   * Read during this call only (its own prefetch_next is ignored); its device
   * buffers must stay allocated until the next call has run.  The earlier
   * decode kernels (long or ragged K) and the tensor-core paths ignore it. */
  const struct spear_layer* prefetch_next;
} spear_layer;

enum { SPEAR_GATE_SCALAR = 0, SPEAR_GATE_RANK_MLP = 1 };

/* Workspace bytes needed by spear_linear_forward* for any 1 <= M <= M_max
 * (0 on invalid arguments).  The workspace holds split-K partials, the EC
 * projection, arrival counters and a device status word. */
size_t spear_workspace_bytes(const spear_layer* layer, int M_max);

/* Put a freshly allocated workspace into its initial state (zeroes it on
 * stream).  Needed once after allocation and after any SPEAR_ERR_TIMEOUT;
 * the kernels leave it in that state after every successful call. */
int spear_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* y = layer(x) (see the top of this file).
 * x          device bf16 M x K;  y  device bf16 M x N, written.
 * ws         device workspace of ws_bytes >= spear_workspace_bytes(layer, M),
 *            initialised once by spear_workspace_init.  A workspace must not
 *            be used by two calls that may run concurrently.
 * gate_out   optional (NULL): device fp32 [M], receives g_m (0 when r == 0).
 * mask_count optional (NULL): device int32, receives #{m : g_m < gate_tau}.
 * The kernel path is chosen by the dispatcher (see spear_dispatch_choice).
 * Device-side failures (a bounded wait that expired) are reported through
 * the workspace's status word, read by spear_read_status. */
int spear_linear_forward(const spear_layer* layer, const uint16_t* x, int M,
                         uint16_t* y, void* ws, size_t ws_bytes, float* gate_out,
                         int* mask_count, void* stream);

/* As spear_linear_forward with an explicit SPEAR_PATH_* (tests, tuning). */
int spear_linear_forward_path(const spear_layer* layer, const uint16_t* x, int M,
                              uint16_t* y, void* ws, size_t ws_bytes,
                              float* gate_out, int* mask_count, int path,
                              void* stream);

/* Synchronise stream, read and clear the workspace's device status word.
 * *device_status receives SPEAR_OK or the first device-side error code. */
int spear_read_status(void* ws, int* device_status, void* stream);

/* ---- failure injection (tests of the device-side error path only) -----------
 * Makes one bounded device wait impossible to satisfy in the launches that
 * follow, until called again with kernel 0: the wait expects a publication
 * tag that no launch writes, and gives up after wait_cycles SM clock cycles
 * instead of about a second.
 *   kernel 1: the decode kernel's wait for the published EC rows;
 *   kernel 2: the tensor-core kernel's wait for the gated projection.
 * The launch then reports SPEAR_ERR_TIMEOUT in its status word (workspace, or
 * the allocation-free call's array), every role of the kernel stops at its
 * next check, waits for the copies it has in flight and exits; y is left
 * unspecified.  No fault, trap or unbounded wait is involved.  As after any
 * timeout, re-initialise the workspace (spear_workspace_init) before the next
 * call.  Process-wide, not thread-safe against concurrent layer calls.
 * SPEAR_ERR_INVALID_ARG for another kernel value or wait_cycles < 1. */
int spear_test_inject_timeout(int kernel, long long wait_cycles);

/* ---- device-check build --------------------------------------------------
 * The library can be built a second time with -DSPEAR_DEVICE_CHECKS
 * (libspear_checked.so beside libspear.so): device-side bounds checks on the
 * kernels' output stores (row < M, channels < N) and on their workspace
 * partial slots, flags and published EC rows.  A failed check writes
 * SPEAR_ERR_DEVICE_CHECK to the status word (spear_read_status), skips the
 * access it guards and never traps; y is then unspecified.  In the normal
 * build the checks compile away.
 *
 * spear_device_checks_enabled: 1 in the device-check build, 0 otherwise.
 *
 * spear_test_force_device_check (test hook): kernel 1 makes the decode
 * kernel's output-store check fail, kernel 2 the tensor-core kernel's, in
 * the launches that follow until called with 0 (process-wide).  The
 * guarded stores are skipped, so no out-of-range access is ever made; the
 * launch reports SPEAR_ERR_DEVICE_CHECK.  No effect in the normal build.
 * SPEAR_ERR_INVALID_ARG for another kernel value. */
int spear_device_checks_enabled(void);

/* ---- tracing ---------------------------------------------------------------
 * NVTX ranges named for the call around the layer calls, the preparation
 * calls, the workspace and status calls and the dispatcher's tuning, for a
 * profiler's timeline (ncu --nvtx, or any NVTX tool).  Off by default; on
 * when the environment holds SPEAR_NVTX=1 at the first call, or after
 * spear_set_tracing(1).  With no tool attached a range costs a branch.
 * spear_set_tracing: on != 0 turns it on, 0 off (process-wide); SPEAR_OK.
 * spear_tracing_enabled: 1 when on. */
int spear_set_tracing(int on);
int spear_tracing_enabled(void);
int spear_test_force_device_check(int kernel);

/* ---- allocation-free decode call ---------------------------------------------
 * Not part of the method on the pages (they have no counterpart): an
 * interface for callers that cannot allocate device memory where they run
 * the layer -- code executing while another component owns the CUDA
 * allocator (a serving engine's memory pool), token loops in which an
 * allocation would synchronise the device, or plugin hosts that pass only
 * input and output buffers.
 * Same result as spear_linear_forward_path(..., SPEAR_PATH_DECODE, ...), but
 * the scratch lives in a 40 KB device array inside the library instead of a
 * caller workspace.  Limit: 1 <= M <= 16 (larger M returns
 * SPEAR_ERR_UNSUPPORTED_SHAPE); every layer shape of the decode path.
 * x, y: 16-byte aligned; gate_out, mask_count: 4-byte aligned (or NULL).
 * No device memory is allocated or freed.  Every call looks up the array's
 * device address (cudaGetSymbolAddress) on the current device; the first
 * lookup on a device may load the library's device code, so make the first
 * call on each device before any stream capture.  Each call clears the
 * array's launch header on `stream` before its kernel.  The array is shared
 * by all calls on a device: calls whose executions may overlap on the GPU
 * (other streams, unordered host threads) race and must not be issued.
 * Device-side failures (a bounded wait that expired) go to the array's own
 * status word, which later calls do not clear: read it with
 * spear_read_status_noalloc. */
int spear_linear_forward_decode_noalloc(const spear_layer* layer, const uint16_t* x, int M,
                                        uint16_t* y, float* gate_out, int* mask_count,
                                        void* stream);

/* Synchronise stream, then read and clear the status word of the
 * allocation-free call's array on the current device.  *device_status
 * receives SPEAR_OK or the first device-side error code recorded since the
 * last read. */
int spear_read_status_noalloc(int* device_status, void* stream);

/* ---- a-7: dispatcher ----------------------------------------------------------
 * Phase-aware choice between the fused and the unfused EC path (SPEAR,
 * gist.science technical summary, section 2.2 A "Dispatch de fusion de noyau
 * adaptatif sensible a la phase": decode fuses the EC into the low-bit GEMM,
 * prefill runs it as a separate kernel; the choice here comes from measured
 * kernel times, the pages' latency tables of section 2.2 C).
 * The table is keyed by (K, N, r, group, gate form, bottleneck width, M
 * bucket); M buckets are powers of two (M rounded up).  Before tuning: DECODE
 * for M <= 16, else FUSED. */
int spear_dispatch_choice(const spear_layer* layer, int M);

/* Time every applicable path for each M in Ms[0..nM) with CUDA events
 * (median of `reps` runs, each preceded by writing flush_bytes of the
 * optional device buffer `flush` to evict L2) and record the fastest in the
 * table.  x: device bf16 M_max x K input, y: device bf16 M_max x N scratch
 * output (M_max = max of Ms).  times_us (optional host array [nM*4]) receives
 * the median of each path (DECODE, FUSED, UNFUSED, SEMIFUSED; negative = not
 * run).
 * Synchronises the stream. */
int spear_dispatch_tune(const spear_layer* layer, const int* Ms, int nM,
                        const uint16_t* x, uint16_t* y, void* ws, size_t ws_bytes,
                        void* flush, size_t flush_bytes, int reps, float* times_us,
                        void* stream);

/* Set one table entry by hand (path is a SPEAR_PATH_* other than AUTO), for
 * a layer with the scalar gate (or without an EC). */
int spear_dispatch_set(int K, int N, int r, int group, int M, int path);
/* Set the entry of this layer's full key -- shape, scale kind and gate form
 * (a rank-gate layer has entries of its own, per bottleneck width) -- at M's
 * bucket, with its measured time in microseconds (us < 0: not measured). */
int spear_dispatch_set_layer(const spear_layer* layer, int M, int path, float us);
/* Set one table entry with its measured time in microseconds (us >= 0).
 * Entries made by spear_dispatch_set carry no time; spear_dispatch_tune
 * records the median of the path it picks. */
int spear_dispatch_set_time(int K, int N, int r, int group, int M, int path, float us);
/* Measured time (microseconds) of the table's path for this layer at M's
 * bucket.  SPEAR_ERR_INVALID_ARG if that entry has no time. */
int spear_dispatch_time_us(const spear_layer* layer, int M, float* us);
/* Forget every table entry. */
void spear_dispatch_clear(void);
/* Save / load the table as text (host file path).  The first line names the
 * device the times were measured on ("# spear dispatch table v3 sms=<count>
 * device=<name>"); loading a table made on another device (name or SM count)
 * fails with SPEAR_ERR_INVALID_ARG and leaves the table unchanged.  Entry
 * lines are "K N r group gate_kind gate_hidden M_bucket path time_us"
 * (time -1 or absent: not measured).  A file without the device line is read
 * in the earlier format, "K N r group M_bucket path [time_us]", as
 * scalar-gate entries. */
int spear_dispatch_save(const char* path);
int spear_dispatch_load(const char* path);

/* ---- SLO-constrained prefill chunk size --------------------------------------
 * SPEAR, gist.science technical summary, section 2.2 C ("Ordonnancement par
 * blocs conscient de l'EC et contraint par les SLO"): pick the largest prefill
 * chunk whose predicted step time meets the inter-token latency SLO, from the
 * precomputed kernel latency table.
 * A step pushes decode_tokens + chunk tokens through each of layers[0..n_layers)
 * (host array of layer pointers, EC on some of them or not).  Its predicted
 * time is step_overhead_us plus, per layer, the table's measured time at the
 * step's M bucket.  Candidates are chunks[0..n_chunks) (>= 0, any order).
 * On success *chunk_out is the largest candidate whose prediction is
 * <= slo_us (0 if none is), and *predicted_us (optional) its prediction (-1
 * if none).  SPEAR_ERR_INVALID_ARG if a needed table entry has no measured
 * time (tune those M buckets first).  Host only; no GPU work. */
int spear_slo_chunk(const spear_layer* const* layers, int n_layers, int decode_tokens, float slo_us,
                    float step_overhead_us, const int* chunks, int n_chunks, int* chunk_out,
                    float* predicted_us);

#ifdef __cplusplus
}
#endif

#endif /* SPEAR_H_ */
