/*
 * gdn.h -- C ABI of libgdn.so: the gated delta rule (chunked forward) and the
 * Gated Delta Product one-token decode step on NVIDIA B200 (sm_100a).
 *
 * The rule (per sequence, per head; S is V x K, the library stores h = S^T,
 * K x V, key-major):
 *     S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *     o_t = scale * S_t q_t
 * Chunked evaluation (64-token chunks, intra-chunk WY form, inter-chunk state
 * recurrence, chunk output) follows the three GDN kernels of ZzCompute,
 * PyTorch Helion Hackathon gallery entry 11, items 2-4 ("Chunk Forward H",
 * "Chunk Forward O", "Recompute W/U").  Gates and the decode layout follow
 * NVIDIA Megatron-Core "core.ssm.ops.gdp.decode_prepare".
 *
 * Conventions for every entry point:
 *  - All tensor arguments are DEVICE pointers to memory the caller owns.  The
 *    library never allocates, never frees, never synchronises the host with
 *    the device (except gdn_device_status, which says so) and keeps no state
 *    between calls apart from the device status word.
 *  - `stream` is a cudaStream_t passed as void*; NULL is the legacy default
 *    stream.  Work is enqueued on it and the call returns; results are ready
 *    when the stream reaches that point.  No call reads device memory on the
 *    host, so every call may be captured in a CUDA graph.
 *  - Arguments are checked on the host before anything is launched; a bad
 *    argument returns GDN_ERR_INVALID_ARG and launches nothing.  A failed
 *    launch returns GDN_ERR_CUDA (gdn_last_cuda_error gives the cudaError_t).
 *  - Layouts are row-major with the innermost dimension contiguous unless a
 *    stride argument says otherwise.  Every output element is written by
 *    exactly one thread, with no atomics, so results are bitwise reproducible
 *    run to run on the same device.
 *  - Pointers must be 16-byte aligned (256-byte alignment, as from the CUDA
 *    caching allocators, is recommended).
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1, /* rejected on the host; nothing launched            */
    GDN_ERR_UNSUPPORTED = 2, /* well-formed, but this size/dtype is not built     */
    GDN_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed              */
    GDN_ERR_TIMEOUT = 4,     /* a bounded device-side wait gave up (device status) */
    GDN_ERR_TOO_LARGE = 5    /* exceeds the fixed capacity of gdn_chunk_fwd_noalloc  */
} gdn_status;

typedef enum { GDN_F32 = 0, GDN_BF16 = 1 } gdn_dtype;

/* gdn_chunk_fwd flags (bit set). */
#define GDN_FLAG_EXACT_F32 0x1u    /* use the fp32-FMA kernel even for bf16 q/k/v      */
#define GDN_FLAG_CHUNK32 0x10u     /* fp32-FMA kernel only: 32-token chunks           */
#define GDN_FLAG_CHUNK16 0x20u     /* fp32-FMA kernel only: 16-token chunks           */
#define GDN_FLAG_VSPLIT1 0x100u    /* force one V-slice per (sequence, head)          */
#define GDN_FLAG_VSPLIT2 0x200u    /* force two V-slices                              */
#define GDN_FLAG_VSPLIT4 0x400u    /* force four V-slices                             */

/* Human-readable name of a status code (static string, never NULL). */
const char* gdn_status_string(int status);

/* cudaError_t of the most recent GDN_ERR_CUDA on the calling thread (0 if none). */
int gdn_last_cuda_error(void);

/* Library version as 10000*major + 100*minor + patch. */
int gdn_version(void);

/*
 * gdn_gate_prep -- per-token, per-head gates.
 *   beta = sigmoid(b)
 *   g    = -exp(A_log) * softplus(a + dt_bias),
 *   softplus(x) = log1p(exp(x)), and x itself when x > 20 (strict).
 * Megatron-Core "core.ssm.ops.gdp.decode_prepare", module description and the
 * `softplus` entry (torch's F.softplus at beta = 1, threshold 20; log1p keeps
 * the far-negative tail).  a + dt_bias is one fp32 add; the transcendentals
 * run in fp64 and each output is rounded to fp32 once (no flush to zero).
 *
 *   a, b      : fp32 [n_tok, H], token stride a_stride / b_stride elements
 *               (>= H), head stride 1.
 *   A_log     : fp32 [H].   dt_bias : fp32 [H].
 *   beta, g   : fp32 [n_tok, H] contiguous, written.
 * n_tok == 0 is a no-op.  Errors: INVALID_ARG for NULL pointers, H < 1,
 * n_tok < 0 or a stride < H.
 */
gdn_status gdn_gate_prep(const float* a, const float* b, int64_t n_tok, int H, int64_t a_stride,
                         int64_t b_stride, const float* A_log, const float* dt_bias, float* beta,
                         float* g, void* stream);

/*
 * gdn_chunk_fwd_workspace_size -- bytes of device workspace for gdn_chunk_fwd
 * with these sizes.  The caller allocates it.  It holds the packed-batch
 * schedule (int32 per sequence) and, for bf16 q/k/v with K = V = 128, one
 * 33,296-byte WY image per (chunk, head) plus a 4-byte ready flag each
 * ((ceil(T_total / 64) + n_seq) * H of them): with that room a dense batch
 * runs the tensor-core kernel as one persistent cooperative launch, the prep
 * on every SM not carrying a chain (see gdn_chunk_fwd).  0 when n_seq <= 0.
 */
size_t gdn_chunk_fwd_workspace_size(int n_seq, int64_t T_total, int H, int K, int V,
                                    gdn_dtype qkv_dtype);

/*
 * gdn_chunk_fwd -- chunked forward pass of the gated delta rule.
 *
 *   q, k    : [B, T, H, K] of qkv_dtype (GDN_F32 or GDN_BF16).
 *   v       : [B, T, H, V] of qkv_dtype.
 *   g, beta : fp32 [B, T, H] (natural-log decay gate, write strength).
 *   h0      : fp32 [n_seq, H, K, V] initial states, or NULL for zeros.
 *   cu_seqlens : NULL for a dense batch (n_seq = B sequences of length T), or
 *             int32 [n_seq + 1] device array of packed-sequence offsets with
 *             cu_seqlens[0] = 0, non-decreasing, cu_seqlens[n_seq] = T; then
 *             B must be 1.  Empty sequences are allowed (their h_T = h0).
 *   scale   : multiplies every output (o_t = scale * S_t q_t).
 *   o       : [B, T, H, V] of o_dtype (GDN_F32 or GDN_BF16), written.
 *   hT      : fp32 [n_seq, H, K, V] final states, written; NULL to skip.
 *   workspace / ws_bytes : device scratch of gdn_chunk_fwd_workspace_size(...)
 *             bytes.  Its contents on entry do not matter.  A packed batch
 *             needs its longest-first schedule (4 * n_seq bytes, rounded up
 *             to 256), a single sequence included; a dense batch needs none
 *             and may pass NULL.  The bf16 K = V = 128 path runs as one
 *             cluster of two CTAs per (sequence, head): the WY prep of every
 *             chunk on one, the inter-chunk recurrence and the output on the
 *             other.
 *   flags   : GDN_FLAG_* bits; 0 selects the fastest kernel for the dtype.
 *             (An addition to the call list the method's API describes, which
 *             has no flags argument: pass 0 for exactly that call.)
 * Supported: K, V in {32, 64, 128}.  bf16 q/k/v run on the tcgen05 tensor-core
 * kernel (bf16 operands, fp32 accumulation and fp32 state) when K = V = 128;
 * otherwise, and for fp32 q/k/v, an fp32-FMA kernel that keeps every product
 * in IEEE fp32.  T == 0 writes only hT (= h0 or zeros).
 * Errors: INVALID_ARG (NULL q/k/v/g/beta/o, sizes < 0, B != 1 with
 * cu_seqlens, workspace too small, misaligned pointer), UNSUPPORTED (other
 * K/V/dtypes).  cu_seqlens contents are not checked on the host (that would
 * need a device read); offsets outside [0, T] are undefined behaviour.
 */
gdn_status gdn_chunk_fwd(const void* q, const void* k, const void* v, gdn_dtype qkv_dtype,
                         const float* g, const float* beta, const float* h0,
                         const int32_t* cu_seqlens, int n_seq, int B, int64_t T, int H, int K,
                         int V, float scale, void* o, gdn_dtype o_dtype, float* hT,
                         void* workspace, size_t ws_bytes, unsigned flags, void* stream);

/*
 * gdp_decode_prepare -- split, GQA-expand, Householder-interleave and gate one
 * decode step.  Megatron-Core `gdp_decode_prepare` (function entry, parameter
 * list and return shapes).
 *
 *   x   : bf16 [n, *] rows, row stride x_n_stride elements, each row
 *         [value: M*H*P | key: M*G*N | query: G*N] (inner dim contiguous).
 *   ba  : bf16 [n, *] rows, row stride ba_n_stride elements, each row
 *         [b: M*H | a: H].
 *   A_log, dt_bias : fp32 [H].
 *   q, k : bf16 [n, M, H, N] written;  v : bf16 [n, M, H, P] written.
 *   beta, g : fp32 [n, M, H] written.
 * Readings where the page is silent: the Householder copy is the outer index
 * inside each part ([M,H,P], [M,G,N], [M,H]); head h uses group h / (H/G);
 * the query sits on copy M-1 (zeros elsewhere); the decay g sits on copy 0
 * (zero elsewhere); beta is per copy.  q/k/v are bit copies of x; beta and g
 * are computed as in gdn_gate_prep from the bf16 inputs widened to fp32.
 * Errors: INVALID_ARG (NULL, n < 0, M < 1, H % G != 0, strides shorter than
 * the row), UNSUPPORTED (P or N not in {32, 64, 128}).
 */
gdn_status gdp_decode_prepare(const void* x, int64_t x_n_stride, const void* ba,
                              int64_t ba_n_stride, const float* A_log, const float* dt_bias, int n,
                              int M, int H, int G, int P, int N, void* q, void* k, void* v,
                              float* beta, float* g, void* stream);

/*
 * gdp_decode_step -- the fused decode step: gdp_decode_prepare's split, GQA
 * expansion and gates in registers, then the rule over the M copies of each
 * request, starting from and overwriting its state:
 *     for m in 0..M-1:  S <- exp(g_m) S;  u = beta_m (v_m - S^T k_m);
 *                       S <- S + k_m u^T
 *     o = scale * S^T q_{M-1}
 * (state layout [n, H, N, P]: key rows, value columns).  With qk_l2norm != 0
 * every q and k vector is divided by sqrt(sum x^2 + 1e-6) first.
 *   state : fp32 [n, H, N, P], read and written in place.
 *   o     : bf16 [n, H, P], written.
 * Other arguments and errors as gdp_decode_prepare.
 */
gdn_status gdp_decode_step(const void* x, int64_t x_n_stride, const void* ba, int64_t ba_n_stride,
                           const float* A_log, const float* dt_bias, int n, int M, int H, int G,
                           int P, int N, float* state, void* o, float scale, int qk_l2norm,
                           void* stream);

/*
 * gdp_decode_step_indexed -- gdp_decode_step on a pool of states.  Request r
 * uses state slot s = state_idx ? state_idx[r] : r of `state`.
 *   state     : fp32 [n_slots, H, N, P], the slots named by state_idx read and
 *               written in place (others untouched); may be NULL when
 *               n_slots == 0 (every request padding).
 *   state_idx : int32 [n] device array, or NULL (then n_slots >= n).  Distinct
 *               requests must name distinct slots (two requests on one slot
 *               race).  No host read: the call stays graph-capturable.
 * A negative slot is a padding request: o[r] = 0 and no state is read or
 * written (Megatron-Core "core.ssm.ops.gdp.decode_prepare", module
 * description: the batch is padded upstream, with -1 slots).  A slot >=
 * n_slots is treated the same way and records GDN_ERR_INVALID_ARG in the
 * device status word (read by gdn_device_status).
 * Other arguments and errors as gdp_decode_step; also INVALID_ARG for
 * n_slots < 0, state_idx == NULL with n_slots < n, a misaligned state_idx.
 */
gdn_status gdp_decode_step_indexed(const void* x, int64_t x_n_stride, const void* ba,
                                   int64_t ba_n_stride, const float* A_log, const float* dt_bias,
                                   int n, int M, int H, int G, int P, int N, float* state,
                                   const int32_t* state_idx, int n_slots, void* o, float scale,
                                   int qk_l2norm, void* stream);

/*
 * gdp_decode_layer_step -- one decode token of a Gated Delta Product layer in
 * one launch: the short-convolution update of the projected row (as
 * gdn_conv1d_update, bf16, over all M*H*P + M*G*N + G*N channels of x), then
 * gdp_decode_step_indexed on the convolved row.  Megatron-Core
 * "core.ssm.ops.gdp.decode_prepare", module description: the short-conv update
 * runs between the projection and the recurrent kernel, and a -1 slot zeroes
 * its conv output (so o = 0 and neither state is touched).  The results equal,
 * bit for bit, gdn_conv1d_update (bf16 output) followed by
 * gdp_decode_step_indexed, without the convolved row going through memory.
 *   x          : bf16 [n, *] rows BEFORE the short convolution, row stride
 *                x_n_stride elements, each [value | key | query] as in
 *                gdp_decode_prepare.  ba, A_log, dt_bias as gdp_decode_step.
 *   conv_w     : fp32 [C, W], C = M*H*P + M*G*N + G*N;  conv_bias fp32 [C] or
 *                NULL;  W in 1..4;  activation 1 = SiLU, 0 = none.
 *   conv_state : bf16 [n_slots, C, W-1], in place (NULL allowed when W == 1).
 *   state, state_idx, n_slots, o, scale, qk_l2norm : as gdp_decode_step_indexed;
 *                one slot index names both the conv window and the state.
 *   workspace  : >= gdp_decode_layer_step_workspace_size(n, G) bytes, 4-byte
 *                aligned, ZERO before the first call (cudaMemset); every call
 *                leaves it zero.  It counts, per (request, group), the blocks
 *                that have read the group's key and query windows, so that the
 *                last of them shifts those windows after all have read them.
 *                Calls sharing one workspace must not run concurrently.
 * Errors: as gdp_decode_step_indexed; INVALID_ARG also for W outside 1..4,
 * activation not 0/1, NULL conv_w (or conv_state with W > 1), a missing or
 * short workspace.
 */
size_t gdp_decode_layer_step_workspace_size(int n, int G);
gdn_status gdp_decode_layer_step(const void* x, int64_t x_n_stride, const void* ba,
                                 int64_t ba_n_stride, const float* conv_w, const float* conv_bias,
                                 int W, void* conv_state, int activation, const float* A_log,
                                 const float* dt_bias, int n, int M, int H, int G, int P, int N,
                                 float* state, const int32_t* state_idx, int n_slots, void* o,
                                 float scale, int qk_l2norm, void* workspace, size_t ws_bytes,
                                 void* stream);

/*
 * gdp_prefill -- the Gated Delta Product over a whole prompt: every token row
 * carries the decode layout (x row [value: M*H*P | key: M*G*N | query: G*N],
 * ba row [b: M*H | a: H], as in gdp_decode_prepare), and the rule runs over the
 * M Householder copies of each token in order -- copy m of token t is step
 * t*M + m of a T*M-step sequence, with the query on copy M-1 and the decay on
 * copy 0 (Megatron-Core "core.ssm.ops.gdp.decode_prepare": module description
 * and the gdp_decode_prepare entry, whose outputs are the layouts the
 * recurrent kernel expects for an M-length sequence per request).  o is taken
 * at each token's last copy.  The result equals T successive gdp_decode_step
 * calls with qk_l2norm = 0 (q and k are used as given), computed with the
 * chunked kernels of gdn_chunk_fwd.
 *   x, ba     : bf16 rows, B*T of them (dense) or T_total (cu_seqlens != NULL,
 *               B == 1), row strides x_n_stride / ba_n_stride elements.
 *   h0        : fp32 [n_seq, H, N, P] or NULL (zero).
 *   cu_seqlens: int32 [n_seq+1] token offsets (device) or NULL.
 *   o         : [rows, H, P] of o_dtype;  hT : fp32 [n_seq, H, N, P] or NULL.
 *   workspace : >= gdp_prefill_workspace_size(n_seq, rows, M, H, P, N, o_dtype,
 *               cu_seqlens != NULL) bytes, 16-byte aligned (it holds the
 *               interleaved q/k/v/gates and the output of every copy).
 * Errors: as gdp_decode_prepare and gdn_chunk_fwd; UNSUPPORTED when rows * M
 * reaches 2^31.
 */
size_t gdp_prefill_workspace_size(int n_seq, int64_t rows, int M, int H, int P, int N,
                                  gdn_dtype o_dtype, int packed);
gdn_status gdp_prefill(const void* x, int64_t x_n_stride, const void* ba, int64_t ba_n_stride,
                       const float* A_log, const float* dt_bias, const float* h0,
                       const int32_t* cu_seqlens, int n_seq, int B, int64_t T, int M, int H,
                       int G, int P, int N, float scale, void* o, gdn_dtype o_dtype, float* hT,
                       void* workspace, size_t ws_bytes, void* stream);

/*
 * gdn_chunk_fwd_noalloc -- gdn_chunk_fwd for callers that cannot allocate
 * device memory.  The sources describe no such entry point; it exists because
 * some callers have no way to provide the packed-batch workspace: code running
 * inside a region where the allocator is off limits (an inference server
 * that reserved all device memory for its KV cache up front, a plugin whose
 * host framework owns the allocator and exposes none through a C ABI, a
 * real-time loop that cannot afford cudaMalloc's implicit synchronisation and
 * unbounded latency).
 *
 * Same arguments and results as gdn_chunk_fwd, without workspace / ws_bytes.
 * The scratch it needs (the longest-first schedule of a packed batch, one
 * int32 per sequence) lives in a fixed device array inside libgdn.so, sized
 * for GDN_NOALLOC_MAX_SEQS sequences (16 KiB), which every GPU that loads the
 * library keeps until the process exits.  It calls no allocator at all.
 *  - cu_seqlens != NULL with n_seq > GDN_NOALLOC_MAX_SEQS returns
 *    GDN_ERR_TOO_LARGE and launches nothing (dense batches have no limit).
 *  - The first call in each CUDA context (the primary context of each device,
 *    for runtime-API callers) looks up the array's device address
 *    (cudaGetSymbolAddress, with that context current) and caches it under the
 *    context; make that first call before capturing a stream into a CUDA graph.
 *  - A packed batch of any size, one sequence included, uses the array.
 *  - All calls share the one array, and every call overwrites the entries it
 *    uses before reading them, so nothing carries over between calls; but two
 *    calls that run on the GPU at the same time (different streams, or
 *    different host threads) race on it and must be serialised by the caller.
 */
#define GDN_NOALLOC_MAX_SEQS 4096
gdn_status gdn_chunk_fwd_noalloc(const void* q, const void* k, const void* v, gdn_dtype qkv_dtype,
                                 const float* g, const float* beta, const float* h0,
                                 const int32_t* cu_seqlens, int n_seq, int B, int64_t T, int H,
                                 int K, int V, float scale, void* o, gdn_dtype o_dtype, float* hT,
                                 unsigned flags, void* stream);

/*
 * gdn_conv1d_fwd -- causal depthwise conv1d over a packed batch (the short
 * convolution ahead of the gates).
 * ZzCompute, PyTorch Helion Hackathon gallery entry 11, item 1 ("Causal
 * Conv1d -- Depthwise Causal Convolution": each channel convolved on its own
 * with its past context, filter width 4, boundaries by masked loads):
 *     y[t,c] = bias[c] + sum_{i<W} w[c,i] x[t-(W-1)+i, c],   then y*sigmoid(y)
 *     when activation == 1 (SiLU),
 * per sequence; the taps before a sequence's first token read its initial
 * conv state (its W-1 previous inputs, oldest first) or zero.  Reading: the
 * last tap w[c,W-1] weighs the current input (the pages give no tap order).
 *   x, y        [rows, C] of `dtype` (GDN_F32 or GDN_BF16), rows = B*T dense, or
 *               T (= T_total) with cu_seqlens; y must not overlap x.
 *   w           [C, W] fp32, 1 <= W <= 4;  bias [C] fp32 or NULL.
 *   cu_seqlens  NULL: B sequences of T rows (n_seq must equal B); else int32
 *               [n_seq+1], nondecreasing from 0 to T, B must be 1.
 *   init_state  [n_seq, C, W-1] of `dtype`, or NULL for zeros.
 *   final_state [n_seq, C, W-1] of `dtype`, or NULL: each sequence's last W-1
 *               inputs, oldest first (initial-state values where it is shorter);
 *               must not be init_state.
 * Accumulation is fp32 (fmaf, taps in order), one rounding to `dtype`.  All
 * rows are HBM-streamed once, plus a W-1 row halo per 64-row run.
 * Returns GDN_ERR_INVALID_ARG for bad sizes/pointers, GDN_ERR_CUDA on launch
 * failure.
 */
gdn_status gdn_conv1d_fwd(const void* x, int dtype, const float* w, const float* bias, int W,
                          const int32_t* cu_seqlens, int n_seq, int B, int64_t T, int C,
                          const void* init_state, void* final_state, int activation, void* y,
                          void* stream);

/*
 * gdn_conv1d_update -- one decode token through the short convolution.
 * For request r with slot s = state_idx ? state_idx[r] : r:
 *     window = [conv_state[s, c, 0..W-2], x[r, c]];  y[r,c] = bias[c] + w[c,:].window
 *     (SiLU when activation == 1);  conv_state[s, c, :] = window[1..W-1].
 * A negative slot is padding: y[r,:] = 0 and no state is read or written
 * (Megatron-Core "core.ssm.ops.gdp.decode_prepare", module description: "a -1
 * slot zeroes its conv output").  A slot >= n_slots is treated the same way and
 * records GDN_ERR_INVALID_ARG in the device status word.
 *   x, y        [n, C] of `dtype`; y must not overlap x.
 *   conv_state  [n_slots, C, W-1] of `dtype`, in place; may be NULL when W == 1.
 *   state_idx   int32 [n] or NULL (then n_slots >= n and slot = r).  Distinct
 *               requests must name distinct slots.
 */
gdn_status gdn_conv1d_update(const void* x, int dtype, const float* w, const float* bias, int W,
                             void* conv_state, const int32_t* state_idx, int n, int n_slots, int C,
                             int activation, void* y, void* stream);

/*
 * Context parallelism over T.  The rule is linear in (h0, v) jointly, so a
 * sequence split into segments runs as: each segment from a zero state
 * (o_loc, h_loc); its transition matrix M (h_T of the segment with v = 0 and
 * h0 = I, key x key); the state entering segment r is s_{r-1}, where
 * s_0 = h_loc_0 and s_j = M_j s_{j-1} + h_loc_j; and segment r's output is
 * o_loc plus the output of a v = 0 pass from s_{r-1}.  These two calls are
 * the pieces of that which are not gdn_chunk_fwd itself.  (ZzCompute's "Chunk
 * Forward H" carries the state across chunks; this carries it across
 * segments the same way.)
 *
 * gdn_state_combine -- out[i] = A[i] X[i] (+ C[i]) for `count` matrices:
 *   A fp32 [count, K, K]; X, C, out fp32 [count, K, V]; C may be NULL; out may
 *   equal C but not X.  K in {32, 64, 128}; count <= 65535.
 * gdn_accumulate_f32 -- y[i] += x[i] for n fp32 elements.
 */
gdn_status gdn_state_combine(const float* A, const float* X, const float* C, float* out,
                             int64_t count, int K, int V, void* stream);
gdn_status gdn_accumulate_f32(float* y, const float* x, int64_t n, void* stream);

/*
 * gdn_device_status -- reads and clears the device status word on the current
 * device.  Kernels that wait on the device (mbarrier waits in the tensor-core
 * kernel) give up after a bounded number of polls, record GDN_ERR_TIMEOUT
 * there and return, so the context stays usable.  This call SYNCHRONISES the
 * stream.  Returns GDN_OK when nothing was recorded.
 */
gdn_status gdn_device_status(void* stream);

/* gdn_get_device_status -- the same call under the name of the method's API
 * call list (reads and clears the device status word; synchronises). */
gdn_status gdn_get_device_status(void* stream);

/*
 * gdn_selftest_wait_timeout -- launches one block that waits on an mbarrier
 * nothing will ever complete, polling at most `polls` times, then records
 * GDN_ERR_TIMEOUT in the device status word and returns.  Exercises the
 * failure path of the bounded waits without hanging or faulting the device.
 */
gdn_status gdn_selftest_wait_timeout(unsigned polls, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
