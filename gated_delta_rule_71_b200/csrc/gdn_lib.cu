// gdn_lib.cu -- the C ABI of libgdn.so (declared in include/gdn.h): host-side
// argument checks, kernel selection and launches.  One translation unit holds
// every kernel so that the device status word is a single symbol.
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "gdn.h"
#include "common.cuh"
#include "gates_decode.cuh"
#include "chunk_simt.cuh"
#include "chunk_tc.cuh"
#include "conv1d.cuh"
#include "decode_step.cuh"

namespace {

thread_local int t_last_cuda_error = 0;

gdn_status cuda_check(cudaError_t e) {
    if (e == cudaSuccess) return GDN_OK;
    t_last_cuda_error = (int)e;
    return GDN_ERR_CUDA;
}

gdn_status launch_check() { return cuda_check(cudaGetLastError()); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

int num_sms() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

bool head_dim_ok(int d) { return d == 32 || d == 64 || d == 128; }

// ------------------------------------------------------------- chunk (fp32)

template <int C, typename TIn, typename TOut>
gdn_status launch_simt(const gdn::ChunkArgs& a, int n_blocks, cudaStream_t st) {
    const size_t smem = (size_t)gdn::simt_smem_floats(C, a.K, a.VS) * sizeof(float);
    auto kern = gdn::chunk_fwd_simt_kernel<C, TIn, TOut>;
    gdn_status s = cuda_check(
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    if (s != GDN_OK) return s;
    kern<<<n_blocks, 256, smem, st>>>(a);
    return launch_check();
}

template <int C>
gdn_status launch_simt_dt(const gdn::ChunkArgs& a, gdn_dtype in, gdn_dtype out, int nb,
                          cudaStream_t st) {
    using bf = __nv_bfloat16;
    if (in == GDN_F32 && out == GDN_F32) return launch_simt<C, float, float>(a, nb, st);
    if (in == GDN_F32 && out == GDN_BF16) return launch_simt<C, float, bf>(a, nb, st);
    if (in == GDN_BF16 && out == GDN_F32) return launch_simt<C, bf, float>(a, nb, st);
    return launch_simt<C, bf, bf>(a, nb, st);
}

constexpr size_t kSimtSmemMax = 227 * 1024;

size_t ws_schedule_bytes(int n_seq) { return ((size_t)n_seq * 4 + 255) / 256 * 256; }

}  // namespace

namespace {

// ------------------------------------------------------------------ conv1d

template <typename T, int NV, int W, bool ACT>
gdn_status launch_conv_fwd(const gdn::ConvArgs& a, cudaStream_t st) {
    const int groups = a.C / NV;
    const int64_t runs = (a.rows + gdn::kConvRun - 1) / gdn::kConvRun;
    dim3 grid((groups + 127) / 128, (unsigned)(runs < 65535 ? runs : 65535));
    gdn::conv1d_fwd_kernel<T, NV, W, ACT><<<grid, 128, 0, st>>>(a);
    return launch_check();
}

template <typename T, int NV, bool ACT>
gdn_status conv_fwd_w(const gdn::ConvArgs& a, int W, cudaStream_t st) {
    switch (W) {
        case 1: return launch_conv_fwd<T, NV, 1, ACT>(a, st);
        case 2: return launch_conv_fwd<T, NV, 2, ACT>(a, st);
        case 3: return launch_conv_fwd<T, NV, 3, ACT>(a, st);
        default: return launch_conv_fwd<T, NV, 4, ACT>(a, st);
    }
}

// The TMA-streamed variant (bf16, W = 4, C % 256 == 0, 16-byte aligned x, y):
// strips of 256 channels x ranges of whole 32-row tiles, about one wave of
// four CTAs per SM.  Returns GDN_ERR_UNSUPPORTED when the tensor map cannot
// be built, so the caller can launch the register-streamed kernel instead.
template <bool ACT>
gdn_status launch_conv_fwd_tma(const gdn::ConvArgs& a, cudaStream_t st) {
    using namespace gdn;
    ConvTmaParams p;
    memset(&p, 0, sizeof(p));
    tcf::EncodeTiled enc = tcf::get_encode();
    if (!enc) return GDN_ERR_UNSUPPORTED;
    cuuint64_t dims[2] = {(cuuint64_t)a.C, (cuuint64_t)a.rows};
    cuuint64_t strides[1] = {(cuuint64_t)a.C * 2};
    cuuint32_t box[2] = {(cuuint32_t)cvt::TC, (cuuint32_t)cvt::TR};
    cuuint32_t estr[2] = {1, 1};
    CUtensorMap* maps[2] = {&p.tx, &p.ty};
    const void* ptrs[2] = {a.x, a.y};
    for (int i = 0; i < 2; ++i)
        if (enc(maps[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptrs[i]), dims,
                strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return GDN_ERR_UNSUPPORTED;
    p.a = a;
    const int strips = a.C / cvt::TC;
    const int64_t tiles = (a.rows + cvt::TR - 1) / cvt::TR;
    int64_t per = (int64_t)num_sms() * 4 / strips;  // row ranges per strip
    if (per < 1) per = 1;
    const int64_t tiles_per_cta = (tiles + per - 1) / per;
    p.rows_per_cta = tiles_per_cta * cvt::TR;
    const int64_t ny = (a.rows + p.rows_per_cta - 1) / p.rows_per_cta;
    if (ny > 65535) return GDN_ERR_UNSUPPORTED;
    auto kern = conv1d_fwd_tma_kernel<ACT>;
    gdn_status s = cuda_check(
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)cvt::SMEM));
    if (s != GDN_OK) return s;
    kern<<<dim3((unsigned)strips, (unsigned)ny), cvt::kThreads, cvt::SMEM, st>>>(p);
    return launch_check();
}

template <typename T>
gdn_status conv_fwd_t(const gdn::ConvArgs& a, int W, bool act, bool vec, cudaStream_t st) {
    constexpr int NV = gdn::ConvVec<T>::N;
    if (vec) return act ? conv_fwd_w<T, NV, true>(a, W, st) : conv_fwd_w<T, NV, false>(a, W, st);
    return act ? conv_fwd_w<T, 1, true>(a, W, st) : conv_fwd_w<T, 1, false>(a, W, st);
}

template <typename T, int NV, int W, bool ACT>
gdn_status launch_conv_upd(const gdn::ConvUpdateArgs& a, cudaStream_t st) {
    dim3 grid((a.C / NV + 127) / 128, (unsigned)((a.n + gdn::kConvReqs - 1) / gdn::kConvReqs));
    gdn::conv1d_update_kernel<T, NV, W, ACT><<<grid, 128, 0, st>>>(a);
    return launch_check();
}

template <typename T, int NV, bool ACT>
gdn_status conv_upd_w(const gdn::ConvUpdateArgs& a, int W, cudaStream_t st) {
    switch (W) {
        case 1: return launch_conv_upd<T, NV, 1, ACT>(a, st);
        case 2: return launch_conv_upd<T, NV, 2, ACT>(a, st);
        case 3: return launch_conv_upd<T, NV, 3, ACT>(a, st);
        default: return launch_conv_upd<T, NV, 4, ACT>(a, st);
    }
}

template <typename T>
gdn_status conv_upd_t(const gdn::ConvUpdateArgs& a, int W, bool act, bool vec,
                             cudaStream_t st) {
    constexpr int NV = gdn::ConvVec<T>::N;
    if (vec) return act ? conv_upd_w<T, NV, true>(a, W, st) : conv_upd_w<T, NV, false>(a, W, st);
    return act ? conv_upd_w<T, 1, true>(a, W, st) : conv_upd_w<T, 1, false>(a, W, st);
}

// The decode step (FUSED: behind the short-convolution update of its row).
// 64-column state slabs for P >= 64 (two blocks per (request, head) at P = 128),
// so four blocks fit per SM and one block's state loads overlap another's
// arithmetic.
template <bool FUSED>
gdn_status launch_decode(const void* x, int64_t xs, const void* ba, int64_t bas,
                         const float* A_log, const float* dt_bias, int n, int M, int H, int G,
                         int P, int N, float* state, const int32_t* state_idx, int n_slots,
                         void* o, float scale, int l2, const gdn::dec::ConvIn& cv,
                         cudaStream_t st) {
    using bf = __nv_bfloat16;
    const int nb = n * H;
#define GDN_DEC(NN, PP)                                                                          \
    if (N == NN && P == PP) {                                                                    \
        constexpr int PB = PP >= 64 ? 64 : PP;                                                   \
        gdn::dec::step_kernel<NN, PP, PB, FUSED><<<nb * (PP / PB), 256, 0, st>>>(                \
            (const bf*)x, xs, (const bf*)ba, bas, A_log, dt_bias, M, H, G, state, state_idx,     \
            n_slots, (bf*)o, scale, l2, cv);                                                     \
        return launch_check();                                                                   \
    }
    GDN_DEC(128, 128) GDN_DEC(128, 64) GDN_DEC(128, 32)
    GDN_DEC(64, 128) GDN_DEC(64, 64) GDN_DEC(64, 32)
    GDN_DEC(32, 128) GDN_DEC(32, 64) GDN_DEC(32, 32)
#undef GDN_DEC
    return GDN_ERR_UNSUPPORTED;
}

}  // namespace

extern "C" {

const char* gdn_status_string(int s) {
    switch (s) {
        case GDN_OK: return "GDN_OK";
        case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG: argument rejected on the host";
        case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED: size or dtype not built";
        case GDN_ERR_CUDA: return "GDN_ERR_CUDA: a CUDA call or launch failed";
        case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT: a bounded device wait gave up";
        case GDN_ERR_TOO_LARGE:
            return "GDN_ERR_TOO_LARGE: more packed sequences than gdn_chunk_fwd_noalloc's fixed "
                   "schedule array holds (GDN_NOALLOC_MAX_SEQS)";
        default: return "unknown gdn_status";
    }
}

int gdn_last_cuda_error(void) { return t_last_cuda_error; }

int gdn_version(void) { return 100; }

gdn_status gdn_gate_prep(const float* a, const float* b, int64_t n_tok, int H, int64_t a_stride,
                         int64_t b_stride, const float* A_log, const float* dt_bias, float* beta,
                         float* g, void* stream) {
    if (n_tok < 0 || H < 1 || a_stride < H || b_stride < H) return GDN_ERR_INVALID_ARG;
    if (n_tok == 0) return GDN_OK;
    if (!a || !b || !A_log || !dt_bias || !beta || !g) return GDN_ERR_INVALID_ARG;
    const int64_t total = n_tok * H;
    const int64_t want = (total + 255) / 256;
    const int blocks = (int)(want < (int64_t)num_sms() * 16 ? want : (int64_t)num_sms() * 16);
    gdn::gate_prep_kernel<<<blocks, 256, 0, as_stream(stream)>>>(a, b, n_tok, H, a_stride,
                                                                 b_stride, A_log, dt_bias, beta, g);
    return launch_check();
}

size_t gdn_chunk_fwd_workspace_size(int n_seq, int64_t T_total, int H, int K, int V,
                                    gdn_dtype qkv_dtype) {
    (void)K;
    (void)V;
    (void)qkv_dtype;
    if (n_seq <= 0 || H < 1 || T_total < 0) return 0;
    return ws_schedule_bytes(n_seq);
}

gdn_status gdn_chunk_fwd(const void* q, const void* k, const void* v, gdn_dtype qkv_dtype,
                         const float* g, const float* beta, const float* h0,
                         const int32_t* cu_seqlens, int n_seq, int B, int64_t T, int H, int K,
                         int V, float scale, void* o, gdn_dtype o_dtype, float* hT,
                         void* workspace, size_t ws_bytes, unsigned flags, void* stream) {
    if (B < 0 || T < 0 || H < 1 || n_seq < 0) return GDN_ERR_INVALID_ARG;
    if ((qkv_dtype != GDN_F32 && qkv_dtype != GDN_BF16) ||
        (o_dtype != GDN_F32 && o_dtype != GDN_BF16))
        return GDN_ERR_INVALID_ARG;
    if (cu_seqlens) {
        if (B != 1) return GDN_ERR_INVALID_ARG;
    } else {
        n_seq = B;
    }
    if (!head_dim_ok(K) || !head_dim_ok(V)) return GDN_ERR_UNSUPPORTED;
    if (n_seq == 0) return GDN_OK;
    if (B * T > 0 && (!q || !k || !v || !g || !beta || !o)) return GDN_ERR_INVALID_ARG;
    for (const void* p : {q, k, v, (const void*)h0, (const void*)o, (const void*)hT})
        if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;
    for (const void* p : {(const void*)g, (const void*)beta, (const void*)cu_seqlens})
        if (p && (reinterpret_cast<uintptr_t>(p) & 3u)) return GDN_ERR_INVALID_ARG;
    const size_t ws_need = cu_seqlens ? ws_schedule_bytes(n_seq) : 0;
    if (ws_need && (!workspace || ws_bytes < ws_need || !aligned16(workspace)))
        return GDN_ERR_INVALID_ARG;
    if (!cu_seqlens && (int64_t)n_seq * T * H > ((int64_t)1 << 40)) return GDN_ERR_UNSUPPORTED;

    cudaStream_t st = as_stream(stream);
    const int32_t* order = nullptr;
    if (cu_seqlens && n_seq > 1) {
        int32_t* ord = static_cast<int32_t*>(workspace);
        gdn::schedule_kernel<<<1, 1024, 0, st>>>(cu_seqlens, n_seq, ord);
        gdn_status s = launch_check();
        if (s != GDN_OK) return s;
        order = ord;
    }

    gdn::ChunkArgs a;
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.h0 = h0;
    a.cu_seqlens = cu_seqlens; a.order = order; a.n_seq = n_seq; a.T = T;
    a.H = H; a.K = K; a.V = V; a.scale = scale; a.o = o; a.hT = hT;

    int nvs_forced = (flags & GDN_FLAG_VSPLIT1) ? 1 : (flags & GDN_FLAG_VSPLIT2) ? 2
                   : (flags & GDN_FLAG_VSPLIT4) ? 4 : 0;

    const bool tc_ok = gdn::kTcAvailable && qkv_dtype == GDN_BF16 && K == 128 && V == 128 &&
                       (cu_seqlens ? T : (int64_t)B * T) > 0 &&
                       (cu_seqlens ? T : (int64_t)B * T) < ((int64_t)1 << 31) &&
                       (nvs_forced == 0 || nvs_forced == 2) &&
                       !(flags & (GDN_FLAG_EXACT_F32 | GDN_FLAG_CHUNK16 | GDN_FLAG_CHUNK32));
    if (tc_ok) {
        a.nvs = 2;
        a.VS = V / 2;
        const int64_t T_total = cu_seqlens ? T : (int64_t)B * T;
        const int rc = gdn::launch_chunk_tc(a, T_total, o_dtype == GDN_BF16, st);
        if (rc == 1) return GDN_ERR_UNSUPPORTED;
        if (rc == 2) {
            const cudaError_t e = cudaGetLastError();
            return cuda_check(e != cudaSuccess ? e : cudaErrorLaunchFailure);
        }
        return launch_check();
    }

    const int C = (flags & GDN_FLAG_CHUNK16) ? 16 : (flags & GDN_FLAG_CHUNK32) ? 32 : 64;
    int nvs = nvs_forced ? nvs_forced : (V > 32 ? V / 32 : 1);
    if (V % nvs) return GDN_ERR_UNSUPPORTED;
    a.nvs = nvs;
    a.VS = V / nvs;
    if ((size_t)gdn::simt_smem_floats(C, K, a.VS) * 4 > kSimtSmemMax) return GDN_ERR_UNSUPPORTED;
    const int64_t nb = (int64_t)n_seq * H * nvs;
    if (nb > 0x7fffffff) return GDN_ERR_UNSUPPORTED;
    if (C == 16) return launch_simt_dt<16>(a, qkv_dtype, o_dtype, (int)nb, st);
    if (C == 32) return launch_simt_dt<32>(a, qkv_dtype, o_dtype, (int)nb, st);
    return launch_simt_dt<64>(a, qkv_dtype, o_dtype, (int)nb, st);
}

static gdn_status decode_args_ok(const void* x, int64_t xs, const void* ba, int64_t bas,
                                 const float* A_log, const float* dt_bias, int n, int M, int H,
                                 int G, int P, int N) {
    if (n < 0 || M < 1 || H < 1 || G < 1 || H % G) return GDN_ERR_INVALID_ARG;
    if (!head_dim_ok(P) || !head_dim_ok(N)) return GDN_ERR_UNSUPPORTED;
    const int64_t row = (int64_t)M * H * P + (int64_t)M * G * N + (int64_t)G * N;
    if (xs < row || bas < (int64_t)M * H + H) return GDN_ERR_INVALID_ARG;
    if (n > 0 && (!x || !ba || !A_log || !dt_bias)) return GDN_ERR_INVALID_ARG;
    return GDN_OK;
}

gdn_status gdp_decode_prepare(const void* x, int64_t x_n_stride, const void* ba,
                              int64_t ba_n_stride, const float* A_log, const float* dt_bias, int n,
                              int M, int H, int G, int P, int N, void* q, void* k, void* v,
                              float* beta, float* g, void* stream) {
    gdn_status s = decode_args_ok(x, x_n_stride, ba, ba_n_stride, A_log, dt_bias, n, M, H, G, P, N);
    if (s != GDN_OK) return s;
    if (n == 0) return GDN_OK;
    if (!q || !k || !v || !beta || !g) return GDN_ERR_INVALID_ARG;
    if (M > 65535) return GDN_ERR_UNSUPPORTED;
    const bool vec = aligned16(x) && aligned16(q) && aligned16(k) && aligned16(v) &&
                     (x_n_stride % 8) == 0;
    using bf = __nv_bfloat16;
    dim3 grid(n, M);
    if (vec)
        gdn::gdp_prepare_kernel<true><<<grid, 256, 0, as_stream(stream)>>>(
            (const bf*)x, x_n_stride, (const bf*)ba, ba_n_stride, A_log, dt_bias, M, H, G, P, N,
            (bf*)q, (bf*)k, (bf*)v, beta, g);
    else
        gdn::gdp_prepare_kernel<false><<<grid, 256, 0, as_stream(stream)>>>(
            (const bf*)x, x_n_stride, (const bf*)ba, ba_n_stride, A_log, dt_bias, M, H, G, P, N,
            (bf*)q, (bf*)k, (bf*)v, beta, g);
    return launch_check();
}

gdn_status gdp_decode_step_indexed(const void* x, int64_t x_n_stride, const void* ba,
                                   int64_t ba_n_stride, const float* A_log, const float* dt_bias,
                                   int n, int M, int H, int G, int P, int N, float* state,
                                   const int32_t* state_idx, int n_slots, void* o, float scale,
                                   int qk_l2norm, void* stream) {
    gdn_status s = decode_args_ok(x, x_n_stride, ba, ba_n_stride, A_log, dt_bias, n, M, H, G, P, N);
    if (s != GDN_OK) return s;
    if (n == 0) return GDN_OK;
    if (!o || n_slots < 0 || (!state_idx && n_slots < n)) return GDN_ERR_INVALID_ARG;
    if (n_slots > 0 && (!state || !aligned16(state))) return GDN_ERR_INVALID_ARG;
    if (state_idx && (reinterpret_cast<uintptr_t>(state_idx) & 3u)) return GDN_ERR_INVALID_ARG;
    if (M > gdn::dec::kMaxM) return GDN_ERR_UNSUPPORTED;
    if ((int64_t)n * H * 2 > 0x7fffffff) return GDN_ERR_UNSUPPORTED;
    using bf = __nv_bfloat16;
    const int nb = n * H;
    cudaStream_t st = as_stream(stream);
    return launch_decode<false>(x, x_n_stride, ba, ba_n_stride, A_log, dt_bias, n, M, H, G, P, N,
                                state, state_idx, n_slots, o, scale, qk_l2norm, gdn::dec::ConvIn{},
                                as_stream(stream));
}

gdn_status gdp_decode_step(const void* x, int64_t x_n_stride, const void* ba, int64_t ba_n_stride,
                           const float* A_log, const float* dt_bias, int n, int M, int H, int G,
                           int P, int N, float* state, void* o, float scale, int qk_l2norm,
                           void* stream) {
    if (n > 0 && !state) return GDN_ERR_INVALID_ARG;
    return gdp_decode_step_indexed(x, x_n_stride, ba, ba_n_stride, A_log, dt_bias, n, M, H, G, P,
                                   N, state, nullptr, n, o, scale, qk_l2norm, stream);
}

size_t gdp_decode_layer_step_workspace_size(int n, int G) {
    if (n <= 0 || G <= 0) return 0;
    return ((size_t)n * G * 4 + 255) / 256 * 256;
}

gdn_status gdp_decode_layer_step(const void* x, int64_t x_n_stride, const void* ba,
                                 int64_t ba_n_stride, const float* conv_w, const float* conv_bias,
                                 int W, void* conv_state, int activation, const float* A_log,
                                 const float* dt_bias, int n, int M, int H, int G, int P, int N,
                                 float* state, const int32_t* state_idx, int n_slots, void* o,
                                 float scale, int qk_l2norm, void* workspace, size_t ws_bytes,
                                 void* stream) {
    gdn_status s = decode_args_ok(x, x_n_stride, ba, ba_n_stride, A_log, dt_bias, n, M, H, G, P, N);
    if (s != GDN_OK) return s;
    if (W < 1 || W > 4 || (activation != 0 && activation != 1)) return GDN_ERR_INVALID_ARG;
    if (n == 0) return GDN_OK;
    if (!o || !conv_w || (W > 1 && !conv_state) || n_slots < 0 || (!state_idx && n_slots < n))
        return GDN_ERR_INVALID_ARG;
    if (n_slots > 0 && (!state || !aligned16(state))) return GDN_ERR_INVALID_ARG;
    if (state_idx && (reinterpret_cast<uintptr_t>(state_idx) & 3u)) return GDN_ERR_INVALID_ARG;
    if (!workspace || ws_bytes < gdp_decode_layer_step_workspace_size(n, G) ||
        (reinterpret_cast<uintptr_t>(workspace) & 3u))
        return GDN_ERR_INVALID_ARG;
    if (M > gdn::dec::kMaxM) return GDN_ERR_UNSUPPORTED;
    if ((int64_t)n * H * 2 > 0x7fffffff) return GDN_ERR_UNSUPPORTED;
    const gdn::dec::ConvIn cv{conv_w, conv_bias, static_cast<__nv_bfloat16*>(conv_state),
                              static_cast<int32_t*>(workspace), W, activation};
    return launch_decode<true>(x, x_n_stride, ba, ba_n_stride, A_log, dt_bias, n, M, H, G, P, N,
                               state, state_idx, n_slots, o, scale, qk_l2norm, cv,
                               as_stream(stream));
}

}  // extern "C"

// ------------------------------------------------------------- GDP prefill

namespace {

size_t align256(size_t b) { return (b + 255) / 256 * 256; }

struct PrefillLayout {
    size_t q, k, v, beta, g, o_all, cu, chunk, total;
};

PrefillLayout prefill_layout(int n_seq, int64_t rows, int M, int H, int P, int N, gdn_dtype odt,
                             bool packed) {
    PrefillLayout L;
    const size_t cr = (size_t)rows * M * H;  // copy rows x heads
    size_t off = 0;
    auto take = [&](size_t bytes) { const size_t at = off; off += align256(bytes); return at; };
    L.q = take(cr * N * 2);
    L.k = take(cr * N * 2);
    L.v = take(cr * P * 2);
    L.beta = take(cr * 4);
    L.g = take(cr * 4);
    L.o_all = take(cr * P * (odt == GDN_BF16 ? 2 : 4));
    L.cu = packed ? take((size_t)(n_seq + 1) * 4) : off;
    L.chunk = off;  // gdn_chunk_fwd's own workspace (schedule, slot images)
    off += align256(gdn_chunk_fwd_workspace_size(n_seq, rows * M, H, N, P, GDN_BF16));
    L.total = off;
    return L;
}

}  // namespace

extern "C" {

size_t gdp_prefill_workspace_size(int n_seq, int64_t rows, int M, int H, int P, int N,
                                  gdn_dtype o_dtype, int packed) {
    if (n_seq < 0 || rows < 0 || M < 1 || H < 1 || P < 1 || N < 1) return 0;
    return prefill_layout(n_seq, rows, M, H, P, N, o_dtype, packed != 0).total;
}

gdn_status gdp_prefill(const void* x, int64_t x_n_stride, const void* ba, int64_t ba_n_stride,
                       const float* A_log, const float* dt_bias, const float* h0,
                       const int32_t* cu_seqlens, int n_seq, int B, int64_t T, int M, int H,
                       int G, int P, int N, float scale, void* o, gdn_dtype o_dtype, float* hT,
                       void* workspace, size_t ws_bytes, void* stream) {
    if (B < 0 || T < 0 || n_seq < 0) return GDN_ERR_INVALID_ARG;
    if (o_dtype != GDN_F32 && o_dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (cu_seqlens) {
        if (B != 1 || n_seq < 1) return GDN_ERR_INVALID_ARG;
    } else {
        n_seq = B;
    }
    const int64_t rows = cu_seqlens ? T : (int64_t)B * T;
    if (rows > 0x7fffffff || rows * (int64_t)(M > 0 ? M : 1) >= ((int64_t)1 << 31))
        return GDN_ERR_UNSUPPORTED;
    gdn_status s = decode_args_ok(x, x_n_stride, ba, ba_n_stride, A_log, dt_bias, (int)rows, M, H,
                                  G, P, N);
    if (s != GDN_OK) return s;
    if (n_seq == 0) return GDN_OK;
    if (rows > 0 && !o) return GDN_ERR_INVALID_ARG;
    for (const void* p : {(const void*)h0, (const void*)o, (const void*)hT})
        if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;
    const PrefillLayout L = prefill_layout(n_seq, rows, M, H, P, N, o_dtype, cu_seqlens != nullptr);
    if (!workspace || ws_bytes < L.total || !aligned16(workspace)) return GDN_ERR_INVALID_ARG;
    cudaStream_t st = as_stream(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    float* beta = reinterpret_cast<float*>(ws + L.beta);
    float* g = reinterpret_cast<float*>(ws + L.g);
    if (rows > 0) {
        s = gdp_decode_prepare(x, x_n_stride, ba, ba_n_stride, A_log, dt_bias, (int)rows, M, H, G,
                               P, N, ws + L.q, ws + L.k, ws + L.v, beta, g, stream);
        if (s != GDN_OK) return s;
    }
    const int32_t* cu_m = nullptr;
    if (cu_seqlens) {
        int32_t* c = reinterpret_cast<int32_t*>(ws + L.cu);
        gdn::gdp_scale_offsets_kernel<<<(n_seq + 256) / 256, 256, 0, st>>>(cu_seqlens, n_seq, M, c);
        s = launch_check();
        if (s != GDN_OK) return s;
        cu_m = c;
    }
    s = gdn_chunk_fwd(ws + L.q, ws + L.k, ws + L.v, GDN_BF16, g, beta, h0, cu_m, n_seq, B, T * M,
                      H, N, P, scale, ws + L.o_all, o_dtype, hT,
                      ws + L.chunk, L.total - L.chunk, 0u, stream);
    if (s != GDN_OK || rows == 0) return s;
    const int64_t row_units = (int64_t)H * P * (o_dtype == GDN_BF16 ? 2 : 4) / 16;
    const int64_t want = (rows * row_units + 255) / 256;
    const int blocks = (int)(want < (int64_t)num_sms() * 16 ? want : (int64_t)num_sms() * 16);
    gdn::gdp_last_copy_kernel<<<blocks, 256, 0, st>>>(
        reinterpret_cast<const uint4*>(ws + L.o_all), rows, M, row_units, static_cast<uint4*>(o));
    return launch_check();
}

gdn_status gdn_state_combine(const float* A, const float* X, const float* C, float* out,
                             int64_t count, int K, int V, void* stream) {
    if (count < 0 || !head_dim_ok(K) || V < 1) return count < 0 ? GDN_ERR_INVALID_ARG
                                                                 : GDN_ERR_UNSUPPORTED;
    if (count == 0) return GDN_OK;
    if (!A || !X || !out || out == X) return GDN_ERR_INVALID_ARG;
    if (count > 65535) return GDN_ERR_UNSUPPORTED;
    dim3 grid((V + 31) / 32, (unsigned)count);
    cudaStream_t st = as_stream(stream);
    if (K == 128) gdn::state_combine_kernel<128><<<grid, 256, 0, st>>>(A, X, C, out, V);
    else if (K == 64) gdn::state_combine_kernel<64><<<grid, 256, 0, st>>>(A, X, C, out, V);
    else gdn::state_combine_kernel<32><<<grid, 256, 0, st>>>(A, X, C, out, V);
    return launch_check();
}

gdn_status gdn_accumulate_f32(float* y, const float* x, int64_t n, void* stream) {
    if (n < 0) return GDN_ERR_INVALID_ARG;
    if (n == 0) return GDN_OK;
    if (!y || !x) return GDN_ERR_INVALID_ARG;
    const int64_t want = (n + 255) / 256;
    const int blocks = (int)(want < (int64_t)num_sms() * 16 ? want : (int64_t)num_sms() * 16);
    gdn::accumulate_f32_kernel<<<blocks, 256, 0, as_stream(stream)>>>(y, x, n);
    return launch_check();
}

gdn_status gdn_conv1d_fwd(const void* x, int dtype, const float* w, const float* bias, int W,
                          const int32_t* cu_seqlens, int n_seq, int B, int64_t T, int C,
                          const void* init_state, void* final_state, int activation, void* y,
                          void* stream) {
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (W < 1 || W > 4 || C < 1 || T < 0 || (activation != 0 && activation != 1))
        return GDN_ERR_INVALID_ARG;
    if (cu_seqlens ? (B != 1 || n_seq < 1) : (B < 1 || n_seq != B)) return GDN_ERR_INVALID_ARG;
    const int64_t rows = cu_seqlens ? T : (int64_t)B * T;
    if (rows > 0 && (!x || !w || !y || x == y)) return GDN_ERR_INVALID_ARG;
    if (final_state && final_state == init_state) return GDN_ERR_INVALID_ARG;
    const size_t es = dtype == GDN_BF16 ? 2 : 4;
    const int nv = (int)(16 / es);
    const bool vec = C % nv == 0 && aligned16(x) && aligned16(y) &&
                     (!init_state || aligned16(init_state)) && (!final_state || aligned16(final_state));
    gdn::ConvArgs a{x, w, bias, cu_seqlens, n_seq, T, rows, C, init_state, final_state, y};
    cudaStream_t st = as_stream(stream);
    const bool tma = dtype == GDN_BF16 && W == 4 && C % gdn::cvt::TC == 0 && aligned16(x) &&
                     aligned16(y) && rows < ((int64_t)1 << 30);
    bool rows_done = false;
    if (rows > 0 && tma) {
        gdn_status s = activation == 1 ? launch_conv_fwd_tma<true>(a, st)
                                       : launch_conv_fwd_tma<false>(a, st);
        if (s != GDN_OK && s != GDN_ERR_UNSUPPORTED) return s;
        if (s == GDN_OK) rows_done = true;
    }
    if (rows > 0 && !rows_done) {
        gdn_status s = dtype == GDN_BF16
                           ? conv_fwd_t<__nv_bfloat16>(a, W, activation == 1, vec, st)
                           : conv_fwd_t<float>(a, W, activation == 1, vec, st);
        if (s != GDN_OK) return s;
    }
    if (final_state && W > 1 && (cu_seqlens || T == 0)) {
        // empty sequences keep their initial state (or zeros)
        if (n_seq > 65535) return GDN_ERR_UNSUPPORTED;
        const int64_t n = (int64_t)C * (W - 1);
        dim3 grid((unsigned)((n + 255) / 256 < 64 ? (n + 255) / 256 : 64), (unsigned)n_seq);
        if (dtype == GDN_BF16)
            gdn::conv1d_final_empty_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(a, W - 1);
        else
            gdn::conv1d_final_empty_kernel<float><<<grid, 256, 0, st>>>(a, W - 1);
        return launch_check();
    }
    return GDN_OK;
}

gdn_status gdn_conv1d_update(const void* x, int dtype, const float* w, const float* bias, int W,
                             void* conv_state, const int32_t* state_idx, int n, int n_slots, int C,
                             int activation, void* y, void* stream) {
    if (dtype != GDN_F32 && dtype != GDN_BF16) return GDN_ERR_INVALID_ARG;
    if (W < 1 || W > 4 || C < 1 || n < 0 || n_slots < 0 || (activation != 0 && activation != 1))
        return GDN_ERR_INVALID_ARG;
    if (!state_idx && n_slots < n) return GDN_ERR_INVALID_ARG;
    if (n == 0) return GDN_OK;
    if (!x || !w || !y || x == y || (W > 1 && !conv_state)) return GDN_ERR_INVALID_ARG;
    if (n > 65535 * gdn::kConvReqs) return GDN_ERR_UNSUPPORTED;
    const size_t es = dtype == GDN_BF16 ? 2 : 4;
    const int nv = (int)(16 / es);
    const bool vec = C % nv == 0 && aligned16(x) && aligned16(y) &&
                     (!conv_state || aligned16(conv_state));
    gdn::ConvUpdateArgs a{x, w, bias, conv_state, state_idx, n, n_slots, C, y};
    cudaStream_t st = as_stream(stream);
    return dtype == GDN_BF16 ? conv_upd_t<__nv_bfloat16>(a, W, activation == 1, vec, st)
                             : conv_upd_t<float>(a, W, activation == 1, vec, st);
}

gdn_status gdn_device_status(void* stream) {
    cudaStream_t st = as_stream(stream);
    unsigned int word = 0, zero = 0;
    gdn_status s = cuda_check(cudaMemcpyFromSymbolAsync(&word, gdn::g_status_word, sizeof(word), 0,
                                                        cudaMemcpyDeviceToHost, st));
    if (s != GDN_OK) return s;
    s = cuda_check(cudaMemcpyToSymbolAsync(gdn::g_status_word, &zero, sizeof(zero), 0,
                                           cudaMemcpyHostToDevice, st));
    if (s != GDN_OK) return s;
    s = cuda_check(cudaStreamSynchronize(st));
    if (s != GDN_OK) return s;
    return (gdn_status)word;
}

gdn_status gdn_get_device_status(void* stream) { return gdn_device_status(stream); }

}  // extern "C"

namespace gdn {
__global__ void selftest_wait_kernel(unsigned polls) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, polls);  // nothing ever arrives
    __syncthreads();
}
}  // namespace gdn

extern "C" gdn_status gdn_selftest_wait_timeout(unsigned polls, void* stream) {
    if (polls == 0 || polls > (1u << 20)) return GDN_ERR_INVALID_ARG;
    gdn::selftest_wait_kernel<<<1, 32, 0, as_stream(stream)>>>(polls);
    return launch_check();
}

// ----------------------------------------------------------------------------
// gdn_chunk_fwd_noalloc: the chunked forward for callers that cannot allocate
// device memory (see include/gdn.h).  Its only scratch -- the longest-first
// schedule of a packed batch -- lives in this fixed device array instead of a
// caller-provided workspace.  Host code must not hand the array's name to a
// kernel: on the host it is only a stand-in symbol, so its device address is
// looked up with cudaGetSymbolAddress once per CUDA context (the array has one
// instance per context that loads this module) and cached under that context.
static __device__ __align__(256) int32_t g_noalloc_schedule[GDN_NOALLOC_MAX_SEQS];

namespace {
constexpr int kNoAllocMaxContexts = 64;
std::mutex g_noalloc_mutex;
CUcontext g_noalloc_ctx[kNoAllocMaxContexts] = {};
void* g_noalloc_addr[kNoAllocMaxContexts] = {};
int g_noalloc_used = 0;

// The calling thread's current CUDA context (the device's primary context once
// the runtime has initialised it), through the driver entry point the runtime
// exposes, so the library needs no link against the driver library.
gdn_status current_context(CUcontext* out) {
    static PFN_cuCtxGetCurrent_v4000 fn = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            f = nullptr;
        return reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
    }();
    if (!fn) return GDN_ERR_CUDA;
    *out = nullptr;
    if (fn(out) != CUDA_SUCCESS) return GDN_ERR_CUDA;
    if (!*out) {
        // nothing current on this thread yet: let the runtime make its context current
        gdn_status s = cuda_check(cudaFree(nullptr));
        if (s != GDN_OK) return s;
        if (fn(out) != CUDA_SUCCESS || !*out) return GDN_ERR_CUDA;
    }
    return GDN_OK;
}

// Device address of g_noalloc_schedule in the current context; looked up on the
// first call in that context (this is why that first call must not be made
// while a stream is being captured).
gdn_status noalloc_schedule_addr(void** out) {
    CUcontext ctx = nullptr;
    gdn_status s = current_context(&ctx);
    if (s != GDN_OK) return s;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    for (int i = 0; i < g_noalloc_used; ++i)
        if (g_noalloc_ctx[i] == ctx) {
            *out = g_noalloc_addr[i];
            return GDN_OK;
        }
    void* p = nullptr;
    s = cuda_check(cudaGetSymbolAddress(&p, g_noalloc_schedule));
    if (s != GDN_OK) return s;
    if (g_noalloc_used < kNoAllocMaxContexts) {
        g_noalloc_ctx[g_noalloc_used] = ctx;
        g_noalloc_addr[g_noalloc_used] = p;
        ++g_noalloc_used;
    }
    *out = p;
    return GDN_OK;
}
}  // namespace

extern "C" gdn_status gdn_chunk_fwd_noalloc(const void* q, const void* k, const void* v,
                                            gdn_dtype qkv_dtype, const float* g,
                                            const float* beta, const float* h0,
                                            const int32_t* cu_seqlens, int n_seq, int B,
                                            int64_t T, int H, int K, int V, float scale, void* o,
                                            gdn_dtype o_dtype, float* hT, unsigned flags,
                                            void* stream) {
    void* ws = nullptr;
    size_t ws_bytes = 0;
    if (cu_seqlens) {
        if (n_seq > GDN_NOALLOC_MAX_SEQS) return GDN_ERR_TOO_LARGE;
        if (n_seq >= 1) {
            // gdn_chunk_fwd wants a schedule buffer for every packed batch (even one
            // of a single sequence, whose schedule it does not build); every entry
            // the schedule kernel later reads it first writes, so the array needs
            // no clearing between calls
            gdn_status s = noalloc_schedule_addr(&ws);
            if (s != GDN_OK) return s;
            ws_bytes = sizeof(g_noalloc_schedule);
        }
    }
    return gdn_chunk_fwd(q, k, v, qkv_dtype, g, beta, h0, cu_seqlens, n_seq, B, T, H, K, V, scale,
                         o, o_dtype, hT, ws, ws_bytes, flags, stream);
}
