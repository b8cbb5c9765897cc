// conv1d.cuh -- causal depthwise conv1d (the short convolution ahead of the
// gates) and its one-token decode update.
//
// ZzCompute (PyTorch Helion Hackathon gallery entry 11), item 1, "Causal
// Conv1d -- Depthwise Causal Convolution": every channel is convolved on its
// own with its past context, filter width W = 4 fixed at compile time, the
// sequence boundaries handled by masked loads instead of host padding.  Per
// sequence and channel:
//     y[t,c] = bias[c] + sum_{i<W} w[c,i] x[t-(W-1)+i, c]   (SiLU optional)
// with the taps before the sequence start reading its initial conv state (the
// W-1 previous inputs, oldest first) or zero.  The decode update shifts that
// window by one token; a -1 slot is padding, which zeroes the output and
// leaves the state alone (Megatron-Core "core.ssm.ops.gdp.decode_prepare",
// module description).
//
// Layout: x, y [rows, C] channels-last (rows = tokens of the packed batch);
// w [C, W] fp32; bias [C] fp32; conv state [*, C, W-1] in the activation dtype
// (it holds raw inputs, so carrying it in that dtype loses nothing).
// Both kernels are HBM-bound streams: a warp moves 32 x 16 contiguous bytes per
// row; each thread walks a run of rows keeping the W-1 previous inputs in
// registers, so a row is read once (plus a W-1 row halo per run).
#pragma once

#include "common.cuh"

namespace gdn {

struct ConvArgs {
    const void* x;
    const float* w;
    const float* bias;
    const int32_t* cu;  // [n_seq + 1] or null (dense: n_seq sequences of T rows)
    int n_seq;
    int64_t T;
    int64_t rows;
    int C;
    const void* init;   // [n_seq, C, W-1] or null
    void* fin;          // [n_seq, C, W-1] or null
    void* y;
};

constexpr int kConvRun = 64;   // rows per thread
constexpr int kConvBatch = 8;  // rows loaded ahead of use

template <typename T> struct ConvVec { static constexpr int N = 16 / sizeof(T); };

// NV consecutive channels of one row (16-byte units when NV fills 16 bytes).
template <typename T, int NV>
__device__ __forceinline__ void conv_load(const T* p, float (&v)[NV]) {
    if constexpr (NV * sizeof(T) == 16) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
        const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
        for (int i = 0; i < NV; ++i) v[i] = to_f32(e[i]);
    } else {
#pragma unroll
        for (int i = 0; i < NV; ++i) v[i] = to_f32(p[i]);
    }
}
template <typename T, int NV>
__device__ __forceinline__ void conv_store(T* p, const float (&v)[NV]) {
    if constexpr (NV * sizeof(T) == 16) {
        uint4 u;
        T* e = reinterpret_cast<T*>(&u);
#pragma unroll
        for (int i = 0; i < NV; ++i) e[i] = from_f32<T>(v[i]);
        *reinterpret_cast<uint4*>(p) = u;
    } else {
#pragma unroll
        for (int i = 0; i < NV; ++i) p[i] = from_f32<T>(v[i]);
    }
}

// SiLU with the fast exponential and divide (bf16 outputs carry 8 bits; the
// fp32 error of __expf / __fdividef stays below 2^-20 relative here).
__device__ __forceinline__ float conv_silu(float y) { return __fdividef(y, 1.0f + __expf(-y)); }

// One row's NV channels as loaded (16-byte unit, or NV scalars), converted later.
template <typename T, int NV, bool V16 = (NV * sizeof(T) == 16)>
struct ConvRaw {
    T e[NV];
    __device__ __forceinline__ void load(const T* p) {
#pragma unroll
        for (int i = 0; i < NV; ++i) e[i] = p[i];
    }
    __device__ __forceinline__ float get(int i) const { return to_f32(e[i]); }
};
template <typename T, int NV>
struct ConvRaw<T, NV, true> {
    uint4 u;
    __device__ __forceinline__ void load(const T* p) { u = __ldg(reinterpret_cast<const uint4*>(p)); }
    __device__ __forceinline__ float get(int i) const { return to_f32(reinterpret_cast<const T*>(&u)[i]); }
};

// Sequence holding row r: [st, en) of sequence s.
__device__ __forceinline__ void conv_find_seq(const ConvArgs& a, int64_t r, int& s, int64_t& st,
                                              int64_t& en) {
    if (!a.cu) {
        s = (int)(r / a.T);
        st = (int64_t)s * a.T;
        en = st + a.T;
        return;
    }
    int lo = 0, hi = a.n_seq;  // last s with cu[s] <= r (skips empty sequences)
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a.cu[mid] <= r)
            lo = mid;
        else
            hi = mid - 1;
    }
    s = lo;
    st = a.cu[s];
    en = a.cu[s + 1];
}

// Grid: x over groups of NV channels (128 threads per block), y over runs of
// kConvRun rows (grid-stride).  A run may cross sequence boundaries: the window
// restarts from the next sequence's initial state there.
template <typename T, int NV, int W, bool ACT>
__global__ void __launch_bounds__(128, 4) conv1d_fwd_kernel(const ConvArgs a) {
    constexpr int H = W - 1;
    const int c0 = (blockIdx.x * blockDim.x + threadIdx.x) * NV;
    if (c0 >= a.C) return;
    const T* x = static_cast<const T*>(a.x);
    const T* init = static_cast<const T*>(a.init);
    T* y = static_cast<T*>(a.y);
    T* fin = static_cast<T*>(a.fin);
    float wt[W][NV], bs[NV];
#pragma unroll
    for (int j = 0; j < NV; ++j) {
#pragma unroll
        for (int i = 0; i < W; ++i) wt[i][j] = a.w[(int64_t)(c0 + j) * W + i];
        bs[j] = a.bias ? a.bias[c0 + j] : 0.f;
    }
    for (int64_t r0 = (int64_t)blockIdx.y * kConvRun; r0 < a.rows;
         r0 += (int64_t)gridDim.y * kConvRun) {
        int s;
        int64_t st, en;
        conv_find_seq(a, r0, s, st, en);
        float win[H > 0 ? H : 1][NV];
        // the H inputs before row r0: this sequence's rows, else its initial state
        auto fill = [&](int64_t r) {
#pragma unroll
            for (int i = 0; i < H; ++i) {
                const int64_t pos = r - H + i;
                if (pos >= st) {
                    conv_load<T, NV>(x + pos * a.C + c0, win[i]);
                } else if (init) {
                    const int64_t b = ((int64_t)s * a.C + c0) * H + (H + (pos - st));
#pragma unroll
                    for (int j = 0; j < NV; ++j) win[i][j] = to_f32(init[b + (int64_t)j * H]);
                } else {
#pragma unroll
                    for (int j = 0; j < NV; ++j) win[i][j] = 0.f;
                }
            }
        };
        fill(r0);
        const int64_t r1 = (r0 + kConvRun < a.rows) ? r0 + kConvRun : a.rows;
        // rows in batches of kConvBatch: every load of a batch is in flight before
        // the first one is used
        for (int64_t rb = r0; rb < r1; rb += kConvBatch) {
            ConvRaw<T, NV> raw[kConvBatch];
#pragma unroll
            for (int k = 0; k < kConvBatch; ++k)
                if (rb + k < r1) raw[k].load(x + (rb + k) * a.C + c0);
#pragma unroll
            for (int k = 0; k < kConvBatch; ++k) {
                const int64_t r = rb + k;
                if (r >= r1) break;
                if (r == en) {  // next (non-empty) sequence
                    do {
                        ++s;
                        st = a.cu ? (int64_t)a.cu[s] : (int64_t)s * a.T;
                        en = a.cu ? (int64_t)a.cu[s + 1] : st + a.T;
                    } while (en <= r);
                    fill(r);  // all W-1 taps precede the new sequence: no row loads
                }
                float xc[NV], o[NV];
#pragma unroll
                for (int j = 0; j < NV; ++j) xc[j] = raw[k].get(j);
#pragma unroll
                for (int j = 0; j < NV; ++j) {
                    float acc = bs[j];
#pragma unroll
                    for (int i = 0; i < H; ++i) acc = fmaf(wt[i][j], win[i][j], acc);
                    acc = fmaf(wt[H][j], xc[j], acc);
                    o[j] = ACT ? conv_silu(acc) : acc;
                }
                conv_store<T, NV>(y + r * a.C + c0, o);
#pragma unroll
                for (int i = 0; i + 1 < H; ++i)
#pragma unroll
                    for (int j = 0; j < NV; ++j) win[i][j] = win[i + 1][j];
                if constexpr (H > 0) {
#pragma unroll
                    for (int j = 0; j < NV; ++j) win[H - 1][j] = xc[j];
                }
                if (fin && r == en - 1) {  // the sequence's last W-1 inputs, oldest first
                    const int64_t b = ((int64_t)s * a.C + c0) * H;
#pragma unroll
                    for (int j = 0; j < NV; ++j)
#pragma unroll
                        for (int i = 0; i < H; ++i)
                            fin[b + (int64_t)j * H + i] = from_f32<T>(win[i][j]);
                }
            }
        }
    }
}

// Final state of empty sequences: their initial state (or zeros), unchanged.
template <typename T>
__global__ void __launch_bounds__(256) conv1d_final_empty_kernel(const ConvArgs a, int H) {
    const int s = blockIdx.y;
    const int64_t len = a.cu ? (int64_t)a.cu[s + 1] - a.cu[s] : a.T;
    if (len > 0) return;
    const T* init = static_cast<const T*>(a.init);
    T* fin = static_cast<T*>(a.fin);
    const int64_t n = (int64_t)a.C * H;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x)
        fin[(int64_t)s * n + i] = init ? init[(int64_t)s * n + i] : from_f32<T>(0.f);
}

struct ConvUpdateArgs {
    const void* x;       // [n, C]
    const float* w;
    const float* bias;
    void* state;         // [n_slots, C, W-1]
    const int32_t* idx;  // [n] or null
    int n;
    int n_slots;
    int C;
    void* y;             // [n, C]
};

constexpr int kConvReqs = 8;  // requests per thread in the update (weights loaded once)

// Grid: x over groups of NV channels (128 threads per block), y over groups of
// kConvReqs requests.  Requests must name distinct slots (each slot's window is
// read and written by the threads of one request).
template <typename T, int NV, int W, bool ACT>
__global__ void __launch_bounds__(128) conv1d_update_kernel(const ConvUpdateArgs a) {
    constexpr int H = W - 1;
    const int c0 = (blockIdx.x * blockDim.x + threadIdx.x) * NV;
    if (c0 >= a.C) return;
    const T* x = static_cast<const T*>(a.x);
    T* y = static_cast<T*>(a.y);
    T* state = static_cast<T*>(a.state);
    float wt[W][NV], bs[NV];
#pragma unroll
    for (int j = 0; j < NV; ++j) {
#pragma unroll
        for (int i = 0; i < W; ++i) wt[i][j] = a.w[(int64_t)(c0 + j) * W + i];
        bs[j] = a.bias ? a.bias[c0 + j] : 0.f;
    }
    const int rend = (blockIdx.y + 1) * kConvReqs < a.n ? (blockIdx.y + 1) * kConvReqs : a.n;
    for (int r = blockIdx.y * kConvReqs; r < rend; ++r) {
        const int slot = a.idx ? a.idx[r] : r;
        float o[NV];
        if (slot < 0 || slot >= a.n_slots) {
            if (slot >= a.n_slots) record_status(GDN_ERR_INVALID_ARG);
#pragma unroll
            for (int j = 0; j < NV; ++j) o[j] = 0.f;
            conv_store<T, NV>(y + (int64_t)r * a.C + c0, o);
            continue;
        }
        float xc[NV];
        conv_load<T, NV>(x + (int64_t)r * a.C + c0, xc);
        T* sp = state + ((int64_t)slot * a.C + c0) * H;  // NV*H contiguous values
        if constexpr (NV * sizeof(T) == 16) {
            // the window is H 16-byte units; element e = j*H + i sits in unit e / NV
            uint4 wu[H > 0 ? H : 1], nu[H > 0 ? H : 1];
#pragma unroll
            for (int u = 0; u < H; ++u) wu[u] = reinterpret_cast<const uint4*>(sp)[u];
#pragma unroll
            for (int j = 0; j < NV; ++j) {
                float acc = bs[j];
#pragma unroll
                for (int i = 0; i < H; ++i) {
                    const int e = j * H + i;
                    acc = fmaf(wt[i][j], to_f32(reinterpret_cast<const T*>(&wu[e / NV])[e % NV]), acc);
                }
                acc = fmaf(wt[H][j], xc[j], acc);
                o[j] = ACT ? conv_silu(acc) : acc;
#pragma unroll
                for (int i = 0; i < H; ++i) {
                    const int e = j * H + i;
                    const T v = (i + 1 < H) ? reinterpret_cast<const T*>(&wu[(e + 1) / NV])[(e + 1) % NV]
                                            : from_f32<T>(xc[j]);
                    reinterpret_cast<T*>(&nu[e / NV])[e % NV] = v;
                }
            }
#pragma unroll
            for (int u = 0; u < H; ++u) reinterpret_cast<uint4*>(sp)[u] = nu[u];
        } else {
#pragma unroll
            for (int j = 0; j < NV; ++j) {
                float win[H > 0 ? H : 1];
#pragma unroll
                for (int i = 0; i < H; ++i) win[i] = to_f32(sp[j * H + i]);
                float acc = bs[j];
#pragma unroll
                for (int i = 0; i < H; ++i) acc = fmaf(wt[i][j], win[i], acc);
                acc = fmaf(wt[H][j], xc[j], acc);
                o[j] = ACT ? conv_silu(acc) : acc;
#pragma unroll
                for (int i = 0; i + 1 < H; ++i) sp[j * H + i] = from_f32<T>(win[i + 1]);
                if constexpr (H > 0) sp[j * H + H - 1] = from_f32<T>(xc[j]);
            }
        }
        conv_store<T, NV>(y + (int64_t)r * a.C + c0, o);
    }
}

}  // namespace gdn
