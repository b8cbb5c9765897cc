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
#include "tc_ptx.cuh"

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

// SiLU as y / (1 + 2^(-y log2 e)) from the hardware's approximate base-2
// exponential and reciprocal (ex2.approx.ftz / rcp.approx.ftz, each within a
// few fp32 ulp).  Rounding -y log2 e perturbs the exponential by at most
// |y| 2^-24 relative, so for |y| < 64 the result is within 2^-17 of SiLU
// relative, far inside the 8 bits of a bf16 output; below y = -87 the
// reciprocal flushes to zero and so does the result (|SiLU| < 2^-119 there).
// The packed form does the same per lane (each f32x2 lane one IEEE op), so
// every conv kernel gives the same bits.
__device__ __forceinline__ float conv_ex2(float t) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(t));
    return r;
}
__device__ __forceinline__ float conv_rcp(float d) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(d));
    return r;
}
constexpr float kNegLog2e = -1.4426950408889634f;
__device__ __forceinline__ float conv_silu(float y) {
    return y * conv_rcp(1.0f + conv_ex2(y * kNegLog2e));
}
__device__ __forceinline__ float2 conv_silu2(float2 y) {
    const float2 t = __fmul2_rn(y, make_float2(kNegLog2e, kNegLog2e));
    const float2 d = __fadd2_rn(make_float2(1.f, 1.f), make_float2(conv_ex2(t.x), conv_ex2(t.y)));
    return __fmul2_rn(y, make_float2(conv_rcp(d.x), conv_rcp(d.y)));
}

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

constexpr int kConvReqs = 16;  // requests per thread in the update (weights loaded once)
constexpr int kConvBatchReqs = 4;  // of which loaded together ahead of their stores

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
    // a channel's W = 4 taps (and four channels' biases) are one 16-byte unit
    const bool w16 = W == 4 && (reinterpret_cast<uintptr_t>(a.w) & 15u) == 0;
    const bool b16 = NV % 4 == 0 && a.bias && (reinterpret_cast<uintptr_t>(a.bias) & 15u) == 0;
#pragma unroll
    for (int j = 0; j < NV; ++j) {
        if (w16) {
            const float4 v = __ldg(reinterpret_cast<const float4*>(a.w + (int64_t)(c0 + j) * W));
            const float t4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < W; ++i) wt[i][j] = t4[i < 4 ? i : 0];
        } else {
#pragma unroll
            for (int i = 0; i < W; ++i) wt[i][j] = a.w[(int64_t)(c0 + j) * W + i];
        }
        if (b16) {
            if (j % 4 == 0) {
                const float4 v = __ldg(reinterpret_cast<const float4*>(a.bias + c0 + j));
                bs[j] = v.x;
                if (j + 1 < NV) bs[j + 1] = v.y;
                if (j + 2 < NV) bs[j + 2] = v.z;
                if (j + 3 < NV) bs[j + 3] = v.w;
            }
        } else {
            bs[j] = a.bias ? a.bias[c0 + j] : 0.f;
        }
    }
    const int rend = (blockIdx.y + 1) * kConvReqs < a.n ? (blockIdx.y + 1) * kConvReqs : a.n;
    if constexpr (NV * sizeof(T) == 16 && H > 0) {
        // 16-byte units: the loads of kConvBatchReqs requests are all issued before
        // any of their stores (the slots are distinct, so no store aliases a load),
        // so a thread waits on memory once per batch instead of once per request
        for (int rb = blockIdx.y * kConvReqs; rb < rend; rb += kConvBatchReqs) {
            int slot[kConvBatchReqs];
            uint4 xu[kConvBatchReqs], wu[kConvBatchReqs][H];
#pragma unroll
            for (int q = 0; q < kConvBatchReqs; ++q) {
                const int r = rb + q;
                slot[q] = r < rend ? (a.idx ? a.idx[r] : r) : -1;
            }
#pragma unroll
            for (int q = 0; q < kConvBatchReqs; ++q) {
                if (slot[q] >= 0 && slot[q] < a.n_slots) {
                    xu[q] = __ldg(reinterpret_cast<const uint4*>(x + (int64_t)(rb + q) * a.C + c0));
                    const uint4* sp =
                        reinterpret_cast<const uint4*>(state + ((int64_t)slot[q] * a.C + c0) * H);
#pragma unroll
                    for (int u = 0; u < H; ++u) wu[q][u] = sp[u];
                }
            }
#pragma unroll
            for (int q = 0; q < kConvBatchReqs; ++q) {
                const int r = rb + q;
                if (r >= rend) break;
                float o[NV];
                if (slot[q] < 0 || slot[q] >= a.n_slots) {
                    if (slot[q] >= a.n_slots) record_status(GDN_ERR_INVALID_ARG);
#pragma unroll
                    for (int j = 0; j < NV; ++j) o[j] = 0.f;
                    conv_store<T, NV>(y + (int64_t)r * a.C + c0, o);
                    continue;
                }
                const T* xe = reinterpret_cast<const T*>(&xu[q]);
                uint4 nu[H];
#pragma unroll
                for (int j = 0; j < NV; ++j) {
                    const float xc = to_f32(xe[j]);
                    float acc = bs[j];
#pragma unroll
                    for (int i = 0; i < H; ++i) {
                        const int e = j * H + i;
                        acc = fmaf(wt[i][j], to_f32(reinterpret_cast<const T*>(&wu[q][e / NV])[e % NV]),
                                   acc);
                    }
                    acc = fmaf(wt[H][j], xc, acc);
                    o[j] = ACT ? conv_silu(acc) : acc;
#pragma unroll
                    for (int i = 0; i < H; ++i) {
                        const int e = j * H + i;
                        const T v = (i + 1 < H)
                                        ? reinterpret_cast<const T*>(&wu[q][(e + 1) / NV])[(e + 1) % NV]
                                        : xe[j];
                        reinterpret_cast<T*>(&nu[e / NV])[e % NV] = v;
                    }
                }
                conv_store<T, NV>(y + (int64_t)r * a.C + c0, o);
                uint4* sp = reinterpret_cast<uint4*>(state + ((int64_t)slot[q] * a.C + c0) * H);
#pragma unroll
                for (int u = 0; u < H; ++u) sp[u] = nu[u];
            }
        }
    } else {
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
}

}  // namespace gdn

// ------------------------------------------------ conv1d forward, TMA stream
// The same computation for bf16, W = 4 and C a multiple of 256, restructured
// so the bytes in flight do not live in registers: a CTA owns a strip of 256
// channels and one contiguous range of rows.  A producer warp streams 32-row x
// 256-channel tiles (16 KB) into a three-stage ring with TMA; four compute
// warps (two channels per thread, so a thread owns one 4-byte column of the
// tile) take a tile's 32 rows into registers and write the 32 outputs back
// over them in place; the producer then stores the tile with TMA and, once
// the store has read it, loads the stage's next tile.
// Inside one sequence the 32 rows of a tile are independent given their
// inputs, so that path is unrolled without branches; a tile that holds a
// sequence boundary or the end of the range takes the row-by-row path.
namespace gdn {
namespace cvt {
constexpr int TR = 32;        // rows per tile
constexpr int TC = 256;       // channels per strip
constexpr int NS = 3;         // ring stages (four CTAs fit on an SM)
constexpr int kThreads = 160; // 4 compute warps + the producer warp
constexpr uint32_t TILE = TR * TC * 2;
constexpr uint32_t OFF_BAR = NS * TILE;
constexpr uint32_t SMEM = OFF_BAR + 2 * NS * 8 + 128;  // + alignment slack
constexpr uint32_t kPolls = 1u << 22;
}  // namespace cvt

struct ConvTmaParams {
    CUtensorMap tx, ty;  // x, y [rows, C] bf16, boxes of TR rows x TC channels, no swizzle
    ConvArgs a;
    int64_t rows_per_cta;  // a multiple of TR
};

template <bool ACT>
__global__ void __launch_bounds__(cvt::kThreads) conv1d_fwd_tma_kernel(
    const __grid_constant__ ConvTmaParams p) {
    using bf = __nv_bfloat16;
    constexpr int H = 3;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    uint8_t* base = smem_raw + (((raw_u32 + 127u) & ~127u) - raw_u32);
    uint64_t* full = reinterpret_cast<uint64_t*>(base + cvt::OFF_BAR);
    uint64_t* done = full + cvt::NS;  // outputs of the stage's tile written
    const ConvArgs& a = p.a;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int cs = blockIdx.x * cvt::TC;  // first channel of the strip
    const int64_t rbeg = (int64_t)blockIdx.y * p.rows_per_cta;
    const int64_t rend = rbeg + p.rows_per_cta < a.rows ? rbeg + p.rows_per_cta : a.rows;
    if (rbeg >= rend) return;
    const int ntiles = (int)((rend - rbeg + cvt::TR - 1) / cvt::TR);
    if (tid == 0) {
        for (int i = 0; i < cvt::NS; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&done[i], 4);  // one arrive per compute warp
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (warp == 4) {  // producer
        if (lane == 0) {
            tc::prefetch_tmap(&p.tx);
            tc::prefetch_tmap(&p.ty);
            auto load = [&](int i) {  // tile i into stage i % NS
                const int st_ = i % cvt::NS;
                tc::mbar_arrive_expect_tx(&full[st_], cvt::TILE);
                tc::tma_load_2d(base + st_ * cvt::TILE, &p.tx, cs,
                                (int)(rbeg + (int64_t)i * cvt::TR), &full[st_]);
            };
            int issued = 0;
            for (; issued < cvt::NS && issued < ntiles; ++issued) load(issued);
            int stored = 0;
            for (int i = 0; i < ntiles; ++i) {
                const int st_ = i % cvt::NS;
                if (!mbar_wait(&done[st_], (i / cvt::NS) & 1, cvt::kPolls)) break;
                tc::tma_store_2d(&p.ty, smem_u32(base + st_ * cvt::TILE), cs,
                                 (int)(rbeg + (int64_t)i * cvt::TR));
                tc::bulk_commit();
                stored = i + 1;
                if (i + cvt::NS < ntiles) {
                    tc::bulk_wait_read0();  // the store has read the stage
                    load(i + cvt::NS);
                    issued = i + cvt::NS + 1;
                }
            }
            tc::bulk_wait0();
            // after a wait gave up: no load may still be landing when the CTA leaves
            for (int i = stored; i < issued; ++i)
                if (!mbar_wait(&full[i % cvt::NS], (i / cvt::NS) & 1, cvt::kPolls)) break;
        }
        return;
    }
    const int c0 = cs + 2 * tid;  // this thread's two channels
    const bf* x = static_cast<const bf*>(a.x);
    const bf* init = static_cast<const bf*>(a.init);
    bf* fin = static_cast<bf*>(a.fin);
    // the two channels side by side: packed fp32 pairs (each lane one IEEE fma)
    float2 wt[4], bs;
#pragma unroll
    for (int i = 0; i < 4; ++i) wt[i] = make_float2(a.w[(int64_t)c0 * 4 + i], a.w[(int64_t)(c0 + 1) * 4 + i]);
    bs = a.bias ? make_float2(a.bias[c0], a.bias[c0 + 1]) : make_float2(0.f, 0.f);
    int s;
    int64_t st, en;
    conv_find_seq(a, rbeg, s, st, en);
    float2 win[H];
    auto fill = [&](int64_t r) {  // the H inputs before row r
#pragma unroll
        for (int i = 0; i < H; ++i) {
            const int64_t pos = r - H + i;
            float v[2];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                if (pos >= st)
                    v[j] = __bfloat162float(x[pos * a.C + c0 + j]);
                else if (init)
                    v[j] = __bfloat162float(init[((int64_t)s * a.C + c0 + j) * H + (H + (pos - st))]);
                else
                    v[j] = 0.f;
            }
            win[i] = make_float2(v[0], v[1]);
        }
    };
    // one row: output from the window and the row's inputs, then shift them in
    auto row = [&](uint32_t in, uint32_t* out) {
        __nv_bfloat162 b2;
        memcpy(&b2, &in, 4);
        const float2 xc = __bfloat1622float2(b2);
        float2 acc = bs;
#pragma unroll
        for (int k = 0; k < H; ++k) acc = __ffma2_rn(wt[k], win[k], acc);
        acc = __ffma2_rn(wt[H], xc, acc);
        if (ACT) acc = conv_silu2(acc);
        const __nv_bfloat162 ob = __floats2bfloat162_rn(acc.x, acc.y);
        uint32_t ou;
        memcpy(&ou, &ob, 4);
        *out = ou;
        win[0] = win[1];
        win[1] = win[2];
        win[2] = xc;
    };
    auto write_fin = [&]() {  // the sequence's last W-1 inputs, oldest first
#pragma unroll
        for (int k = 0; k < H; ++k) {
            fin[((int64_t)s * a.C + c0) * H + k] = __float2bfloat16_rn(win[k].x);
            fin[((int64_t)s * a.C + c0 + 1) * H + k] = __float2bfloat16_rn(win[k].y);
        }
    };
    fill(rbeg);
    bool ok = true;
    for (int i = 0; i < ntiles; ++i) {
        const int si = i % cvt::NS;
        if (ok) ok = mbar_wait(&full[si], (i / cvt::NS) & 1, cvt::kPolls);
        uint32_t* tio = reinterpret_cast<uint32_t*>(base + si * cvt::TILE) + tid;
        const int64_t t0 = rbeg + (int64_t)i * cvt::TR;
        if (t0 + cvt::TR <= en && t0 + cvt::TR <= rend) {
            uint32_t in[cvt::TR];
#pragma unroll
            for (int rr = 0; rr < cvt::TR; ++rr) in[rr] = tio[rr * (cvt::TC / 2)];
#pragma unroll
            for (int rr = 0; rr < cvt::TR; ++rr) row(in[rr], tio + rr * (cvt::TC / 2));
            if (fin && t0 + cvt::TR == en) write_fin();
        } else {
            for (int rr = 0; rr < cvt::TR; ++rr) {
                const int64_t r = t0 + rr;
                if (r >= rend) break;
                if (r == en) {  // next (non-empty) sequence
                    do {
                        ++s;
                        st = a.cu ? (int64_t)a.cu[s] : (int64_t)s * a.T;
                        en = a.cu ? (int64_t)a.cu[s + 1] : st + a.T;
                    } while (en <= r);
                    fill(r);  // all W-1 taps precede the new sequence: no row loads
                }
                row(tio[rr * (cvt::TC / 2)], tio + rr * (cvt::TC / 2));
                if (fin && r == en - 1) write_fin();
            }
        }
        // rows past the range's end are past the tensor's end: the store clips them
        tc::fence_async_smem();  // the outputs are visible to the TMA store
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&done[si]);
    }
}

}  // namespace gdn
