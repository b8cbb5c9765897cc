// decode_step.cuh -- the Gated Delta Product decode step, on its own or fused
// behind the short-convolution update of its input row.
//
// The step: per request r and head h, the M Householder copies of the token
// run the gated delta rule on the fp32 state S [N, P] in turn (decay on copy
// 0, write strength beta per copy), and o = scale * S^T q after the last copy
// (Megatron-Core "core.ssm.ops.gdp.decode_prepare": the split of the
// post-conv row [value M*H*P | key M*G*N | query G*N] and of ba [b M*H | a H],
// the GQA expansion, the query on copy M-1, the gates).  The fused form takes
// the row before the short convolution and convolves it on the way in
// (Megatron-Core decode_prepare, module description: the short-conv update
// runs between the projection and this step; a -1 slot zeroes its conv output
// and leaves every state alone), with the arithmetic of gdn_conv1d_update, so
// the two launches and the fused one agree bit for bit.
//
// Layout of one block (request, head, PB-column slab of the state): warp w owns
// the key rows [w*RPW, (w+1)*RPW) and lane l the columns [l*CPL, (l+1)*CPL), so
// each row is one coalesced warp access.  S^T k and S^T q are sums over the
// warps: each warp leaves its partial sums in shared memory and, after ONE
// barrier, every thread adds the eight partials of its own columns (the
// partials alternate between two buffers, so the next sum needs no second
// barrier to protect this one's reads).
// The state is read once and written once: 2*N*P*4 bytes per (request, head),
// the HBM traffic that bounds the kernel.  Both go with streaming cache hints
// (evict first: the slab is touched once per step, so it should not push the rows
// and gates out of L2), and the plain form keeps to 48 registers so that five
// blocks, five 32 KB slabs, are in flight per SM.
#pragma once

#include "common.cuh"
#include "conv1d.cuh"

namespace gdn {
namespace dec {

constexpr int kWarps = 8;
constexpr int kMaxM = 8;

// Short-convolution inputs of the fused form.  The whole row is convolved:
// channel c of request r reads x[r, c] and the window cstate[slot, c, 0..W-2]
// (oldest first) and leaves the window shifted by one.  Value channels belong to
// one block each, which updates their windows; a key or query channel is read
// by every block of its GQA group (H/G heads x P/PB slabs), and the last of
// them to finish reading (counted in cnt[r, group], which it resets) updates it.
struct ConvIn {
    const float* w;             // [C, W]
    const float* bias;          // [C] or null
    __nv_bfloat16* cstate;      // [n_slots, C, W-1] bf16
    int32_t* cnt;               // [n, G], zero between calls
    int W;
    int act;                    // 1: SiLU
};

// One channel of the short convolution (the order of gdn_conv1d_update's
// arithmetic), rounded to bf16 like its output; returned widened to fp32.
__device__ __forceinline__ float conv_channel(const ConvIn& cv, const __nv_bfloat16* xr,
                                              int64_t slot, int64_t C, int64_t ch) {
    const int H = cv.W - 1;
    float acc = cv.bias ? cv.bias[ch] : 0.f;
    const __nv_bfloat16* win = cv.cstate + (slot * C + ch) * H;
    const float* w = cv.w + ch * cv.W;
    if (H == 3 && (reinterpret_cast<uintptr_t>(cv.w) & 15u) == 0) {
        // W = 4: the channel's taps are one 16-byte load (same products, same order)
        const float4 t = *reinterpret_cast<const float4*>(w);
        const float w0 = __bfloat162float(win[0]), w1 = __bfloat162float(win[1]),
                    w2 = __bfloat162float(win[2]), xc = __bfloat162float(xr[ch]);
        acc = fmaf(t.x, w0, acc);
        acc = fmaf(t.y, w1, acc);
        acc = fmaf(t.z, w2, acc);
        acc = fmaf(t.w, xc, acc);
        if (cv.act) acc = conv_silu(acc);
        return __bfloat162float(__float2bfloat16_rn(acc));
    }
    for (int i = 0; i < H; ++i) acc = fmaf(w[i], __bfloat162float(win[i]), acc);
    acc = fmaf(w[H], __bfloat162float(xr[ch]), acc);
    if (cv.act) acc = conv_silu(acc);
    return __bfloat162float(__float2bfloat16_rn(acc));
}

// The window of channel ch after this token: [old_1 .. old_{W-2}, x].
__device__ __forceinline__ void conv_shift(const ConvIn& cv, const __nv_bfloat16* xr, int64_t slot,
                                           int64_t C, int64_t ch) {
    const int H = cv.W - 1;
    __nv_bfloat16* win = cv.cstate + (slot * C + ch) * H;
    for (int i = 0; i + 1 < H; ++i) win[i] = win[i + 1];
    if (H > 0) win[H - 1] = xr[ch];
}

template <int N, int P, int PB, bool FUSED>
__global__ void __launch_bounds__(256, (PB <= 64 ? (FUSED ? 4 : 5) : 2)) step_kernel(
    const __nv_bfloat16* __restrict__ x, int64_t xs, const __nv_bfloat16* __restrict__ ba,
    int64_t bas, const float* __restrict__ A_log, const float* __restrict__ dt_bias, int M, int H,
    int G, float* __restrict__ state, const int32_t* __restrict__ state_idx, int n_slots,
    __nv_bfloat16* __restrict__ o, float scale, int l2, const ConvIn cv) {
    constexpr int RPW = N / kWarps;  // key rows per warp
    constexpr int CPL = PB / 32;     // value columns per lane
    constexpr int NPART = P / PB;
    static_assert(RPW >= 1 && CPL >= 1 && CPL <= 4 && P % PB == 0, "decode tile");
    __shared__ float kv[kMaxM][N];
    __shared__ float qv[N];
    __shared__ float vv[kMaxM][PB];
    __shared__ float red[2][kWarps][PB];
    __shared__ float gate_b[kMaxM];
    __shared__ float gate_e;
    __shared__ int last_reader;

    const int rh = blockIdx.x / NPART;               // request * H + head
    const int p0 = (blockIdx.x - rh * NPART) * PB;   // first value column of the slab
    const int r = rh / H, h = rh - r * H;
    const int hpg = H / G, grp = h / hpg;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const __nv_bfloat16* xr = x + (int64_t)r * xs;
    const __nv_bfloat16* br = ba + (int64_t)r * bas;
    const int64_t kbase = (int64_t)M * H * P, qbase = kbase + (int64_t)M * G * N;
    const int64_t C = qbase + (int64_t)G * N;  // channels of the row
    const int slot = state_idx ? state_idx[r] : r;
    if (slot < 0 || slot >= n_slots) {  // padding (uniform across the block)
        if (slot >= n_slots && threadIdx.x == 0) record_status(GDN_ERR_INVALID_ARG);
        if (threadIdx.x < PB) o[(int64_t)rh * P + p0 + threadIdx.x] = __float2bfloat16_rn(0.f);
        return;
    }

    // 1. the state loads (the only large traffic): first thing in the plain form,
    //    after the convolution in the fused form (so the convolution's registers
    //    and the state's are not live together, and four blocks still fit per SM)
    float* st = state + ((int64_t)slot * H + h) * N * P + p0 + lane * CPL;
    float s[RPW][CPL];
    auto load_state = [&]() {
#pragma unroll
        for (int rr = 0; rr < RPW; ++rr) {
            const float* src = st + (int64_t)(warp * RPW + rr) * P;
            if constexpr (CPL == 4) {
                const float4 t = *reinterpret_cast<const float4*>(src);
                s[rr][0] = t.x; s[rr][1] = t.y; s[rr][2] = t.z; s[rr][3] = t.w;
            } else if constexpr (CPL == 2) {
                const float2 t = __ldcs(reinterpret_cast<const float2*>(src));
                s[rr][0] = t.x; s[rr][1] = t.y;
            } else {
                s[rr][0] = src[0];
            }
        }
    };
    if constexpr (!FUSED) load_state();

    // 2. the block's inputs: values of its slab, keys and query of its group
    //    (conv outputs in the fused form), normalised, and the gates
    auto chan = [&](int64_t ch) -> float {
        if constexpr (FUSED)
            return conv_channel(cv, xr, slot, C, ch);
        else
            return __bfloat162float(xr[ch]);
    };
    if constexpr (FUSED) {
        // the convolution of every channel the block reads, spread over all its
        // threads (their loads in flight together), into the staging arrays
        for (int i = threadIdx.x; i < (M + 1) * N; i += blockDim.x) {
            const int m = i / N, j = i - m * N;
            const int64_t ch = (m < M) ? kbase + ((int64_t)m * G + grp) * N + j
                                       : qbase + (int64_t)grp * N + j;
            ((m < M) ? kv[m] : qv)[j] = chan(ch);
        }
        for (int i = threadIdx.x; i < M * PB; i += blockDim.x) {
            const int m = i / PB, j = i - m * PB;
            const int64_t ch = ((int64_t)m * H + h) * P + p0 + j;
            vv[m][j] = chan(ch);
            conv_shift(cv, xr, slot, C, ch);  // this block's own channel
        }
        load_state();
        __syncthreads();
    }
    for (int m = warp; m <= M; m += kWarps) {
        const int64_t base = (m < M) ? kbase + ((int64_t)m * G + grp) * N : qbase + (int64_t)grp * N;
        float* row = (m < M) ? kv[m] : qv;
        float e[N / 32];
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < N / 32; ++i) {
            if constexpr (FUSED)
                e[i] = row[lane + 32 * i];
            else
                e[i] = chan(base + lane + 32 * i);
            ss = fmaf(e[i], e[i], ss);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        const float inv = l2 ? 1.0f / sqrtf(ss + 1e-6f) : 1.0f;
#pragma unroll
        for (int i = 0; i < N / 32; ++i) row[lane + 32 * i] = e[i] * inv;
    }
    if constexpr (!FUSED) {
        for (int i = threadIdx.x; i < M * PB; i += blockDim.x) {
            const int m = i / PB, j = i - m * PB;
            vv[m][j] = chan(((int64_t)m * H + h) * P + p0 + j);
        }
    }
    if (threadIdx.x < M) gate_b[threadIdx.x] = write_gate(__bfloat162float(br[threadIdx.x * H + h]));
    if (threadIdx.x == M)
        gate_e = __double2float_rn(
            exp((double)decay_gate(__bfloat162float(br[M * H + h]), dt_bias[h], A_log[h])));
    __syncthreads();

    // sum over the eight warps of each thread's column partials, one barrier
    // (buffer b alternates between consecutive sums)
    auto warp_sum = [&](float (&d)[CPL], int b) {
#pragma unroll
        for (int c = 0; c < CPL; ++c) red[b][warp][lane * CPL + c] = d[c];
        __syncthreads();
#pragma unroll
        for (int c = 0; c < CPL; ++c) d[c] = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w)
#pragma unroll
            for (int c = 0; c < CPL; ++c) d[c] += red[b][w][lane * CPL + c];
    };

    // 3. the rule over the copies (decay on copy 0 only)
    for (int m = 0; m < M; ++m) {
        if (m == 0) {
            const float e0 = gate_e;
#pragma unroll
            for (int rr = 0; rr < RPW; ++rr)
#pragma unroll
                for (int c = 0; c < CPL; ++c) s[rr][c] *= e0;
        }
        float d[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c) d[c] = 0.f;
#pragma unroll
        for (int rr = 0; rr < RPW; ++rr) {
            const float kk = kv[m][warp * RPW + rr];
#pragma unroll
            for (int c = 0; c < CPL; ++c) d[c] = fmaf(s[rr][c], kk, d[c]);
        }
        warp_sum(d, m & 1);
        const float bm = gate_b[m];
#pragma unroll
        for (int c = 0; c < CPL; ++c) d[c] = bm * (vv[m][lane * CPL + c] - d[c]);
#pragma unroll
        for (int rr = 0; rr < RPW; ++rr) {
            const float kk = kv[m][warp * RPW + rr];
#pragma unroll
            for (int c = 0; c < CPL; ++c) s[rr][c] = fmaf(kk, d[c], s[rr][c]);
        }
    }

    // 4. the state back in place, then o = scale * S^T q
#pragma unroll
    for (int rr = 0; rr < RPW; ++rr) {
        float* dst = st + (int64_t)(warp * RPW + rr) * P;
        if constexpr (CPL == 4) {
            *reinterpret_cast<float4*>(dst) = make_float4(s[rr][0], s[rr][1], s[rr][2], s[rr][3]);
        } else if constexpr (CPL == 2) {
            __stcs(reinterpret_cast<float2*>(dst), make_float2(s[rr][0], s[rr][1]));
        } else {
            dst[0] = s[rr][0];
        }
    }
    float d[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) d[c] = 0.f;
#pragma unroll
    for (int rr = 0; rr < RPW; ++rr) {
        const float qq = qv[warp * RPW + rr];
#pragma unroll
        for (int c = 0; c < CPL; ++c) d[c] = fmaf(s[rr][c], qq, d[c]);
    }
    warp_sum(d, M & 1);
    if (warp == 0) {
#pragma unroll
        for (int c = 0; c < CPL; ++c)
            o[(int64_t)rh * P + p0 + lane * CPL + c] = __float2bfloat16_rn(scale * d[c]);
    }

    if constexpr (FUSED) {
        // every block of the group has read the key / query windows (long before
        // this point) once the counter reaches hpg * NPART; the block that takes
        // it there shifts them.  The count is an acquire-release add, so each
        // block's reads come before the last block's writes.
        const int readers = hpg * NPART;
        if (readers > 1) {
            if (threadIdx.x == 0) {
                int32_t* cp = cv.cnt + (int64_t)r * G + grp;
                int old;
                asm volatile("atom.add.acq_rel.gpu.s32 %0, [%1], 1;" : "=r"(old) : "l"(cp) : "memory");
                const int last = old == readers - 1;
                if (last) *cp = 0;  // no other block touches it again in this call
                last_reader = last;
            }
            __syncthreads();
        }
        if (readers == 1 || last_reader)
            for (int i = threadIdx.x; i < (M + 1) * N; i += blockDim.x) {
                const int m = i / N, j = i - m * N;
                const int64_t ch = (m < M) ? kbase + ((int64_t)m * G + grp) * N + j
                                           : qbase + (int64_t)grp * N + j;
                conv_shift(cv, xr, slot, C, ch);
            }
    }
}

}  // namespace dec
}  // namespace gdn
