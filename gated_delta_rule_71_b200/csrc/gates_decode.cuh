// gates_decode.cuh -- gate preparation and the Gated Delta Product decode step.
//
// Gates: Megatron-Core "core.ssm.ops.gdp.decode_prepare", module description and
// the `softplus` entry.  Decode layout: the `gdp_decode_prepare` function entry
// (post-conv row [value | key | query], ba row [b | a], outputs [n, M, H, *]).
// The state update is the gated delta rule run over the M Householder copies.
#pragma once

#include "common.cuh"

namespace gdn {

// ---------------------------------------------------------------- gate prep
// Elementwise over [n_tok, H]; grid-stride.  HBM-bound (16 B in, 8 B out per
// element), negligible next to the chunked pass.
__global__ void __launch_bounds__(256) gate_prep_kernel(const float* __restrict__ a,
                                                        const float* __restrict__ b,
                                                        int64_t n_tok, int H, int64_t a_stride,
                                                        int64_t b_stride,
                                                        const float* __restrict__ A_log,
                                                        const float* __restrict__ dt_bias,
                                                        float* __restrict__ beta,
                                                        float* __restrict__ g) {
    const int64_t total = n_tok * H;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / H;
        const int h = (int)(i - t * H);
        g[i] = decay_gate(a[t * a_stride + h], dt_bias[h], A_log[h]);
        beta[i] = write_gate(b[t * b_stride + h]);
    }
}

// ------------------------------------------------------------- decode prepare
// One block per (request, Householder copy).  Copies move in 16-byte units when
// every source/destination offset is 16-byte aligned (VEC), else per element.
template <bool VEC>
__global__ void __launch_bounds__(256) gdp_prepare_kernel(
    const __nv_bfloat16* __restrict__ x, int64_t xs, const __nv_bfloat16* __restrict__ ba,
    int64_t bas, const float* __restrict__ A_log, const float* __restrict__ dt_bias, int M, int H,
    int G, int P, int N, __nv_bfloat16* __restrict__ q, __nv_bfloat16* __restrict__ k,
    __nv_bfloat16* __restrict__ v, float* __restrict__ beta, float* __restrict__ g) {
    const int r = blockIdx.x, m = blockIdx.y;
    const int hpg = H / G;
    const __nv_bfloat16* xr = x + (int64_t)r * xs;
    const __nv_bfloat16* br = ba + (int64_t)r * bas;
    const int64_t kbase = (int64_t)M * H * P, qbase = kbase + (int64_t)M * G * N;
    const int64_t orow = (int64_t)r * M + m;  // [n, M] row of every output
    using U = typename std::conditional<VEC, uint4, uint16_t>::type;
    constexpr int E = sizeof(U) / 2;  // bf16 elements per unit
    // value: the H*P slab of copy m is contiguous in x and in v
    {
        const U* src = reinterpret_cast<const U*>(xr + (int64_t)m * H * P);
        U* dst = reinterpret_cast<U*>(v + orow * H * P);
        for (int i = threadIdx.x; i < H * P / E; i += blockDim.x) dst[i] = src[i];
    }
    // key and query: head h reads group h / hpg
    const int nN = N / E;
    for (int i = threadIdx.x; i < H * nN; i += blockDim.x) {
        const int h = i / nN, c = i - h * nN, grp = h / hpg;
        const U* ks = reinterpret_cast<const U*>(xr + kbase + ((int64_t)m * G + grp) * N);
        reinterpret_cast<U*>(k + (orow * H + h) * N)[c] = ks[c];
        U qv;
        if (m == M - 1) {
            qv = reinterpret_cast<const U*>(xr + qbase + (int64_t)grp * N)[c];
        } else {
            memset(&qv, 0, sizeof(U));
        }
        reinterpret_cast<U*>(q + (orow * H + h) * N)[c] = qv;
    }
    for (int h = threadIdx.x; h < H; h += blockDim.x) {
        beta[orow * H + h] = write_gate(__bfloat162float(br[m * H + h]));
        g[orow * H + h] =
            (m == 0) ? decay_gate(__bfloat162float(br[M * H + h]), dt_bias[h], A_log[h]) : 0.0f;
    }
}

// ---------------------------------------------------------------- decode step
// One block (8 warps) per (request, head).  The request's state sits in slot
// state_idx[r] of the state pool (slot r when state_idx is NULL); a negative
// slot is a padding request: o = 0 and its state is neither read nor written
// (Megatron-Core "core.ssm.ops.gdp.decode_prepare", module description: the
// batch is padded upstream with -1 slots).  A slot >= n_slots is handled the
// same way and records GDN_ERR_INVALID_ARG in the device status word.  The
// value columns of the state never interact, so a (request, head) is split
// over P / PB blocks of PB columns each (smaller blocks: more of them resident
// per SM to overlap one block's loads with another's arithmetic).  The block's
// fp32 state slab [N, PB] lives in registers: warp w owns key rows
// [w*N/8, (w+1)*N/8), lane l owns columns [l*PB/32, (l+1)*PB/32), so every row
// is read and written as one coalesced warp access.  Column reductions over the key
// axis go through shared memory.  The state is read once and written once:
// the kernel is HBM-bound on 2*N*P*4 bytes per (request, head).
constexpr int kDecWarps = 8;
constexpr int kDecMaxM = 8;

template <int N, int P, int PB>
__global__ void __launch_bounds__(256, (PB <= 64 ? 4 : 2)) gdp_step_kernel(
    const __nv_bfloat16* __restrict__ x, int64_t xs, const __nv_bfloat16* __restrict__ ba,
    int64_t bas, const float* __restrict__ A_log, const float* __restrict__ dt_bias, int M, int H,
    int G, float* __restrict__ state, const int32_t* __restrict__ state_idx, int n_slots,
    __nv_bfloat16* __restrict__ o, float scale, int l2) {
    constexpr int RPW = N / kDecWarps;  // rows per warp
    constexpr int CPL = PB / 32;        // columns per lane
    constexpr int NPART = P / PB;
    __shared__ float kv[kDecMaxM][N];
    __shared__ float vv[kDecMaxM][PB];
    __shared__ float qv[N];
    __shared__ float red[kDecWarps][PB];
    __shared__ float uu[PB];
    __shared__ float gate_b[kDecMaxM];
    __shared__ float gate_e;

    const int rh = blockIdx.x / NPART;  // request * H + head
    const int p0 = (blockIdx.x - rh * NPART) * PB;  // first value column of this block
    const int r = rh / H, h = rh - r * H;
    const int hpg = H / G, grp = h / hpg;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const __nv_bfloat16* xr = x + (int64_t)r * xs;
    const __nv_bfloat16* br = ba + (int64_t)r * bas;
    const int64_t kbase = (int64_t)M * H * P, qbase = kbase + (int64_t)M * G * N;
    const int slot = state_idx ? state_idx[r] : r;
    if (slot < 0 || slot >= n_slots) {  // padding (uniform across the block)
        if (slot >= n_slots && threadIdx.x == 0) record_status(GDN_ERR_INVALID_ARG);
        if (threadIdx.x < PB) o[(int64_t)rh * P + p0 + threadIdx.x] = __float2bfloat16_rn(0.f);
        return;
    }

    // 1. issue the state loads first (the only large traffic)
    float* st = state + ((int64_t)slot * H + h) * N * P + p0;
    float s[RPW][CPL];
#pragma unroll
    for (int rr = 0; rr < RPW; ++rr) {
        const float* src = st + (int64_t)(warp * RPW + rr) * P + lane * CPL;
        if constexpr (CPL == 4) {
            float4 t = *reinterpret_cast<const float4*>(src);
            s[rr][0] = t.x; s[rr][1] = t.y; s[rr][2] = t.z; s[rr][3] = t.w;
        } else if constexpr (CPL == 2) {
            float2 t = *reinterpret_cast<const float2*>(src);
            s[rr][0] = t.x; s[rr][1] = t.y;
        } else {
            s[rr][0] = src[0];
        }
    }

    // 2. split / GQA-expand / normalise the M copies and the query into smem
    for (int m = warp; m <= M; m += kDecWarps) {
        const __nv_bfloat16* src = (m < M) ? xr + kbase + ((int64_t)m * G + grp) * N
                                           : xr + qbase + (int64_t)grp * N;
        float e[N / 32];
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < N / 32; ++i) {
            e[i] = __bfloat162float(src[lane + 32 * i]);
            ss = fmaf(e[i], e[i], ss);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        const float inv = l2 ? 1.0f / sqrtf(ss + 1e-6f) : 1.0f;
        float* dst = (m < M) ? kv[m] : qv;
#pragma unroll
        for (int i = 0; i < N / 32; ++i) dst[lane + 32 * i] = e[i] * inv;
    }
    for (int i = threadIdx.x; i < M * PB; i += blockDim.x) {
        const int m = i / PB, j = i - m * PB;
        vv[m][j] = __bfloat162float(xr[((int64_t)m * H + h) * P + p0 + j]);
    }
    if (threadIdx.x < M) gate_b[threadIdx.x] = write_gate(__bfloat162float(br[threadIdx.x * H + h]));
    if (threadIdx.x == M)
        gate_e = __double2float_rn(
            exp((double)decay_gate(__bfloat162float(br[M * H + h]), dt_bias[h], A_log[h])));
    __syncthreads();

    // 3. the rule over the copies (decay on copy 0 only)
    for (int m = 0; m < M; ++m) {
        if (m == 0) {
            const float e0 = gate_e;
#pragma unroll
            for (int rr = 0; rr < RPW; ++rr)
#pragma unroll
                for (int c = 0; c < CPL; ++c) s[rr][c] *= e0;
        }
        float pp[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c) pp[c] = 0.f;
#pragma unroll
        for (int rr = 0; rr < RPW; ++rr) {
            const float kk = kv[m][warp * RPW + rr];
#pragma unroll
            for (int c = 0; c < CPL; ++c) pp[c] = fmaf(s[rr][c], kk, pp[c]);
        }
#pragma unroll
        for (int c = 0; c < CPL; ++c) red[warp][lane * CPL + c] = pp[c];
        __syncthreads();
        if (threadIdx.x < PB) {
            float d = 0.f;
#pragma unroll
            for (int w = 0; w < kDecWarps; ++w) d += red[w][threadIdx.x];
            uu[threadIdx.x] = gate_b[m] * (vv[m][threadIdx.x] - d);
        }
        __syncthreads();
        float u[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c) u[c] = uu[lane * CPL + c];
#pragma unroll
        for (int rr = 0; rr < RPW; ++rr) {
            const float kk = kv[m][warp * RPW + rr];
#pragma unroll
            for (int c = 0; c < CPL; ++c) s[rr][c] = fmaf(kk, u[c], s[rr][c]);
        }
    }

    // 4. write the state back in place, then the output at the last copy
#pragma unroll
    for (int rr = 0; rr < RPW; ++rr) {
        float* dst = st + (int64_t)(warp * RPW + rr) * P + lane * CPL;
        if constexpr (CPL == 4) {
            *reinterpret_cast<float4*>(dst) = make_float4(s[rr][0], s[rr][1], s[rr][2], s[rr][3]);
        } else if constexpr (CPL == 2) {
            *reinterpret_cast<float2*>(dst) = make_float2(s[rr][0], s[rr][1]);
        } else {
            dst[0] = s[rr][0];
        }
    }
    {
        float pp[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c) pp[c] = 0.f;
#pragma unroll
        for (int rr = 0; rr < RPW; ++rr) {
            const float qq = qv[warp * RPW + rr];
#pragma unroll
            for (int c = 0; c < CPL; ++c) pp[c] = fmaf(s[rr][c], qq, pp[c]);
        }
#pragma unroll
        for (int c = 0; c < CPL; ++c) red[warp][lane * CPL + c] = pp[c];
        __syncthreads();
        if (threadIdx.x < PB) {
            float d = 0.f;
#pragma unroll
            for (int w = 0; w < kDecWarps; ++w) d += red[w][threadIdx.x];
            o[(int64_t)rh * P + p0 + threadIdx.x] = __float2bfloat16_rn(scale * d);
        }
    }
}

}  // namespace gdn

namespace gdn {

// --------------------------------------------------------------- GDP prefill
// The prefill runs the rule over the copy-interleaved sequence that
// gdp_decode_prepare builds from T token rows (T*M rows, copy-minor), so the
// packed-batch offsets scale by M and each token's output is the one at its
// last copy.
__global__ void gdp_scale_offsets_kernel(const int32_t* __restrict__ cu, int n, int M,
                                         int32_t* __restrict__ out) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i <= n; i += gridDim.x * blockDim.x)
        out[i] = cu[i] * M;
}

// o[r] = o_all[r*M + M-1] for rows of `row_units` 16-byte units.
__global__ void __launch_bounds__(256) gdp_last_copy_kernel(const uint4* __restrict__ o_all,
                                                            int64_t rows, int M,
                                                            int64_t row_units,
                                                            uint4* __restrict__ o) {
    const int64_t total = rows * row_units;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / row_units, u = i - r * row_units;
        o[i] = o_all[(r * M + M - 1) * row_units + u];
    }
}

}  // namespace gdn

namespace gdn {

// ------------------------------------------------------- context parallelism
// out[i] = A[i] X[i] + C[i] for a batch of (K x K) . (K x V) fp32 products: the
// state entering a sequence segment from the previous segment's transition
// matrix, incoming state and local final state.  One block per (matrix, 32
// output columns); the K x 32 slab of X and 32-row panels of A go through
// shared memory.  Small next to the chunked passes it joins.
template <int K>
__global__ void __launch_bounds__(256) state_combine_kernel(const float* __restrict__ A,
                                                            const float* __restrict__ X,
                                                            const float* __restrict__ Cm,
                                                            float* __restrict__ out, int V) {
    __shared__ float xs[K][33];
    __shared__ float as[32][K + 1];
    const int i = blockIdx.y, c0 = 32 * blockIdx.x;
    const int64_t aoff = (int64_t)i * K * K, xoff = (int64_t)i * K * V;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 8 row groups
    for (int e = threadIdx.x; e < K * 32; e += 256) {
        const int r = e >> 5, c = e & 31;
        xs[r][c] = (c0 + c < V) ? X[xoff + (int64_t)r * V + c0 + c] : 0.f;
    }
    for (int rp = 0; rp < K; rp += 32) {
        __syncthreads();
        for (int e = threadIdx.x; e < 32 * K; e += 256) {
            const int r = e / K, kk = e - r * K;
            as[r][kk] = A[aoff + (int64_t)(rp + r) * K + kk];
        }
        __syncthreads();
        for (int r = ty; r < 32; r += 8) {
            float acc = 0.f;
#pragma unroll 8
            for (int kk = 0; kk < K; ++kk) acc = fmaf(as[r][kk], xs[kk][tx], acc);
            const int row = rp + r, col = c0 + tx;
            if (col < V) {
                const int64_t o = xoff + (int64_t)row * V + col;
                out[o] = acc + (Cm ? Cm[o] : 0.f);
            }
        }
    }
}

// y[i] += x[i] (fp32), grid-stride.
__global__ void __launch_bounds__(256) accumulate_f32_kernel(float* __restrict__ y,
                                                             const float* __restrict__ x,
                                                             int64_t n) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x)
        y[i] += x[i];
}

}  // namespace gdn
