// gates_decode.cuh -- gate preparation, the decode prepare and the CP helpers.
//
// Gates: Megatron-Core "core.ssm.ops.gdp.decode_prepare", module description and
// the `softplus` entry.  Decode layout: the `gdp_decode_prepare` function entry
// (post-conv row [value | key | query], ba row [b | a], outputs [n, M, H, *]).
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

// The decode step itself is in decode_step.cuh.

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
