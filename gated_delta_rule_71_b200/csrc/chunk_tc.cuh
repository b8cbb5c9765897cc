// chunk_tc.cuh -- fused tensor-core chunked forward of the gated delta rule
// (bf16 q/k/v, K = V = 128, fp32 state, fp32 accumulation), sm_100a.
//
// One CTA owns one (sequence, head, 64-wide value slice) and walks its chunks
// in order; the three steps of ZzCompute (PyTorch Helion Hackathon gallery
// entry 11) -- item 4 "Recompute W/U" (in-chunk cumsum, A, T = (I+A)^-1),
// item 2 "Chunk Forward H" (state recurrence) and item 3 "Chunk Forward O"
// (chunk output) -- run in one kernel so q/k/v/g/beta are read from HBM once and
// o/h_T written once.  Per chunk (64 tokens, G2 = log2-scaled cumsum of g):
//   S    = [K; Q] K^T                               (MMA, M=128 N=64 K=128)
//   A    = strictly-lower beta_r 2^(G2_r-G2_s) (K K^T)_rs,  T = (I + A)^-1 (SIMT fp32)
//   P    = lower-incl 2^(G2_r-G2_s) (Q K^T)_rs                              (SIMT)
//   [KH; QH] = [K; Q] h                             (MMA, B = bf16 copy of h)
//   R    = beta (V - 2^G2 * KH)                                        (SIMT)
//   Ut   = T R             ( = U - W h of the WY form)  (MMA, A = [T; P])
//   h'   = 2^G2_L h + K^T (2^(G2_L-G2) * Ut)            (MMA, then fp32 update)
//   O    = scale (2^G2 * QH + P Ut)                      (MMA, A = [T; P])
// Warp roles (384 threads): warp 0 issues TMA loads into a 2-stage ring and
// owns tensor memory; warps 4-7 ("prep") build A, T and P for each chunk one
// chunk ahead; warps 8-11 ("chain") carry the fp32 state in registers through
// the serial part and write the output.  Every MMA is issued by one thread of
// the warpgroup that consumes it, with completion signalled on an mbarrier.
// Every wait is bounded: a wait that gives up sets an abort flag (all later
// waits fall through, so every named barrier is still reached) and records
// GDN_ERR_TIMEOUT in the device status word.
#pragma once

#include <cudaTypedefs.h>

#include "chunk_simt.cuh"
#include "tc_ptx.cuh"

namespace gdn {

constexpr bool kTcAvailable = true;

namespace tcf {

constexpr int C = 64;    // chunk
constexpr int KD = 128;  // key dim
constexpr int VD = 128;  // value dim
constexpr int VS = 64;   // value slice per CTA
constexpr int kThreads = 384;
constexpr uint32_t kPolls = 1u << 22;
constexpr float kLog2e = 1.4426950408889634f;

// shared memory (byte offsets from a 1024-aligned base)
constexpr uint32_t SZ_KQ = 32768;  // [2 key halves][K rows 0-63 | Q rows 64-127][128 B]
constexpr uint32_t SZ_V = 8192;    // [64 rows][64 bf16]
constexpr uint32_t SZ_TP = 16384;  // [T rows 0-63 | P rows 64-127][64 bf16]
constexpr uint32_t OFF_KQ = 0;
constexpr uint32_t OFF_V = OFF_KQ + 2 * SZ_KQ;
constexpr uint32_t OFF_TP = OFF_V + 2 * SZ_V;
constexpr uint32_t OFF_HB = OFF_TP + 2 * SZ_TP;  // h bf16 [128 key rows][64 v]
constexpr uint32_t OFF_RB = OFF_HB + 16384;      // R  [64 rows][64 v]
constexpr uint32_t OFF_UB = OFF_RB + 8192;       // Ut
constexpr uint32_t OFF_WB = OFF_UB + 8192;       // 2^(G2_L-G2) Ut
constexpr int AFP = 68;                          // fp32 row pitch of A / T
constexpr uint32_t OFF_AF = OFF_WB + 8192;
constexpr uint32_t OFF_TF = OFF_AF + 64 * AFP * 4;
constexpr int XTP = 24;  // pitch of the 16x16 temporaries (conflict-free B fragments)
constexpr uint32_t OFF_XT = OFF_TF + 64 * AFP * 4;  // fp32 [3][16][20]
struct Scal {
    float G2[64];    // in-chunk inclusive cumsum of g, log2 units
    float beta[64];
    float gam[64];   // 2^G2
    float w[64];     // 2^(G2_L - G2)
    float ginv[64];  // 2^-G2 (only when the chunk's decay stays in fp32 range)
    float eGL;       // 2^G2_L
    float pad[3];
};
constexpr int OSP = 68;                              // fp32 row pitch of the output stage
constexpr uint32_t OFF_OS = OFF_XT + 3 * 16 * XTP * 4;   // fp32 [64][68] output rows
constexpr uint32_t OFF_SC = OFF_OS + 64 * OSP * 4;
constexpr uint32_t OFF_BAR = OFF_SC + 2 * sizeof(Scal);
constexpr uint32_t OFF_MISC = OFF_BAR + 16 * 8;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 64 + 1024;

// tensor memory columns (fp32 accumulators, 128 lanes each)
constexpr uint32_t COL_S = 0;
constexpr uint32_t COL_H = 64;   // two buffers
constexpr uint32_t COL_U = 192;
constexpr uint32_t COL_D = 256;
constexpr uint32_t COL_O = 320;  // two buffers
constexpr uint32_t TMEM_COLS = 512;

struct Params {
    CUtensorMap tm_q, tm_k, tm_v;
    const float* g;
    const float* beta;
    const float* h0;
    const int32_t* cu;
    const int32_t* order;
    int64_t T;
    int H;
    float scale;
    void* o;
    float* hT;
};

// Bounded wait that honours the block's abort flag.
__device__ __forceinline__ bool wait(uint64_t* bar, uint32_t phase, volatile uint32_t* abort) {
    if (*abort) return false;
    const uint32_t a = smem_u32(bar);
    for (uint32_t i = 0; i < kPolls; ++i) {
        if (mbar_try_wait(a, phase)) return true;
        if ((i & 255u) == 255u && *abort) return false;
    }
    *abort = 1u;
    record_status(GDN_ERR_TIMEOUT);
    return false;
}

// 16x16x16 block product on one warp with the warp-level tf32 tensor-core MMA
// (m16n8k8, fp32 accumulate): C (+)= X Y for fp32 X, Y in shared memory (row
// pitches in floats).  tcgen05's smallest tile is 64 rows, so the 16x16
// blocks of the triangular inverse use this form.  Fragment layout (PTX ISA,
// mma.m16n8k8 .tf32): g = lane/4, t = lane%4; A: (g,t) (g+8,t) (g,t+4)
// (g+8,t+4); B: (t,g) (t+4,g); C: (g,2t) (g,2t+1) (g+8,2t) (g+8,2t+1).
__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mm16(float (&c)[2][4], const float* X, int xs, const float* Y,
                                     int ys, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
        const float* x = X + 8 * kk;
        uint32_t a[4] = {to_tf32(x[g * xs + t]), to_tf32(x[(g + 8) * xs + t]),
                         to_tf32(x[g * xs + t + 4]), to_tf32(x[(g + 8) * xs + t + 4])};
        const float* y = Y + 8 * kk * ys;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
            mma_tf32(c[nt], a, to_tf32(y[t * ys + 8 * nt + g]), to_tf32(y[(t + 4) * ys + 8 * nt + g]));
    }
}
__device__ __forceinline__ void mm16_store(const float (&c)[2][4], float* Z, int zs, int lane,
                                           float sign) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        *reinterpret_cast<float2*>(Z + g * zs + 8 * nt + 2 * t) =
            make_float2(sign * c[nt][0], sign * c[nt][1]);
        *reinterpret_cast<float2*>(Z + (g + 8) * zs + 8 * nt + 2 * t) =
            make_float2(sign * c[nt][2], sign * c[nt][3]);
    }
}

// T = (I + A)^-1 for the strictly lower 64x64 A (fp32, pitch AFP) by 16x16
// blocks: diagonal blocks by substitution in fp32, then the off-diagonal
// blocks by distance from the diagonal, T_ij = -T_ii sum_{j<=k<i} A_ik T_kj.
// Writes every T entry on or below the diagonal (diagonal blocks complete,
// with their zero upper halves).  Called by the 128 prep threads; uses
// named barrier 1.
__device__ __forceinline__ void invert_unit_lower(const float* Af, float* Tf, float* Xt, int pw,
                                                  int lane) {
    // diagonal blocks: warp pw owns block pw, lanes 0..15 one column each
    if (lane < 16) {
        const int o = 16 * pw, j = lane;
        float t[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
            for (int s = 0; s < r; s += 2) {
                acc0 = fmaf(Af[(o + r) * AFP + o + s], t[s], acc0);
                if (s + 1 < r) acc1 = fmaf(Af[(o + r) * AFP + o + s + 1], t[s + 1], acc1);
            }
            t[r] = (r < j) ? 0.f : ((r == j) ? 1.f : -(acc0 + acc1));
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) Tf[(o + r) * AFP + o + j] = t[r];
    }
    tc::named_bar(1, 128);
    // distance 1: blocks (1,0), (2,1), (3,2)
    if (pw < 3) {
        const int i = pw + 1, j = pw;
        float* X = Xt + pw * 16 * XTP;
        float c[2][4] = {};
        mm16(c, Af + 16 * i * AFP + 16 * j, AFP, Tf + 16 * j * AFP + 16 * j, AFP, lane);
        mm16_store(c, X, XTP, lane, 1.f);
        __syncwarp();
        float c2[2][4] = {};
        mm16(c2, Tf + 16 * i * AFP + 16 * i, AFP, X, XTP, lane);
        mm16_store(c2, Tf + 16 * i * AFP + 16 * j, AFP, lane, -1.f);
    }
    tc::named_bar(1, 128);
    // distance 2: blocks (2,0), (3,1)
    if (pw < 2) {
        const int i = pw + 2, j = pw;
        float* X = Xt + pw * 16 * XTP;
        float c[2][4] = {};
        mm16(c, Af + 16 * i * AFP + 16 * j, AFP, Tf + 16 * j * AFP + 16 * j, AFP, lane);
        mm16(c, Af + 16 * i * AFP + 16 * (j + 1), AFP, Tf + 16 * (j + 1) * AFP + 16 * j, AFP,
             lane);
        mm16_store(c, X, XTP, lane, 1.f);
        __syncwarp();
        float c2[2][4] = {};
        mm16(c2, Tf + 16 * i * AFP + 16 * i, AFP, X, XTP, lane);
        mm16_store(c2, Tf + 16 * i * AFP + 16 * j, AFP, lane, -1.f);
    }
    tc::named_bar(1, 128);
    // distance 3: block (3,0)
    if (pw == 0) {
        float* X = Xt;
        float c[2][4] = {};
        mm16(c, Af + 48 * AFP + 0, AFP, Tf + 0 * AFP + 0, AFP, lane);
        mm16(c, Af + 48 * AFP + 16, AFP, Tf + 16 * AFP + 0, AFP, lane);
        mm16(c, Af + 48 * AFP + 32, AFP, Tf + 32 * AFP + 0, AFP, lane);
        mm16_store(c, X, XTP, lane, 1.f);
        __syncwarp();
        float c2[2][4] = {};
        mm16(c2, Tf + 48 * AFP + 48, AFP, X, XTP, lane);
        mm16_store(c2, Tf + 48 * AFP + 0, AFP, lane, -1.f);
    }
    tc::named_bar(1, 128);
}

template <bool OBF16>
__global__ void __launch_bounds__(kThreads, 1) chunk_fwd_tc_kernel(const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t sbase = (raw_u32 + 1023u) & ~1023u;
    uint8_t* base = smem_raw + (sbase - raw_u32);

    uint64_t* bars = reinterpret_cast<uint64_t*>(base + OFF_BAR);
    uint64_t* full = bars + 0;
    uint64_t* empty = bars + 2;
    uint64_t* pfull = bars + 4;
    uint64_t* pempty = bars + 6;
    uint64_t* mS = bars + 8;
    uint64_t* mH = bars + 9;
    uint64_t* mU = bars + 10;
    uint64_t* mD = bars + 11;
    uint64_t* mO = bars + 12;
    uint64_t* mDrain = bars + 13;   // chain-side drain after an abort
    uint64_t* mDrainP = bars + 14;  // prep-side drain after an abort
    uint32_t* misc = reinterpret_cast<uint32_t*>(base + OFF_MISC);
    volatile uint32_t* abort_flag = misc + 1;
    float* scan_tmp = reinterpret_cast<float*>(misc + 2);
    Scal* SC = reinterpret_cast<Scal*>(base + OFF_SC);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int H = p.H;
    const int vsl = blockIdx.x & 1;
    const int sh = blockIdx.x >> 1;
    const int head = sh % H;
    const int slot = sh / H;
    const int seq = p.order ? p.order[slot] : slot;
    int64_t cs, ce;
    if (p.cu) {
        cs = p.cu[seq];
        ce = p.cu[seq + 1];
    } else {
        cs = (int64_t)seq * p.T;
        ce = cs + p.T;
    }
    const int nch = (int)((ce - cs + C - 1) / C);
    const int v0 = vsl * VS;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 2);
            mbar_init(&pfull[i], 1);
            mbar_init(&pempty[i], 64);
        }
        mbar_init(mS, 1);
        mbar_init(mH, 1);
        mbar_init(mU, 1);
        mbar_init(mD, 1);
        mbar_init(mO, 1);
        mbar_init(mDrain, 1);
        mbar_init(mDrainP, 1);
        misc[1] = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) tc::tmem_alloc(&misc[0], TMEM_COLS);
    tc::tc_before_sync();
    __syncthreads();
    tc::tc_after_sync();
    const uint32_t tmem = misc[0];

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            tc::prefetch_tmap(&p.tm_q);
            tc::prefetch_tmap(&p.tm_k);
            tc::prefetch_tmap(&p.tm_v);
            for (int c = 0; c < nch; ++c) {
                const int s = c & 1;
                if (c >= 2) wait(&empty[s], ((c >> 1) + 1) & 1, abort_flag);
                tc::mbar_arrive_expect_tx(&full[s], SZ_KQ + SZ_V);
                const int y = (int)(cs + (int64_t)C * c);
                uint8_t* kq = base + OFF_KQ + s * SZ_KQ;
                tc::tma_load_2d(kq + 0, &p.tm_k, head * KD + 0, y, &full[s]);
                tc::tma_load_2d(kq + 8192, &p.tm_q, head * KD + 0, y, &full[s]);
                tc::tma_load_2d(kq + 16384, &p.tm_k, head * KD + 64, y, &full[s]);
                tc::tma_load_2d(kq + 24576, &p.tm_q, head * KD + 64, y, &full[s]);
                tc::tma_load_2d(base + OFF_V + s * SZ_V, &p.tm_v, head * VD + v0, y, &full[s]);
            }
            // never leave with copies in flight
            for (int c = (nch > 2 ? nch - 2 : 0); c < nch; ++c) {
                const uint32_t a = smem_u32(&full[c & 1]);
                for (uint32_t i = 0; i < kPolls && !mbar_try_wait(a, (c >> 1) & 1); ++i) {
                }
            }
        }
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------------------- prep
        const int pt = threadIdx.x - 128, pw = warp - 4;
        float* Af = reinterpret_cast<float*>(base + OFF_AF);
        float* Tf = reinterpret_cast<float*>(base + OFF_TF);
        float* Xt = reinterpret_cast<float*>(base + OFF_XT);
        const uint32_t idS = tc::idesc_bf16(128, 64, 0, 0);
        for (int c = 0; c < nch; ++c) {
            const int s = c & 1, b = c & 1;
            const int64_t t0 = cs + (int64_t)C * c;
            const int len = (int)((ce - t0) < C ? (ce - t0) : C);
            float gv = 0.f, bv = 0.f;
            if (pt < len) {
                gv = p.g[(t0 + pt) * H + head];
                bv = p.beta[(t0 + pt) * H + head];
            }
            wait(&full[s], (c >> 1) & 1, abort_flag);
            const uint32_t kq = sbase + OFF_KQ + s * SZ_KQ;
            if (pt == 0) {
                tc::tc_after_sync();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    tc::mma_bf16(tmem + COL_S, tc::sdesc_sw128(kq + off, 16, 1024),
                                 tc::sdesc_sw128(kq + off, 16, 1024), idS, kk > 0);
                }
                tc::mma_commit(mS);
            }
            // in-chunk inclusive cumsum of g (log2 units) on warps 0-1
            float x = gv * kLog2e;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, x, off);
                if (lane >= off) x += y;
            }
            if (pt == 31) *scan_tmp = x;
            if (c >= 2) wait(&pempty[b], ((c >> 1) + 1) & 1, abort_flag);
            tc::named_bar(1, 128);
            if (pw == 1) x += *scan_tmp;
            Scal* sc = SC + b;
            if (pt < 64) {
                sc->G2[pt] = x;
                sc->beta[pt] = bv;
            }
            tc::named_bar(1, 128);
            const float G2L = sc->G2[63];
            // 2^(G2_r - G2_s) = 2^G2_r * 2^-G2_s whenever the chunk's total decay stays
            // above 2^-126 (no overflow or subnormal factor); else per element
            const bool factored = G2L > -126.f;
            if (pt < 64) {
                sc->gam[pt] = exp2f(x);
                sc->w[pt] = exp2f(G2L - x);
                sc->ginv[pt] = factored ? exp2f(-x) : 0.f;
            }
            if (pt == 0) sc->eGL = exp2f(G2L);
            // S row of this thread: rows 0-63 = K K^T, rows 64-127 = Q K^T
            wait(mS, c & 1, abort_flag);
            tc::tc_after_sync();
            float sv[64];
            {
                const uint32_t ta = tmem + ((uint32_t)(32 * pw) << 16) + COL_S;
                tc::tmem_ld32(ta, *reinterpret_cast<float(*)[32]>(sv));
                tc::tmem_ld32(ta + 32, *reinterpret_cast<float(*)[32]>(sv + 32));
                tc::tmem_wait_ld();
            }
            if (pt == 0) tc::mbar_arrive(&empty[s]);  // stage no longer read by prep
            const uint32_t tp = sbase + OFF_TP + b * SZ_TP;
            tc::named_bar(1, 128);  // ginv visible
            if (pt < 64) {
                const int r = pt;
                const float g2r = sc->G2[r], br = bv;
                float* arow = Af + r * AFP;
                if (factored) {
                    const float coef = br * sc->gam[r];
#pragma unroll
                    for (int j = 0; j < 64; j += 4) {
                        const float4 gi = *reinterpret_cast<const float4*>(sc->ginv + j);
                        float4 av;
                        av.x = (j + 0 < r) ? coef * gi.x * sv[j + 0] : 0.f;
                        av.y = (j + 1 < r) ? coef * gi.y * sv[j + 1] : 0.f;
                        av.z = (j + 2 < r) ? coef * gi.z * sv[j + 2] : 0.f;
                        av.w = (j + 3 < r) ? coef * gi.w * sv[j + 3] : 0.f;
                        *reinterpret_cast<float4*>(arow + j) = av;
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 64; j += 4) {
                        float4 av;
                        av.x = (j + 0 < r) ? br * exp2f(g2r - sc->G2[j + 0]) * sv[j + 0] : 0.f;
                        av.y = (j + 1 < r) ? br * exp2f(g2r - sc->G2[j + 1]) * sv[j + 1] : 0.f;
                        av.z = (j + 2 < r) ? br * exp2f(g2r - sc->G2[j + 2]) * sv[j + 2] : 0.f;
                        av.w = (j + 3 < r) ? br * exp2f(g2r - sc->G2[j + 3]) * sv[j + 3] : 0.f;
                        *reinterpret_cast<float4*>(arow + j) = av;
                    }
                }
            } else {
                const int r = pt - 64;
                const float g2r = sc->G2[r];
                if (factored) {
                    const float coef = sc->gam[r];
#pragma unroll
                    for (int j = 0; j < 64; j += 4) {
                        const float4 gi = *reinterpret_cast<const float4*>(sc->ginv + j);
                        sv[j + 0] = (j + 0 <= r) ? coef * gi.x * sv[j + 0] : 0.f;
                        sv[j + 1] = (j + 1 <= r) ? coef * gi.y * sv[j + 1] : 0.f;
                        sv[j + 2] = (j + 2 <= r) ? coef * gi.z * sv[j + 2] : 0.f;
                        sv[j + 3] = (j + 3 <= r) ? coef * gi.w * sv[j + 3] : 0.f;
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 64; ++j)
                        sv[j] = (j <= r) ? exp2f(g2r - sc->G2[j]) * sv[j] : 0.f;
                }
                tc::store_row_bf16(tp + 8192, r, sv);
            }
            tc::tc_before_sync();
            tc::named_bar(1, 128);
            invert_unit_lower(Af, Tf, Xt, pw, lane);
            {
                // T rows -> bf16 (upper part zero), two threads per row
                const int r = pt >> 1, hf = pt & 1;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const int ch = 4 * hf + q4;
                    float t8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int col = 8 * ch + e;
                        t8[e] = (col <= r) ? Tf[r * AFP + col] : 0.f;
                    }
                    tc::st_shared_v4(tp + tc::sw128_off(r, ch), tc::pack_bf16(t8[0], t8[1]),
                                     tc::pack_bf16(t8[2], t8[3]), tc::pack_bf16(t8[4], t8[5]),
                                     tc::pack_bf16(t8[6], t8[7]));
                }
            }
            tc::fence_async_smem();
            tc::named_bar(1, 128);
            if (pt == 0) tc::mbar_arrive(&pfull[b]);
        }
        if (pt == 0 && *abort_flag) {
            // drain any MMA still running before tensor memory is released
            tc::mma_commit(mDrainP);
            const uint32_t a = smem_u32(mDrainP);
            for (uint32_t i = 0; i < kPolls && !mbar_try_wait(a, 0); ++i) {
            }
        }
    } else if (warp >= 8) {
        // ------------------------------------------------------------ chain
        const int ct = threadIdx.x - 256, cw = warp - 8;
        const uint32_t lane_base = (uint32_t)(32 * cw) << 16;
        const int64_t hrow = ((int64_t)(seq * H + head) * KD + ct) * VD + v0;
        float h[64];
        if (p.h0) {
#pragma unroll
            for (int j = 0; j < 64; j += 4) {
                const float4 t = *reinterpret_cast<const float4*>(p.h0 + hrow + j);
                h[j] = t.x; h[j + 1] = t.y; h[j + 2] = t.z; h[j + 3] = t.w;
            }
        } else {
#pragma unroll
            for (int j = 0; j < 64; ++j) h[j] = 0.f;
        }
        const uint32_t hb = sbase + OFF_HB, rb = sbase + OFF_RB, ub = sbase + OFF_UB,
                       wb = sbase + OFF_WB;
        tc::store_row_bf16(hb, ct, h);
        tc::fence_async_smem();
        tc::named_bar(2, 128);
        const uint32_t idH = tc::idesc_bf16(128, 64, 0, 1);
        const uint32_t idU = tc::idesc_bf16(128, 64, 0, 1);
        const uint32_t idD = tc::idesc_bf16(128, 64, 1, 1);
        for (int c = 0; c < nch; ++c) {
            const int s = c & 1, b = c & 1;
            const int64_t t0 = cs + (int64_t)C * c;
            const int len = (int)((ce - t0) < C ? (ce - t0) : C);
            const uint32_t kq = sbase + OFF_KQ + s * SZ_KQ;
            const uint32_t tp = sbase + OFF_TP + b * SZ_TP;
            const uint32_t colH = COL_H + 64u * (c & 1), colO = COL_O + 64u * (c & 1);
            const Scal* sc = SC + b;
            wait(&full[s], (c >> 1) & 1, abort_flag);
            wait(&pfull[b], (c >> 1) & 1, abort_flag);
            if (ct == 0) {
                tc::tc_after_sync();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_bf16(tmem + colH,
                                 tc::sdesc_sw128(kq + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                                 tc::sdesc_sw128(hb + kk * 2048, 8192, 1024), idH, kk > 0);
                tc::mma_commit(mH);
            }
            wait(mH, c & 1, abort_flag);
            tc::tc_after_sync();
            if (ct < 64) {
                // R = beta (V - gamma * K h) for row r = ct
                const int r = ct;
                const float br = sc->beta[r], gr = sc->gam[r];
                const uint32_t vt = sbase + OFF_V + s * SZ_V;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    float x[32];
                    tc::tmem_ld32(tmem + lane_base + colH + 32 * hf, x);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const int ch = 4 * hf + q4;
                        const uint4 raw = tc::ld_shared_v4(vt + tc::sw128_off(r, ch));
                        const __nv_bfloat162* vv = reinterpret_cast<const __nv_bfloat162*>(&raw);
                        float o8[8];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 f = __bfloat1622float2(vv[e]);
                            o8[2 * e] = br * (f.x - gr * x[8 * q4 + 2 * e]);
                            o8[2 * e + 1] = br * (f.y - gr * x[8 * q4 + 2 * e + 1]);
                        }
                        tc::st_shared_v4(rb + tc::sw128_off(r, ch), tc::pack_bf16(o8[0], o8[1]),
                                         tc::pack_bf16(o8[2], o8[3]), tc::pack_bf16(o8[4], o8[5]),
                                         tc::pack_bf16(o8[6], o8[7]));
                    }
                }
            }
            tc::fence_async_smem();
            tc::tc_before_sync();
            tc::named_bar(2, 128);
            if (ct == 0) {
                tc::tc_after_sync();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_bf16(tmem + COL_U, tc::sdesc_sw128(tp + kk * 32, 16, 1024),
                                 tc::sdesc_sw128(rb + kk * 2048, 8192, 1024), idU, kk > 0);
                tc::mma_commit(mU);
            }
            wait(mU, c & 1, abort_flag);
            tc::tc_after_sync();
            if (ct < 64) {
                const int r = ct;
                const float wr = sc->w[r];
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    float x[32];
                    tc::tmem_ld32(tmem + lane_base + COL_U + 32 * hf, x);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const int ch = 4 * hf + q4;
                        const float* u = x + 8 * q4;
                        tc::st_shared_v4(ub + tc::sw128_off(r, ch), tc::pack_bf16(u[0], u[1]),
                                         tc::pack_bf16(u[2], u[3]), tc::pack_bf16(u[4], u[5]),
                                         tc::pack_bf16(u[6], u[7]));
                        tc::st_shared_v4(wb + tc::sw128_off(r, ch),
                                         tc::pack_bf16(wr * u[0], wr * u[1]),
                                         tc::pack_bf16(wr * u[2], wr * u[3]),
                                         tc::pack_bf16(wr * u[4], wr * u[5]),
                                         tc::pack_bf16(wr * u[6], wr * u[7]));
                    }
                }
            }
            tc::fence_async_smem();
            tc::tc_before_sync();
            tc::named_bar(2, 128);
            if (ct == 0) {
                tc::tc_after_sync();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_bf16(tmem + COL_D, tc::sdesc_sw128(kq + kk * 2048, 16384, 1024),
                                 tc::sdesc_sw128(wb + kk * 2048, 8192, 1024), idD, kk > 0);
                tc::mma_commit(mD);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_bf16(tmem + colO, tc::sdesc_sw128(tp + kk * 32, 16, 1024),
                                 tc::sdesc_sw128(ub + kk * 2048, 8192, 1024), idU, kk > 0);
                tc::mma_commit(mO);
            }
            wait(mD, c & 1, abort_flag);
            tc::tc_after_sync();
            {
                // h <- 2^G2_L h + K^T (w Ut), then the bf16 copy for the next chunk
                const float e = sc->eGL;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    float x[32];
                    tc::tmem_ld32(tmem + lane_base + COL_D + 32 * hf, x);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) h[32 * hf + j] = fmaf(e, h[32 * hf + j], x[j]);
                }
                tc::store_row_bf16(hb, ct, h);
            }
            if (ct == 0) tc::mbar_arrive(&empty[s]);  // stage no longer read by the chain
            tc::fence_async_smem();
            tc::tc_before_sync();
            tc::named_bar(2, 128);
            if (ct >= 64) {
                // output rows of this chunk: O = scale (gamma QH + P Ut)
                const int r = ct - 64;
                wait(mO, c & 1, abort_flag);
                tc::tc_after_sync();
                const float gr = sc->gam[r], scl = p.scale;
                float* ost = reinterpret_cast<float*>(base + OFF_OS);
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    float qh[32], pu[32];
                    tc::tmem_ld32(tmem + lane_base + colH + 32 * hf, qh);
                    tc::tmem_ld32(tmem + lane_base + colO + 32 * hf, pu);
                    tc::tmem_wait_ld();
                    float* orow = ost + r * OSP + 32 * hf;
#pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        *reinterpret_cast<float4*>(orow + j) =
                            make_float4(scl * fmaf(gr, qh[j], pu[j]),
                                        scl * fmaf(gr, qh[j + 1], pu[j + 1]),
                                        scl * fmaf(gr, qh[j + 2], pu[j + 2]),
                                        scl * fmaf(gr, qh[j + 3], pu[j + 3]));
                }
                tc::named_bar(3, 64);
                // coalesced stores: consecutive threads cover consecutive 16-byte
                // pieces of one output row
                const int ot = ct - 64;
                if constexpr (OBF16) {
                    __nv_bfloat16* obase = static_cast<__nv_bfloat16*>(p.o);
#pragma unroll 2
                    for (int it = 0; it < 8; ++it) {
                        const int rr = 8 * it + (ot >> 3), c8 = 8 * (ot & 7);
                        if (rr < len) {
                            const float4 a = *reinterpret_cast<const float4*>(ost + rr * OSP + c8);
                            const float4 bq =
                                *reinterpret_cast<const float4*>(ost + rr * OSP + c8 + 4);
                            uint4 w4;
                            w4.x = tc::pack_bf16(a.x, a.y);
                            w4.y = tc::pack_bf16(a.z, a.w);
                            w4.z = tc::pack_bf16(bq.x, bq.y);
                            w4.w = tc::pack_bf16(bq.z, bq.w);
                            *reinterpret_cast<uint4*>(obase + ((t0 + rr) * H + head) * VD + v0 +
                                                      c8) = w4;
                        }
                    }
                } else {
                    float* obase = static_cast<float*>(p.o);
#pragma unroll 4
                    for (int it = 0; it < 16; ++it) {
                        const int rr = 4 * it + (ot >> 4), c4 = 4 * (ot & 15);
                        if (rr < len)
                            *reinterpret_cast<float4*>(obase + ((t0 + rr) * H + head) * VD + v0 +
                                                       c4) =
                                *reinterpret_cast<const float4*>(ost + rr * OSP + c4);
                    }
                }
                tc::tc_before_sync();
                tc::mbar_arrive(&pempty[b]);
            }
        }
        if (p.hT) {
            float* dst = p.hT + hrow;
#pragma unroll
            for (int j = 0; j < 64; j += 4)
                *reinterpret_cast<float4*>(dst + j) = make_float4(h[j], h[j + 1], h[j + 2], h[j + 3]);
        }
        if (ct == 0 && *abort_flag) {
            // drain any MMA still running before tensor memory is released
            tc::mma_commit(mDrain);
            const uint32_t a = smem_u32(mDrain);
            for (uint32_t i = 0; i < kPolls && !mbar_try_wait(a, 0); ++i) {
            }
        }
    }
    tc::tc_before_sync();
    __syncthreads();
    tc::tc_after_sync();
    if (warp == 0) tc::tmem_dealloc(tmem, TMEM_COLS);
}

using EncodeTiled = PFN_cuTensorMapEncodeTiled_v12000;

inline EncodeTiled get_encode() {
    static EncodeTiled fn = nullptr;
    if (!fn) {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiled>(f);
    }
    return fn;
}

// [rows, cols] bf16 row-major, box of 64 rows x 64 columns, 128-byte swizzle.
inline bool make_map(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols) {
    EncodeTiled enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, 64};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tcf

// Launches the fused kernel for (n_seq, H) with two value slices.  Returns 0 on
// success, 1 when the tensor maps could not be built, 2 on a launch error.
inline int launch_chunk_tc(const ChunkArgs& a, int64_t T_total, bool obf16, cudaStream_t st) {
    tcf::Params p;
    memset(&p, 0, sizeof(p));
    const uint64_t cols = (uint64_t)a.H * 128;
    if (!tcf::make_map(&p.tm_q, a.q, (uint64_t)T_total, cols) ||
        !tcf::make_map(&p.tm_k, a.k, (uint64_t)T_total, cols) ||
        !tcf::make_map(&p.tm_v, a.v, (uint64_t)T_total, cols))
        return 1;
    p.g = a.g;
    p.beta = a.beta;
    p.h0 = a.h0;
    p.cu = a.cu_seqlens;
    p.order = a.order;
    p.T = a.T;
    p.H = a.H;
    p.scale = a.scale;
    p.o = a.o;
    p.hT = a.hT;
    const int64_t nb = (int64_t)a.n_seq * a.H * 2;
    auto kern = obf16 ? tcf::chunk_fwd_tc_kernel<true> : tcf::chunk_fwd_tc_kernel<false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)tcf::SMEM_BYTES) != cudaSuccess)
        return 2;
    kern<<<(unsigned)nb, tcf::kThreads, tcf::SMEM_BYTES, st>>>(p);
    return 0;
}

}  // namespace gdn
