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
constexpr int XTP = 20;
constexpr uint32_t OFF_XT = OFF_TF + 64 * AFP * 4;  // fp32 [3][16][20]
struct Scal {
    float G2[64];
    float beta[64];
    float gam[64];
    float w[64];
    float eGL;
    float pad[3];
};
constexpr uint32_t OFF_SC = OFF_XT + 3 * 16 * XTP * 4;
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

// 16x16x16 fp32 product on one warp: acc[2][4] covers rows 2*(lane/4)+{0,1},
// columns 4*(lane%4)+{0..3}.  Row pitches in floats; Y rows 16-byte aligned.
__device__ __forceinline__ void mm16(float (&acc)[2][4], const float* X, int xs, const float* Y,
                                     int ys, int lane) {
    const int r0 = 2 * (lane >> 2), c0 = 4 * (lane & 3);
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        const float a0 = X[r0 * xs + k], a1 = X[(r0 + 1) * xs + k];
        const float4 y = *reinterpret_cast<const float4*>(Y + k * ys + c0);
        acc[0][0] = fmaf(a0, y.x, acc[0][0]);
        acc[0][1] = fmaf(a0, y.y, acc[0][1]);
        acc[0][2] = fmaf(a0, y.z, acc[0][2]);
        acc[0][3] = fmaf(a0, y.w, acc[0][3]);
        acc[1][0] = fmaf(a1, y.x, acc[1][0]);
        acc[1][1] = fmaf(a1, y.y, acc[1][1]);
        acc[1][2] = fmaf(a1, y.z, acc[1][2]);
        acc[1][3] = fmaf(a1, y.w, acc[1][3]);
    }
}
__device__ __forceinline__ void mm16_store(const float (&acc)[2][4], float* Z, int zs, int lane,
                                           float sign) {
    const int r0 = 2 * (lane >> 2), c0 = 4 * (lane & 3);
#pragma unroll
    for (int i = 0; i < 2; ++i)
        *reinterpret_cast<float4*>(Z + (r0 + i) * zs + c0) =
            make_float4(sign * acc[i][0], sign * acc[i][1], sign * acc[i][2], sign * acc[i][3]);
}
// Same product restricted to 4 rows (row block rb of 4) on one warp:
// acc[2] covers row 4*rb + lane/8, columns 2*(lane%8)+{0,1}.
__device__ __forceinline__ void mm16_rows4(float (&acc)[2], const float* X, int xs, const float* Y,
                                           int ys, int rb, int lane) {
    const int r = 4 * rb + (lane >> 3), c0 = 2 * (lane & 7);
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        const float a = X[r * xs + k];
        const float2 y = *reinterpret_cast<const float2*>(Y + k * ys + c0);
        acc[0] = fmaf(a, y.x, acc[0]);
        acc[1] = fmaf(a, y.y, acc[1]);
    }
}

// T = (I + A)^-1 for the strictly lower 64x64 A (fp32, pitch AFP) by 16x16
// blocks: diagonal blocks by substitution, then off-diagonal blocks by
// distance from the diagonal, T_ij = -T_ii sum_{j<=k<i} A_ik T_kj.
// Writes every T entry on or below the diagonal (diagonal blocks complete).
// Called by the 128 prep threads; uses named barrier 1.
__device__ __forceinline__ void invert_unit_lower(const float* Af, float* Tf, float* Xt, int pw,
                                                  int lane) {
    // diagonal blocks: warp pw owns block pw, lanes 0..15 one column each
    if (lane < 16) {
        const int o = 16 * pw, j = lane;
        float t[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float acc = 0.f;
#pragma unroll
            for (int s = 0; s < r; ++s) acc = fmaf(Af[(o + r) * AFP + o + s], t[s], acc);
            t[r] = (r < j) ? 0.f : ((r == j) ? 1.f : -acc);
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) Tf[(o + r) * AFP + o + j] = t[r];
    }
    tc::named_bar(1, 128);
    // distance 1: blocks (1,0), (2,1), (3,2)
    if (pw < 3) {
        const int i = pw + 1, j = pw;
        float* X = Xt + pw * 16 * XTP;
        float acc[2][4] = {};
        mm16(acc, Af + 16 * i * AFP + 16 * j, AFP, Tf + 16 * j * AFP + 16 * j, AFP, lane);
        mm16_store(acc, X, XTP, lane, 1.f);
        __syncwarp();
        float acc2[2][4] = {};
        mm16(acc2, Tf + 16 * i * AFP + 16 * i, AFP, X, XTP, lane);
        mm16_store(acc2, Tf + 16 * i * AFP + 16 * j, AFP, lane, -1.f);
    }
    tc::named_bar(1, 128);
    // distance 2: blocks (2,0), (3,1)
    if (pw < 2) {
        const int i = pw + 2, j = pw;
        float* X = Xt + pw * 16 * XTP;
        float acc[2][4] = {};
        mm16(acc, Af + 16 * i * AFP + 16 * j, AFP, Tf + 16 * j * AFP + 16 * j, AFP, lane);
        mm16(acc, Af + 16 * i * AFP + 16 * (j + 1), AFP, Tf + 16 * (j + 1) * AFP + 16 * j, AFP,
             lane);
        mm16_store(acc, X, XTP, lane, 1.f);
        __syncwarp();
        float acc2[2][4] = {};
        mm16(acc2, Tf + 16 * i * AFP + 16 * i, AFP, X, XTP, lane);
        mm16_store(acc2, Tf + 16 * i * AFP + 16 * j, AFP, lane, -1.f);
    }
    tc::named_bar(1, 128);
    // distance 3: block (3,0), rows split over the four warps
    {
        float* X = Xt;
        float acc[2] = {0.f, 0.f};
        mm16_rows4(acc, Af + 48 * AFP + 0, AFP, Tf + 0 * AFP + 0, AFP, pw, lane);
        mm16_rows4(acc, Af + 48 * AFP + 16, AFP, Tf + 16 * AFP + 0, AFP, pw, lane);
        mm16_rows4(acc, Af + 48 * AFP + 32, AFP, Tf + 32 * AFP + 0, AFP, pw, lane);
        const int r = 4 * pw + (lane >> 3), c0 = 2 * (lane & 7);
        *reinterpret_cast<float2*>(X + r * XTP + c0) = make_float2(acc[0], acc[1]);
        tc::named_bar(1, 128);
        float acc2[2] = {0.f, 0.f};
        mm16_rows4(acc2, Tf + 48 * AFP + 48, AFP, X, XTP, pw, lane);
        *reinterpret_cast<float2*>(Tf + (48 + r) * AFP + c0) = make_float2(-acc2[0], -acc2[1]);
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
            if (pt < 64) {
                sc->gam[pt] = exp2f(x);
                sc->w[pt] = exp2f(G2L - x);
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
            if (pt < 64) {
                const int r = pt;
                const float g2r = sc->G2[r], br = bv;
                float* arow = Af + r * AFP;
#pragma unroll
                for (int j = 0; j < 64; j += 4) {
                    float4 av;
                    av.x = (j + 0 < r) ? br * exp2f(g2r - sc->G2[j + 0]) * sv[j + 0] : 0.f;
                    av.y = (j + 1 < r) ? br * exp2f(g2r - sc->G2[j + 1]) * sv[j + 1] : 0.f;
                    av.z = (j + 2 < r) ? br * exp2f(g2r - sc->G2[j + 2]) * sv[j + 2] : 0.f;
                    av.w = (j + 3 < r) ? br * exp2f(g2r - sc->G2[j + 3]) * sv[j + 3] : 0.f;
                    *reinterpret_cast<float4*>(arow + j) = av;
                }
            } else {
                const int r = pt - 64;
                const float g2r = sc->G2[r];
#pragma unroll
                for (int j = 0; j < 64; ++j)
                    sv[j] = (j <= r) ? exp2f(g2r - sc->G2[j]) * sv[j] : 0.f;
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
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    float qh[32], pu[32];
                    tc::tmem_ld32(tmem + lane_base + colH + 32 * hf, qh);
                    tc::tmem_ld32(tmem + lane_base + colO + 32 * hf, pu);
                    tc::tmem_wait_ld();
                    if (r < len) {
                        const int64_t orow = ((t0 + r) * H + head) * VD + v0 + 32 * hf;
                        if constexpr (OBF16) {
                            __nv_bfloat16* op = static_cast<__nv_bfloat16*>(p.o) + orow;
#pragma unroll
                            for (int j = 0; j < 32; j += 8) {
                                uint4 w4;
                                w4.x = tc::pack_bf16(scl * fmaf(gr, qh[j], pu[j]),
                                                     scl * fmaf(gr, qh[j + 1], pu[j + 1]));
                                w4.y = tc::pack_bf16(scl * fmaf(gr, qh[j + 2], pu[j + 2]),
                                                     scl * fmaf(gr, qh[j + 3], pu[j + 3]));
                                w4.z = tc::pack_bf16(scl * fmaf(gr, qh[j + 4], pu[j + 4]),
                                                     scl * fmaf(gr, qh[j + 5], pu[j + 5]));
                                w4.w = tc::pack_bf16(scl * fmaf(gr, qh[j + 6], pu[j + 6]),
                                                     scl * fmaf(gr, qh[j + 7], pu[j + 7]));
                                *reinterpret_cast<uint4*>(op + j) = w4;
                            }
                        } else {
                            float* op = static_cast<float*>(p.o) + orow;
#pragma unroll
                            for (int j = 0; j < 32; j += 4)
                                *reinterpret_cast<float4*>(op + j) =
                                    make_float4(scl * fmaf(gr, qh[j], pu[j]),
                                                scl * fmaf(gr, qh[j + 1], pu[j + 1]),
                                                scl * fmaf(gr, qh[j + 2], pu[j + 2]),
                                                scl * fmaf(gr, qh[j + 3], pu[j + 3]));
                        }
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
