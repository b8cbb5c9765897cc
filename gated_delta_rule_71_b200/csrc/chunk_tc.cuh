// chunk_tc.cuh -- fused tensor-core chunked forward of the gated delta rule
// (bf16 q/k/v, K = V = 128, fp32 state, fp32 accumulation), sm_100a.
//
// The three GDN steps of ZzCompute (PyTorch Helion Hackathon gallery entry 11)
// -- item 4 "Recompute W/U" (in-chunk cumsum, A, T = (I+A)^-1), item 2 "Chunk
// Forward H" (state recurrence) and item 3 "Chunk Forward O" (chunk output) --
// run in one launch, so q/k/v/g/beta are read from HBM once and o/h_T written
// once.  Per chunk (64 tokens, G2 = log2-scaled in-chunk cumsum of g):
//   S    = [K; Q] K^T                               (MMA, M=128 N=64 K=128)
//   A    = strictly-lower beta_r 2^(G2_r-G2_s) (K K^T)_rs,  T = (I + A)^-1
//   P    = lower-incl 2^(G2_r-G2_s) (Q K^T)_rs
//   [KH; QH] = [K; Q] h                             (MMA, B = bf16 copy of h)
//   R    = beta (V - 2^G2 * KH)
//   Ut   = T R             ( = U - W h of the WY form)  (MMA, A = [T; P])
//   h'   = 2^G2_L h + K^T (2^(G2_L-G2) * Ut)            (MMA, then fp32 update)
//   O    = scale (2^G2 * QH + P Ut)                      (MMA, A = [T; P])
//
// Each (sequence, head) runs on a cluster of two CTAs, one per SM:
//  * rank 0, "prep": three warpgroups, each owning every third chunk, its own
//    TMA stage and its own slot in the chain CTA.  A warpgroup computes S on
//    tcgen05, the A and P rows, and T by 16x16 blocks, and writes T, P (bf16)
//    and the per-row gate factors straight into the chain CTA's shared memory
//    (DSMEM), then releases them with cluster-scope mbarrier arrives.  Three
//    chunks are in flight, so the serial triangular inverse is off the chain.
//  * rank 1, "chain": four warpgroups, one per 32 value columns, carry the
//    fp32 state in registers (one key row per thread) through the serial part
//    with N = 128 tcgen05 MMAs and write the output rows.
// TMA loads are issued by the thread that releases a stage, so no producer
// warp waits.  Every wait is bounded: a wait that gives up sets the CTA's
// abort flag (all later waits fall through, so every barrier is still
// reached), records GDN_ERR_TIMEOUT, and the issuing threads drain their
// copies and MMAs before tensor memory is released.
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
constexpr int kThreads = 512;
constexpr int NPREP = 3;  // prep warpgroups (chunks in flight in the prep CTA)
constexpr uint32_t kPolls = 1u << 22;
constexpr float kLog2e = 1.4426950408889634f;

// ---- shared memory, prep CTA (byte offsets from a 1024-aligned base)
constexpr uint32_t SZ_KQ = 32768;  // [2 key halves][K rows 0-63 | Q rows 64-127][128 B]
constexpr int AFP = 68;            // fp32 row pitch of A / T
constexpr int XTP = 24;            // pitch of the 16x16 temporaries (conflict-free B fragments)
constexpr uint32_t SZ_AF = 64 * AFP * 4;
constexpr uint32_t SZ_XT = 3 * 16 * XTP * 4;
struct PrepScal {   // per prep warpgroup
    float G2[64];   // in-chunk inclusive cumsum of g, log2 units
    float ginv[64]; // 2^-G2 (only when the chunk's decay stays in fp32 range)
    float gam[64];  // 2^G2
    float pad;
    float scan_tmp;
    float pad2[2];
};
constexpr uint32_t P_OFF_KQ = 0;                                  // NPREP stages
constexpr uint32_t P_OFF_AF = P_OFF_KQ + NPREP * SZ_KQ;           // NPREP x A
constexpr uint32_t P_OFF_TF = P_OFF_AF + NPREP * SZ_AF;           // NPREP x T
constexpr uint32_t P_OFF_XT = P_OFF_TF + NPREP * SZ_AF;           // NPREP x temporaries
constexpr uint32_t P_OFF_SC = P_OFF_XT + NPREP * SZ_XT;           // NPREP x PrepScal
constexpr uint32_t P_END = P_OFF_SC + NPREP * sizeof(PrepScal);

// ---- shared memory, chain CTA
constexpr uint32_t SZ_V = 16384;   // [2 atoms of 64 v][64 rows][128 B]
constexpr uint32_t SZ_TP = 16384;  // [T rows 0-63 | P rows 64-127][64 bf16]
struct ChainScal {  // per slot, written by the prep CTA
    float beta[64];
    float gam[64];  // 2^G2
    float w[64];    // 2^(G2_L - G2)
    float eGL;      // 2^G2_L
    float pad[3];
};
constexpr uint32_t C_OFF_KQ = 0;                                // 2 stages
constexpr uint32_t C_OFF_V = C_OFF_KQ + 2 * SZ_KQ;              // 1 buffer (refilled after R)
constexpr uint32_t C_OFF_TP = C_OFF_V + SZ_V;                   // NPREP slots
constexpr uint32_t C_OFF_HB = C_OFF_TP + NPREP * SZ_TP;         // h bf16 [2 atoms][128][128 B]
constexpr uint32_t C_OFF_RB = C_OFF_HB + 32768;                 // R [2 atoms][64][128 B]
constexpr uint32_t C_OFF_UB = C_OFF_RB + 16384;                 // Ut
constexpr uint32_t C_OFF_WB = C_OFF_UB + 16384;                 // 2^(G2_L-G2) Ut
constexpr uint32_t C_OFF_OS = C_OFF_UB;                         // fp32 output rows [64][128]
constexpr uint32_t C_OFF_SC = C_OFF_WB + 16384;                 // NPREP x ChainScal
constexpr uint32_t C_END = C_OFF_SC + NPREP * sizeof(ChainScal);

constexpr uint32_t BODY = (P_END > C_END ? P_END : C_END);
constexpr uint32_t OFF_BAR = (BODY + 15) & ~15u;
constexpr uint32_t OFF_MISC = OFF_BAR + 32 * 8;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 64 + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// ---- tensor memory columns
constexpr uint32_t P_COL_S = 0;  // NPREP x 64 in the prep CTA
constexpr uint32_t P_TMEM_COLS = 256;
constexpr uint32_t C_COL_H = 0;    // two buffers of 128
constexpr uint32_t C_COL_U = 256;  // Ut, then [T Ut; P Ut]
constexpr uint32_t C_COL_D = 384;  // K^T (w Ut)
constexpr uint32_t C_TMEM_COLS = 512;

// barrier slots
enum : int {
    B_FULL = 0,        // [NPREP] prep: TMA stage; chain uses [0..1]
    B_MS = 3,          // [NPREP] prep: S ready
    B_FREE = 6,        // [NPREP] prep: chain slot free (remote arrivals)
    B_TPF = 9,         // [NPREP] chain: slot filled (remote arrivals, 128 each)
    B_MH = 12, B_MU, B_MD, B_MO, B_DRAIN,
    B_FULLV,           // chain: V tile
};

struct Params {
    CUtensorMap tm_q, tm_k, tm_v, tm_o;  // tm_o: fp32 output, 32 x 64 boxes
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

// Bounded wait that honours the CTA's abort flag.  `cluster` selects
// acquire at cluster scope (arrivals from the other CTA).
__device__ __forceinline__ bool wait(uint64_t* bar, uint32_t phase, volatile uint32_t* abort,
                                     bool cluster = false) {
    if (*abort) return false;
    const uint32_t a = smem_u32(bar);
    for (uint32_t i = 0; i < kPolls; ++i) {
        if (cluster ? tc::mbar_try_wait_cluster(a, phase) : mbar_try_wait(a, phase)) return true;
        if ((i & 255u) == 255u && *abort) return false;
    }
    *abort = 1u;
    record_status(GDN_ERR_TIMEOUT);
    return false;
}

// Bounded wait that ignores the abort flag (used to drain on the way out).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t phase) {
    const uint32_t a = smem_u32(bar);
    for (uint32_t i = 0; i < kPolls && !mbar_try_wait(a, phase); ++i) {
    }
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
// with their zero upper halves).  Called by the 128 threads of one prep
// warpgroup; uses named barrier `bid`.
__device__ __forceinline__ void invert_unit_lower(const float* Af, float* Tf, float* Xt, int pw,
                                                  int lane, int bid) {
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
    tc::named_bar(bid, 128);
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
    tc::named_bar(bid, 128);
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
    tc::named_bar(bid, 128);
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
    tc::named_bar(bid, 128);
}


template <bool OBF16>
__global__ void __launch_bounds__(kThreads, 1) chunk_fwd_tc_kernel(const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t sbase = (raw_u32 + 1023u) & ~1023u;
    uint8_t* base = smem_raw + (sbase - raw_u32);

    uint64_t* bars = reinterpret_cast<uint64_t*>(base + OFF_BAR);
    uint32_t* misc = reinterpret_cast<uint32_t*>(base + OFF_MISC);
    volatile uint32_t* abort_flag = misc + 1;

    const uint32_t rank = tc::cluster_ctarank();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int H = p.H;
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

    if (threadIdx.x == 0) {
        for (int i = 0; i < 32; ++i)
            mbar_init(&bars[i], (i >= B_TPF && i < B_TPF + NPREP) ? 128u : 1u);
        misc[1] = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    const uint32_t ncols = rank == 0 ? P_TMEM_COLS : C_TMEM_COLS;
    if (warp == 0) tc::tmem_alloc(&misc[0], ncols);
    tc::tc_before_sync();
    __syncthreads();
    tc::cluster_sync();  // both CTAs' barriers initialised before any remote arrive
    tc::tc_after_sync();
    const uint32_t tmem = misc[0];

    if (rank == 0) {
        // ================================================================ prep
        const int wg = warp >> 2;  // 0..3; warpgroups 1..NPREP work
        if (wg >= 1 && wg <= NPREP) {
            const int pg = wg - 1, pt = threadIdx.x - 128 * wg, pw = warp & 3;
            const int bid = 1 + pg;
            uint8_t* kq_p = base + P_OFF_KQ + pg * SZ_KQ;
            const uint32_t kq = sbase + P_OFF_KQ + pg * SZ_KQ;
            float* Af = reinterpret_cast<float*>(base + P_OFF_AF + pg * SZ_AF);
            float* Tf = reinterpret_cast<float*>(base + P_OFF_TF + pg * SZ_AF);
            float* Xt = reinterpret_cast<float*>(base + P_OFF_XT + pg * SZ_XT);
            PrepScal* ls = reinterpret_cast<PrepScal*>(base + P_OFF_SC) + pg;
            uint64_t* full = &bars[B_FULL + pg];
            uint64_t* mS = &bars[B_MS + pg];
            uint64_t* sfree = &bars[B_FREE + pg];
            // the chain CTA's slot for this warpgroup
            const uint32_t r_tp = tc::mapa(sbase + C_OFF_TP + pg * SZ_TP, 1);
            const uint32_t r_sc = tc::mapa(sbase + C_OFF_SC + pg * (uint32_t)sizeof(ChainScal), 1);
            const uint32_t r_tpf = tc::mapa(smem_u32(&bars[B_TPF + pg]), 1);
            const uint32_t idS = tc::idesc_bf16(128, 64, 0, 0);
            auto issue_load = [&](int c) {
                const int y = (int)(cs + (int64_t)C * c);
                tc::mbar_arrive_expect_tx(full, SZ_KQ);
                tc::tma_load_2d(kq_p + 0, &p.tm_k, head * KD + 0, y, full);
                tc::tma_load_2d(kq_p + 8192, &p.tm_q, head * KD + 0, y, full);
                tc::tma_load_2d(kq_p + 16384, &p.tm_k, head * KD + 64, y, full);
                tc::tma_load_2d(kq_p + 24576, &p.tm_q, head * KD + 64, y, full);
            };
            int last_loaded = -1;
            if (pt == 0 && pg < nch) {
                tc::prefetch_tmap(&p.tm_q);
                tc::prefetch_tmap(&p.tm_k);
                issue_load(pg);
                last_loaded = pg;
            }
            for (int c = pg, n = 0; c < nch; c += NPREP, ++n) {
                const int64_t t0 = cs + (int64_t)C * c;
                const int len = (int)((ce - t0) < C ? (ce - t0) : C);
                float gv = 0.f, bv = 0.f;
                if (pt < len) {
                    gv = p.g[(t0 + pt) * H + head];
                    bv = p.beta[(t0 + pt) * H + head];
                }
                wait(full, n & 1, abort_flag);
                if (pt == 0) {
                    tc::tc_after_sync();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                        tc::mma_bf16(tmem + P_COL_S + 64 * pg, tc::sdesc_sw128(kq + off, 16, 1024),
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
                if (pt == 31) ls->scan_tmp = x;
                if (n >= 1) wait(sfree, (n - 1) & 1, abort_flag, true);  // chain done with the slot
                tc::named_bar(bid, 128);
                if (pw == 1) x += ls->scan_tmp;
                if (pt < 64) ls->G2[pt] = x;
                tc::named_bar(bid, 128);
                const float G2L = ls->G2[63];
                // 2^(G2_r - G2_s) = 2^G2_r * 2^-G2_s whenever the chunk's total decay
                // stays above 2^-126 (no overflow or subnormal factor); else per element
                const bool factored = G2L > -126.f;
                if (pt < 64) {
                    const float gm = exp2f(x);
                    ls->gam[pt] = gm;
                    ls->ginv[pt] = factored ? exp2f(-x) : 0.f;
                    tc::st_cluster_f32(r_sc + 4 * (0 * 64 + pt), bv);
                    tc::st_cluster_f32(r_sc + 4 * (1 * 64 + pt), gm);
                    tc::st_cluster_f32(r_sc + 4 * (2 * 64 + pt), exp2f(G2L - x));
                    if (pt == 0) tc::st_cluster_f32(r_sc + 4 * (3 * 64), exp2f(G2L));
                }
                // S row of this thread: rows 0-63 = K K^T, rows 64-127 = Q K^T
                wait(mS, n & 1, abort_flag);
                tc::tc_after_sync();
                float sv[64];
                {
                    const uint32_t ta = tmem + ((uint32_t)(32 * pw) << 16) + P_COL_S + 64 * pg;
                    tc::tmem_ld32(ta, *reinterpret_cast<float(*)[32]>(sv));
                    tc::tmem_ld32(ta + 32, *reinterpret_cast<float(*)[32]>(sv + 32));
                    tc::tmem_wait_ld();
                }
                // the stage is no longer read: fetch this warpgroup's next chunk into it
                if (pt == 0 && c + NPREP < nch) {
                    issue_load(c + NPREP);
                    last_loaded = c + NPREP;
                }
                tc::named_bar(bid, 128);  // ginv / gam visible
                if (pt < 64) {
                    const int r = pt;
                    const float g2r = ls->G2[r], br = bv;
                    float* arow = Af + r * AFP;
                    if (factored) {
                        const float coef = br * ls->gam[r];
#pragma unroll
                        for (int j = 0; j < 64; j += 4) {
                            const float4 gi = *reinterpret_cast<const float4*>(ls->ginv + j);
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
                            av.x = (j + 0 < r) ? br * exp2f(g2r - ls->G2[j + 0]) * sv[j + 0] : 0.f;
                            av.y = (j + 1 < r) ? br * exp2f(g2r - ls->G2[j + 1]) * sv[j + 1] : 0.f;
                            av.z = (j + 2 < r) ? br * exp2f(g2r - ls->G2[j + 2]) * sv[j + 2] : 0.f;
                            av.w = (j + 3 < r) ? br * exp2f(g2r - ls->G2[j + 3]) * sv[j + 3] : 0.f;
                            *reinterpret_cast<float4*>(arow + j) = av;
                        }
                    }
                } else {
                    const int r = pt - 64;
                    const float g2r = ls->G2[r];
                    if (factored) {
                        const float coef = ls->gam[r];
#pragma unroll
                        for (int j = 0; j < 64; j += 4) {
                            const float4 gi = *reinterpret_cast<const float4*>(ls->ginv + j);
                            sv[j + 0] = (j + 0 <= r) ? coef * gi.x * sv[j + 0] : 0.f;
                            sv[j + 1] = (j + 1 <= r) ? coef * gi.y * sv[j + 1] : 0.f;
                            sv[j + 2] = (j + 2 <= r) ? coef * gi.z * sv[j + 2] : 0.f;
                            sv[j + 3] = (j + 3 <= r) ? coef * gi.w * sv[j + 3] : 0.f;
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 64; ++j)
                            sv[j] = (j <= r) ? exp2f(g2r - ls->G2[j]) * sv[j] : 0.f;
                    }
                    // P row -> the chain CTA's slot (rows 64-127 of the stacked operand)
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch)
                        tc::st_cluster_v4(r_tp + 8192 + tc::sw128_off(r, ch),
                                          tc::pack_bf16(sv[8 * ch + 0], sv[8 * ch + 1]),
                                          tc::pack_bf16(sv[8 * ch + 2], sv[8 * ch + 3]),
                                          tc::pack_bf16(sv[8 * ch + 4], sv[8 * ch + 5]),
                                          tc::pack_bf16(sv[8 * ch + 6], sv[8 * ch + 7]));
                }
                tc::tc_before_sync();
                tc::named_bar(bid, 128);
                invert_unit_lower(Af, Tf, Xt, pw, lane, bid);
                {
                    // T rows -> bf16 (upper part zero) into the chain CTA's slot
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
                        tc::st_cluster_v4(r_tp + tc::sw128_off(r, ch), tc::pack_bf16(t8[0], t8[1]),
                                          tc::pack_bf16(t8[2], t8[3]), tc::pack_bf16(t8[4], t8[5]),
                                          tc::pack_bf16(t8[6], t8[7]));
                    }
                }
                // publish: the chain CTA's MMAs read the slot through the async proxy
                tc::fence_async_cluster();
                tc::mbar_arrive_cluster(r_tpf);
            }
            if (pt == 0) {
                // never leave with a copy or an MMA in flight
                if (last_loaded >= 0) drain_wait(full, (last_loaded / NPREP) & 1);
                if (*abort_flag) {
                    tc::mma_commit(&bars[B_DRAIN]);
                    drain_wait(&bars[B_DRAIN], 0);
                }
            }
        }
    } else {
        // =============================================================== chain
        const int ct = threadIdx.x, wg = warp >> 2, q = warp & 3;  // wg: 32 value columns
        const int row = 32 * q + lane;                               // key row / token row
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const int atom = wg >> 1, hcol = wg & 1;  // 64-column atom and its half
        const int v0 = 32 * wg;
        const int64_t hrow = ((int64_t)(seq * H + head) * KD + row) * VD + v0;
        float h[32];
        if (p.h0) {
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
                const float4 t = *reinterpret_cast<const float4*>(p.h0 + hrow + j);
                h[j] = t.x; h[j + 1] = t.y; h[j + 2] = t.z; h[j + 3] = t.w;
            }
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) h[j] = 0.f;
        }
        const uint32_t hb = sbase + C_OFF_HB, rb = sbase + C_OFF_RB, ub = sbase + C_OFF_UB,
                       wb = sbase + C_OFF_WB;
        tc::store_half_row_bf16(hb + atom * 16384, row, hcol, h);
        uint64_t* mH = &bars[B_MH];
        uint64_t* mU = &bars[B_MU];
        uint64_t* mD = &bars[B_MD];
        uint64_t* mO = &bars[B_MO];
        const uint32_t idH = tc::idesc_bf16(128, 128, 0, 1);
        const uint32_t idD = tc::idesc_bf16(128, 128, 1, 1);
        auto issue_load = [&](int c) {
            const int s = c & 1;
            const int y = (int)(cs + (int64_t)C * c);
            uint64_t* full = &bars[B_FULL + s];
            uint8_t* kq = base + C_OFF_KQ + s * SZ_KQ;
            tc::mbar_arrive_expect_tx(full, SZ_KQ);
            tc::tma_load_2d(kq + 0, &p.tm_k, head * KD + 0, y, full);
            tc::tma_load_2d(kq + 8192, &p.tm_q, head * KD + 0, y, full);
            tc::tma_load_2d(kq + 16384, &p.tm_k, head * KD + 64, y, full);
            tc::tma_load_2d(kq + 24576, &p.tm_q, head * KD + 64, y, full);
        };
        auto issue_load_v = [&](int c) {
            const int y = (int)(cs + (int64_t)C * c);
            uint64_t* fv = &bars[B_FULLV];
            uint8_t* vt = base + C_OFF_V;
            tc::mbar_arrive_expect_tx(fv, SZ_V);
            tc::tma_load_2d(vt + 0, &p.tm_v, head * VD + 0, y, fv);
            tc::tma_load_2d(vt + 8192, &p.tm_v, head * VD + 64, y, fv);
        };
        int last_loaded = -1;
        if (ct == 0) {
            tc::prefetch_tmap(&p.tm_q);
            tc::prefetch_tmap(&p.tm_k);
            tc::prefetch_tmap(&p.tm_v);
            for (int c = 0; c < 2 && c < nch; ++c) {
                issue_load(c);
                last_loaded = c;
            }
            if (nch > 0) issue_load_v(0);
        }
        int last_v = nch > 0 ? 0 : -1;
        tc::fence_async_smem();
        tc::named_bar(1, 512);
        const uint32_t r_free0 = tc::mapa(smem_u32(&bars[B_FREE]), 0);
        for (int c = 0; c < nch; ++c) {
            const int s = c & 1, j = c % NPREP, n3 = c / NPREP;
            const int64_t t0 = cs + (int64_t)C * c;
            const int len = (int)((ce - t0) < C ? (ce - t0) : C);
            const uint32_t kq = sbase + C_OFF_KQ + s * SZ_KQ;
            const uint32_t tp = sbase + C_OFF_TP + j * SZ_TP;
            const uint32_t colH = C_COL_H + 128u * (c & 1);
            const ChainScal* sc = reinterpret_cast<const ChainScal*>(base + C_OFF_SC) + j;
            wait(&bars[B_FULL + s], (c >> 1) & 1, abort_flag);
            wait(&bars[B_TPF + j], n3 & 1, abort_flag, true);
            if (ct == 0) {
                tc::fence_async_smem();
                tc::tc_after_sync();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_bf16(tmem + colH,
                                 tc::sdesc_sw128(kq + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                                 tc::sdesc_sw128(hb + kk * 2048, 16384, 1024), idH, kk > 0);
                tc::mma_commit(mH);
            }
            wait(mH, c & 1, abort_flag);
            tc::tc_after_sync();
            if (q < 2) {
                // R = beta (V - gamma * K h) for token row `row`, this warpgroup's 32 columns
                wait(&bars[B_FULLV], c & 1, abort_flag);
                const float br = sc->beta[row], gr = sc->gam[row];
                const uint32_t vt = sbase + C_OFF_V + atom * 8192;
                float x[32];
                tc::tmem_ld32(tmem + lane_base + colH + v0, x);
                tc::tmem_wait_ld();
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const int ch = 4 * hcol + q4;
                    const uint4 raw = tc::ld_shared_v4(vt + tc::sw128_off(row, ch));
                    const __nv_bfloat162* vv = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __bfloat1622float2(vv[e]);
                        x[8 * q4 + 2 * e] = br * (f.x - gr * x[8 * q4 + 2 * e]);
                        x[8 * q4 + 2 * e + 1] = br * (f.y - gr * x[8 * q4 + 2 * e + 1]);
                    }
                }
                tc::store_half_row_bf16(rb + atom * 8192, row, hcol, x);
            }
            if (q == 2 && lane == 0) tc::bulk_wait_read0();  // last chunk's output staging read
            tc::fence_async_smem();
            tc::tc_before_sync();
            tc::named_bar(1, 512);
            if (ct == 0) {
                tc::tc_after_sync();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_bf16(tmem + C_COL_U, tc::sdesc_sw128(tp + kk * 32, 16, 1024),
                                 tc::sdesc_sw128(rb + kk * 2048, 8192, 1024), idH, kk > 0);
                tc::mma_commit(mU);
                if (c + 1 < nch) {  // this chunk's V has been read: fetch the next one
                    issue_load_v(c + 1);
                    last_v = c + 1;
                }
            }
            wait(mU, c & 1, abort_flag);
            tc::tc_after_sync();
            if (q < 2) {
                const float wr = sc->w[row];
                float x[32];
                tc::tmem_ld32(tmem + lane_base + C_COL_U + v0, x);
                tc::tmem_wait_ld();
                tc::store_half_row_bf16(ub + atom * 8192, row, hcol, x);
#pragma unroll
                for (int e = 0; e < 32; ++e) x[e] *= wr;
                tc::store_half_row_bf16(wb + atom * 8192, row, hcol, x);
            }
            tc::fence_async_smem();
            tc::tc_before_sync();
            tc::named_bar(1, 512);
            if (ct == 0) {
                tc::tc_after_sync();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_bf16(tmem + C_COL_D, tc::sdesc_sw128(kq + kk * 2048, 16384, 1024),
                                 tc::sdesc_sw128(wb + kk * 2048, 8192, 1024), idD, kk > 0);
                tc::mma_commit(mD);
            } else if (ct == 64) {
                // the output product is off the chain: issued by an output-warp thread
                tc::tc_after_sync();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_bf16(tmem + C_COL_U, tc::sdesc_sw128(tp + kk * 32, 16, 1024),
                                 tc::sdesc_sw128(ub + kk * 2048, 8192, 1024), idH, kk > 0);
                tc::mma_commit(mO);
            }
            wait(mD, c & 1, abort_flag);
            tc::tc_after_sync();
            {
                // h <- 2^G2_L h + K^T (w Ut), then the bf16 copy for the next chunk
                const float e = sc->eGL;
                float x[32];
                tc::tmem_ld32(tmem + lane_base + C_COL_D + v0, x);
                tc::tmem_wait_ld();
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) h[jj] = fmaf(e, h[jj], x[jj]);
                tc::store_half_row_bf16(hb + atom * 16384, row, hcol, h);
            }
            if (ct == 0 && c + 2 < nch) {
                // K/Q of this stage are no longer read (MMA_H, MMA_dH done)
                issue_load(c + 2);
                last_loaded = c + 2;
            }
            tc::fence_async_smem();
            tc::tc_before_sync();
            tc::named_bar(1, 512);
            if (q >= 2) {
                // output rows: O = scale (gamma QH + P Ut)
                const int r = row - 64;
                wait(mO, c & 1, abort_flag);
                tc::tc_after_sync();
                const float gr = sc->gam[r], scl = p.scale;
                float qh[32], pu[32];
                tc::tmem_ld32(tmem + lane_base + colH + v0, qh);
                tc::tmem_ld32(tmem + lane_base + C_COL_U + v0, pu);
                tc::tmem_wait_ld();
                // slot j (T, P, gate factors) is consumed once MMA_O is done and
                // gamma read: hand it back to prep before the stores
                tc::tc_before_sync();
                tc::named_bar(6, 256);
                if (ct == 64) tc::mbar_arrive_cluster(r_free0 + 8 * j);
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) qh[jj] = scl * fmaf(gr, qh[jj], pu[jj]);
                if (!OBF16 && len == C) {
                    // full chunk: stage this warpgroup's 64 x 32 fp32 block in the
                    // 128-byte swizzle layout (the Ut / wUt buffers are free once
                    // MMA_dH and MMA_O have completed) and let TMA store it
                    const uint32_t stg = sbase + C_OFF_OS + wg * 8192;
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch)
                        tc::st_shared_v4(stg + tc::sw128_off(r, ch), __float_as_uint(qh[4 * ch]),
                                         __float_as_uint(qh[4 * ch + 1]),
                                         __float_as_uint(qh[4 * ch + 2]),
                                         __float_as_uint(qh[4 * ch + 3]));
                    tc::fence_async_smem();
                    tc::named_bar(2 + wg, 64);
                    if (q == 2 && lane == 0) {
                        tc::tma_store_2d(&p.tm_o, stg, head * VD + v0, (int)t0);
                        tc::bulk_commit();
                    }
                } else if (r < len) {
                    // a sequence's ragged last chunk (or bf16 output): direct row stores
                    const int64_t orow = ((t0 + r) * H + head) * VD + v0;
                    if constexpr (OBF16) {
                        __nv_bfloat16* op = static_cast<__nv_bfloat16*>(p.o) + orow;
#pragma unroll
                        for (int jj = 0; jj < 32; jj += 8) {
                            uint4 w4;
                            w4.x = tc::pack_bf16(qh[jj], qh[jj + 1]);
                            w4.y = tc::pack_bf16(qh[jj + 2], qh[jj + 3]);
                            w4.z = tc::pack_bf16(qh[jj + 4], qh[jj + 5]);
                            w4.w = tc::pack_bf16(qh[jj + 6], qh[jj + 7]);
                            *reinterpret_cast<uint4*>(op + jj) = w4;
                        }
                    } else {
                        float* op = static_cast<float*>(p.o) + orow;
#pragma unroll
                        for (int jj = 0; jj < 32; jj += 4)
                            *reinterpret_cast<float4*>(op + jj) =
                                make_float4(qh[jj], qh[jj + 1], qh[jj + 2], qh[jj + 3]);
                    }
                }
            }
        }
        if (q == 2 && lane == 0) tc::bulk_wait0();  // output stores complete
        if (p.hT) {
            float* dst = p.hT + hrow;
#pragma unroll
            for (int jj = 0; jj < 32; jj += 4)
                *reinterpret_cast<float4*>(dst + jj) = make_float4(h[jj], h[jj + 1], h[jj + 2], h[jj + 3]);
        }
        if (ct == 0) {
            for (int c = (last_loaded > 0 ? last_loaded - 1 : 0); c <= last_loaded && c < nch; ++c)
                if (c >= 0) drain_wait(&bars[B_FULL + (c & 1)], (c >> 1) & 1);
            if (last_v >= 0) drain_wait(&bars[B_FULLV], last_v & 1);
            if (*abort_flag) {
                tc::mma_commit(&bars[B_DRAIN]);
                drain_wait(&bars[B_DRAIN], 0);
            }
        }
    }
    tc::tc_before_sync();
    __syncthreads();
    tc::cluster_sync();  // no CTA leaves while the other may still touch its memory
    tc::tc_after_sync();
    if (warp == 0) tc::tmem_dealloc(tmem, ncols);
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

// [rows, cols] row-major, 128-byte swizzle; bf16 inputs use 64 x 64 boxes,
// the fp32 output 32-column x 64-row boxes.
inline bool make_map(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols,
                     bool f32 = false) {
    EncodeTiled enc = get_encode();
    if (!enc) return false;
    const uint64_t esz = f32 ? 4 : 2;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * esz};
    cuuint32_t box[2] = {f32 ? 32u : 64u, 64u};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
               const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tcf

// Launches the fused kernel: one cluster of two CTAs per (sequence, head).
// Returns 0 on success, 1 when the tensor maps could not be built, 2 on a
// launch error.
inline int launch_chunk_tc(const ChunkArgs& a, int64_t T_total, bool obf16, cudaStream_t st) {
    tcf::Params p;
    memset(&p, 0, sizeof(p));
    const uint64_t cols = (uint64_t)a.H * 128;
    if (!tcf::make_map(&p.tm_q, a.q, (uint64_t)T_total, cols) ||
        !tcf::make_map(&p.tm_k, a.k, (uint64_t)T_total, cols) ||
        !tcf::make_map(&p.tm_v, a.v, (uint64_t)T_total, cols) ||
        (!obf16 && !tcf::make_map(&p.tm_o, a.o, (uint64_t)T_total, cols, true)))
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
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3((unsigned)nb, 1, 1);
    cfg.blockDim = dim3(tcf::kThreads, 1, 1);
    cfg.dynamicSmemBytes = tcf::SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, p) != cudaSuccess) return 2;
    return 0;
}

}  // namespace gdn
