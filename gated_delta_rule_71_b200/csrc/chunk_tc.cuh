// chunk_tc.cuh -- fused tensor-core chunked forward of the gated delta rule
// (bf16 q/k/v, K = V = 128, fp32 state, fp32 accumulation), sm_100a.
//
// The three GDN steps of ZzCompute (PyTorch Helion Hackathon gallery entry 11)
// -- item 4 "Recompute W/U" (in-chunk cumsum, A, T = (I+A)^-1, W, U), item 2
// "Chunk Forward H" (state recurrence) and item 3 "Chunk Forward O" (chunk
// output) -- run in one launch, so q/k/v/g/beta are read from HBM once and
// o/h_T written once.  The state is carried transposed, S = h^T (value rows,
// key columns, the rule's own orientation).  Per chunk (64 tokens, G2 =
// log2-scaled in-chunk cumsum of g, w_t = 2^(G2_L - G2_t)):
//   A   = strictly-lower beta_r 2^(G2_r-G2_s) (K K^T)_rs,  T = (I + A)^-1
//   P   = lower-incl 2^(G2_r-G2_s) (Q K^T)_rs
//   Tb  = T diag(beta),  W = T diag(beta 2^G2) K
//   Ut^T = V^T Tb^T - S W^T                      ( = (U - W h)^T of the WY form)
//   S'  = 2^G2_L S + (w Ut)^T K
//   o_t = scale (2^G2_t (S Q^T)_{:,t} + (Ut^T P^T)_{:,t})
// Each (sequence, head) runs on a cluster of two CTAs, one per SM:
//  * rank 0, "prep": three warpgroups, each owning every third chunk and its
//    own TMA stage: S_kk = [K; Q] K^T and W on tcgen05, the A and P rows and
//    T by 16x16 blocks.  It assembles [W | Tb | P] (bf16) and the gate factors
//    in its own stage as the stage's inputs fall free, and ships them to the
//    chain CTA's shared memory with one bulk copy that completes on the
//    chain's mbarrier.
//  * rank 1, "chain": four warpgroups carry S in fp32 registers (value row =
//    tensor-memory lane, 32 key columns per warpgroup) and keep its bf16 copy
//    in tensor memory, where it is the A operand of the chain's MMAs, so the
//    serial part is two tcgen05 products per chunk with no shared-memory
//    round trip.  The output comes out of tensor memory transposed: each warp
//    writes 128 contiguous bytes per token.
// TMA loads are issued by the thread that frees a stage.  Every wait is
// bounded: a wait that gives up sets the CTA's abort flag (later waits fall
// through, so every barrier is still reached), records GDN_ERR_TIMEOUT, and
// the issuing threads drain their copies and MMAs before tensor memory is
// released.
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
constexpr int kThreads = 576;  // 16 warps of warpgroup work, an MMA warp and a TMA warp
constexpr int NPREP = 3;  // prep warpgroups (chunks in flight in the prep CTA)
constexpr uint32_t kPolls = 1u << 22;
constexpr float kLog2e = 1.4426950408889634f;

// ---- shared memory, prep CTA
// The stage holds [K half 0 | Q half 0 | K half 1 | Q half 1] (8 KB each) as
// loaded; as its parts fall free it is rewritten in place into the slot image
// sent to the chain CTA: [W half 0 | W half 1 | Tb | P].
constexpr uint32_t SZ_KQ = 32768;
constexpr int AFP = 68;            // fp32 row pitch of A / T
constexpr int XTP = 24;            // pitch of the 16x16 temporaries (conflict-free B fragments)
constexpr uint32_t SZ_AF = 64 * AFP * 4;
constexpr uint32_t SZ_XT = 3 * 16 * XTP * 4;
struct PrepScal {    // per prep warpgroup
    float G2[64];    // in-chunk inclusive cumsum of g, log2 units
    float ginv[64];  // 2^-G2 (only when the chunk's decay stays in fp32 range)
    float gam[64];   // 2^G2
    float beta[64];
    float scan_tmp;
    float pad[3];
};
constexpr uint32_t P_OFF_KQ = 0;                                   // NPREP stages
constexpr uint32_t P_OFF_AF = P_OFF_KQ + NPREP * SZ_KQ;            // NPREP x A
constexpr uint32_t P_OFF_TF = P_OFF_AF + NPREP * SZ_AF;            // NPREP x T
constexpr uint32_t P_OFF_XT = P_OFF_TF + NPREP * SZ_AF;            // NPREP x temporaries
constexpr uint32_t P_OFF_SC = P_OFF_XT + NPREP * SZ_XT;            // NPREP x PrepScal
constexpr uint32_t P_OFF_CS = P_OFF_SC + NPREP * sizeof(PrepScal); // NPREP x staged gate factors
constexpr uint32_t P_END = P_OFF_CS + NPREP * 528;

// ---- shared memory, chain CTA
// K, V and Q each have two buffers of [2 halves][64 tokens][128 B]: a K buffer
// is free once dS of its chunk is done, a V buffer once U0 is, a Q buffer once
// S Q^T is, so each tile is fetched more than a chunk ahead of its use.
constexpr uint32_t SZ_T = 16384;
constexpr uint32_t SZ_SLOT = 32768;  // slot: W [2 key halves][64][128 B] | Tb [64][128 B] | P [64][128 B]
constexpr uint32_t SL_W = 0, SL_TB = 16384, SL_P = 24576;
constexpr uint32_t SZ_OS = 32768;    // output stage: 4 boxes [64 tokens][32 values fp32], 128B swizzle
struct ChainScal {  // per slot, written by the prep CTA (bulk copy)
    float w[64];    // 2^(G2_L - G2)
    float gam[64];  // 2^G2
    float eGL;      // 2^G2_L
    float pad[3];
};
constexpr uint32_t C_OFF_K = 0;                                 // 2 buffers each
constexpr uint32_t C_OFF_V = C_OFF_K + 2 * SZ_T;
constexpr uint32_t C_OFF_Q = C_OFF_V + 2 * SZ_T;
constexpr uint32_t C_OFF_SL = C_OFF_Q + 2 * SZ_T;               // NPREP slots
constexpr uint32_t C_OFF_OS = C_OFF_SL + NPREP * SZ_SLOT;
constexpr uint32_t C_OFF_SC = C_OFF_OS + SZ_OS;                 // NPREP x ChainScal
constexpr uint32_t C_END = C_OFF_SC + NPREP * sizeof(ChainScal);

constexpr uint32_t BODY = (P_END > C_END ? P_END : C_END);
constexpr uint32_t OFF_BAR = (BODY + 15) & ~15u;
constexpr int NBARS = 40;
constexpr uint32_t OFF_MISC = OFF_BAR + NBARS * 8;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 64 + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(sizeof(ChainScal) == 528, "gate-factor image size");

// ---- tensor memory columns
constexpr uint32_t P_TMEM_COLS = 512;  // prep: per warpgroup 128 (S_kk, then W)
constexpr uint32_t C_COL_SB = 0;       // chain: bf16 S (128 keys packed in 64 columns)
constexpr uint32_t C_COL_U = 64;       // Ut^T fp32 (64 tokens)
constexpr uint32_t C_COL_UB = 128;     // Ut^T bf16 (32)
constexpr uint32_t C_COL_WB = 160;     // (w Ut)^T bf16 (32)
constexpr uint32_t C_COL_DS = 192;     // dS fp32 (128 keys)
constexpr uint32_t C_COL_O1 = 320;     // (S Q^T) fp32, two buffers of 64
constexpr uint32_t C_COL_O2 = 448;     // (Ut^T P^T) fp32 (64)
constexpr uint32_t C_TMEM_COLS = 512;

// barrier slots
enum : int {
    B_FULL = 0,   // [NPREP] prep: TMA stage; chain uses [0..1]
    B_MS = 3,     // [NPREP] prep: S_kk ready
    B_FREE = 6,   // [NPREP] prep: chain slot free (remote arrivals)
    B_TPF = 9,    // [NPREP] chain: slot filled (bulk-copy transactions)
    B_MW = 12,    // [NPREP] prep: W ready
    B_MA = 15, B_MD, B_MO, B_DRAIN, B_DRAINP,
    B_S2,         // chain: Ut^T written (16 warp arrivals)
    B_S4,         // chain: bf16 S written (16 warp arrivals)
    B_VF,         // [2] chain: V tile loaded (K tiles use B_FULL 0..1)
    B_QF = B_VF + 2,  // [2] chain: Q tile loaded
    B_KFREE = B_QF + 2,     // [2] chain: K buffer read (dS issued before the commit)
    B_QFREE = B_KFREE + 2,  // [2] chain: Q buffer read (S Q^T)
    B_VFREE = B_QFREE + 2,  // [2] chain: V buffer read (U0)
    B_SLOTDONE = B_VFREE + 2,  // [NPREP] chain: slot consumed (MMA commit + 16 warp arrivals)
};
static_assert(B_SLOTDONE + NPREP <= NBARS, "barrier slots");

// Launch forms of the kernel.  kFused: one cluster of (prep, chain) per
// (sequence, head), the slot images pushed into the chain CTA with
// cluster bulk copies.  kPersist (dense batches): one cooperative launch over
// every SM; CTAs [0, n_chain) carry one chain each, the others build the
// images of every (chunk, head) of the batch in chunk-major order, write each
// to global memory and publish it with a ready flag, which the chain CTA waits
// for (bounded) before it bulk-loads the image into its slot.
enum : int { kFused = 0, kPersist = 1 };
constexpr uint32_t kScalBytes = (uint32_t)sizeof(ChainScal);

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
    // persistent form: images [n_img][SZ_SLOT] then gate factors [n_img][kScalBytes];
    // image gi * H + head for chunk gi = seq * nch_dense + c of the dense batch
    uint8_t* img;
    int nch_dense;
    int n_seq;
    int64_t n_img;
    uint32_t* ready;  // [n_img] image ready flags (zeroed before the launch)
    int n_chain;      // CTAs carrying chains
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

__device__ __forceinline__ uint32_t pack2(float lo, float hi) { return tc::pack_bf16(lo, hi); }

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


template <bool OBF16, int MODE>
__global__ void __launch_bounds__(kThreads, 1) chunk_fwd_tc_kernel(const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t sbase = (raw_u32 + 1023u) & ~1023u;
    uint8_t* base = smem_raw + (sbase - raw_u32);

    uint64_t* bars = reinterpret_cast<uint64_t*>(base + OFF_BAR);
    uint32_t* misc = reinterpret_cast<uint32_t*>(base + OFF_MISC);
    volatile uint32_t* abort_flag = misc + 1;

    const uint32_t rank = MODE == kFused ? tc::cluster_ctarank()
                                         : (blockIdx.x < (unsigned)p.n_chain ? 1u : 0u);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int H = p.H;
    // the (sequence, head) of this cluster or chain CTA (persistent prep CTAs
    // take their (chunk, head) jobs from a strided list instead)
    int head = 0, seq = 0, nch = 0;
    int64_t cs = 0, ce = 0;
    if (MODE == kFused || rank == 1) {
        const int sh = MODE == kFused ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
        head = sh % H;
        const int slot = sh / H;
        seq = p.order ? p.order[slot] : slot;
        if (p.cu) {
            cs = p.cu[seq];
            ce = p.cu[seq + 1];
        } else {
            cs = (int64_t)seq * p.T;
            ce = cs + p.T;
        }
        nch = (int)((ce - cs + C - 1) / C);
    }

    if (threadIdx.x == 0) {
        for (int i = 0; i < NBARS; ++i)
            mbar_init(&bars[i], (i == B_S2 || i == B_S4)                           ? 16u
                                : (i >= B_SLOTDONE && i < B_SLOTDONE + NPREP) ? 17u
                                                                              : 1u);
        misc[1] = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        // chain: arm the slot barriers for the first images before the prep CTA
        // can start a copy (it waits at the cluster barrier below)
        if (MODE == kFused && rank == 1)
            for (int i = 0; i < NPREP; ++i)
                tc::mbar_arrive_expect_tx(&bars[B_TPF + i], SZ_SLOT + (uint32_t)sizeof(ChainScal));
    }
    const uint32_t ncols = rank == 0 ? P_TMEM_COLS : C_TMEM_COLS;
    if (warp == 0) tc::tmem_alloc(&misc[0], ncols);
    tc::tc_before_sync();
    __syncthreads();
    if (MODE == kFused) tc::cluster_sync();  // both CTAs' barriers initialised before any remote arrive
    tc::tc_after_sync();
    const uint32_t tmem = misc[0];

    if (rank == 0) {
        // ================================================================ prep
        const int wg = warp >> 2;  // warpgroups 1..NPREP work
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
            uint64_t* mW = &bars[B_MW + pg];
            uint64_t* sfree = &bars[B_FREE + pg];
            const uint32_t tcol = tmem + 128u * pg;  // S_kk (64 columns), then W (128)
            // this warpgroup's slot in the chain CTA, and the staged gate factors
            uint32_t r_sl = 0, r_sc = 0, r_tpf = 0;
            if (MODE == kFused) {
                r_sl = tc::mapa(sbase + C_OFF_SL + pg * SZ_SLOT, 1);
                r_sc = tc::mapa(sbase + C_OFF_SC + pg * (uint32_t)sizeof(ChainScal), 1);
                r_tpf = tc::mapa(smem_u32(&bars[B_TPF + pg]), 1);
            }
            ChainScal* cst = reinterpret_cast<ChainScal*>(base + P_OFF_CS + pg * 528);
            const uint32_t cst_u32 = sbase + P_OFF_CS + pg * 528;
            const uint32_t idS = tc::idesc_bf16(128, 64, 0, 0);
            const uint32_t idW = tc::idesc_bf16(128, 128, 0, 1);
            // this warpgroup's k-th job: chunk c (first row t0, sequence end ce) of head
            struct Job {
                int head;
                int64_t t0, ce, gi;
            };
            const int64_t chains = (int64_t)p.n_seq * H;
            const int64_t njobs = MODE == kFused ? 0 : chains * p.nch_dense;
            auto job_at = [&](int k, Job& jb) -> bool {
                if constexpr (MODE == kFused) {
                    const int c = pg + k * NPREP;
                    if (c >= nch) return false;
                    jb.head = head;
                    jb.t0 = cs + (int64_t)C * c;
                    jb.ce = ce;
                    jb.gi = 0;
                    return true;
                } else {
                    // chunk-major over the (dense) batch's chains, so every chain's
                    // chunk c is built before any chain's chunk c + 1
                    const int pb = (int)blockIdx.x - p.n_chain, npb = (int)gridDim.x - p.n_chain;
                    const int64_t j = (int64_t)pb * NPREP + pg + (int64_t)k * npb * NPREP;
                    if (j >= njobs) return false;
                    const int64_t c = j / chains, ch = j - c * chains;
                    const int64_t sq = ch / H;
                    jb.head = (int)(ch - sq * H);
                    jb.gi = sq * p.nch_dense + c;
                    jb.t0 = sq * p.T + (int64_t)C * c;
                    jb.ce = (sq + 1) * p.T;
                    return true;
                }
            };
            auto issue_load = [&](const Job& jb) {
                const int y = (int)jb.t0;
                tc::mbar_arrive_expect_tx(full, SZ_KQ);
                tc::tma_load_2d(kq_p + 0, &p.tm_k, jb.head * KD + 0, y, full);
                tc::tma_load_2d(kq_p + 8192, &p.tm_q, jb.head * KD + 0, y, full);
                tc::tma_load_2d(kq_p + 16384, &p.tm_k, jb.head * KD + 64, y, full);
                tc::tma_load_2d(kq_p + 24576, &p.tm_q, jb.head * KD + 64, y, full);
            };
            Job jb, jn;
            bool have = job_at(0, jb);
            int loads = 0;
            if (pt == 0 && have) {
                tc::prefetch_tmap(&p.tm_q);
                tc::prefetch_tmap(&p.tm_k);
                issue_load(jb);
                loads = 1;
            }
            for (int n = 0; have; ++n) {
                const int64_t t0 = jb.t0;
                const int len = (int)((jb.ce - t0) < C ? (jb.ce - t0) : C);
                const int hd = jb.head;
                float gv = 0.f, bv = 0.f;
                if (pt < len) {
                    gv = p.g[(t0 + pt) * H + hd];
                    bv = p.beta[(t0 + pt) * H + hd];
                }
                wait(full, n & 1, abort_flag);
                if (pt == 0) {
                    tc::tc_after_sync();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                        tc::mma_bf16(tcol, tc::sdesc_sw128(kq + off, 16, 1024),
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
                    ls->beta[pt] = bv;
                    cst->w[pt] = exp2f(G2L - x);
                    cst->gam[pt] = gm;
                    if (pt == 0) cst->eGL = exp2f(G2L);
                }
                // S_kk row of this thread: rows 0-63 = K K^T, rows 64-127 = Q K^T
                wait(mS, n & 1, abort_flag);
                tc::tc_after_sync();
                float sv[64];
                {
                    const uint32_t ta = tcol + ((uint32_t)(32 * pw) << 16);
                    tc::tmem_ld32(ta, *reinterpret_cast<float(*)[32]>(sv));
                    tc::tmem_ld32(ta + 32, *reinterpret_cast<float(*)[32]>(sv + 32));
                    tc::tmem_wait_ld();
                }
                tc::named_bar(bid, 128);  // ginv / gam / beta visible
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
                    // P row -> the slot image (over the stage's second Q half)
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch)
                        tc::st_shared_v4(kq + SL_P + tc::sw128_off(r, ch),
                                         pack2(sv[8 * ch + 0], sv[8 * ch + 1]),
                                         pack2(sv[8 * ch + 2], sv[8 * ch + 3]),
                                         pack2(sv[8 * ch + 4], sv[8 * ch + 5]),
                                         pack2(sv[8 * ch + 6], sv[8 * ch + 7]));
                }
                tc::tc_before_sync();
                tc::named_bar(bid, 128);  // A rows complete
                invert_unit_lower(Af, Tf, Xt, pw, lane, bid);
                uint32_t tb_words[16];  // Tb = T diag(beta), placed once W is done
                {
                    // T rows -> T diag(beta 2^G2) over the stage's first Q half (the A
                    // operand of W); Tb kept in registers
                    const int r = pt >> 1, hf = pt & 1;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const int ch = 4 * hf + q4;
                        float t8[8], u8[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int col = 8 * ch + e;
                            const float tv = (col <= r) ? Tf[r * AFP + col] : 0.f;
                            t8[e] = tv * ls->beta[col];
                            u8[e] = t8[e] * ls->gam[col];
                        }
#pragma unroll
                        for (int e = 0; e < 4; ++e) tb_words[4 * q4 + e] = pack2(t8[2 * e], t8[2 * e + 1]);
                        tc::st_shared_v4(kq + 8192 + tc::sw128_off(r, ch), pack2(u8[0], u8[1]),
                                         pack2(u8[2], u8[3]), pack2(u8[4], u8[5]),
                                         pack2(u8[6], u8[7]));
                    }
                }
                tc::fence_async_smem();
                tc::tc_before_sync();
                tc::named_bar(bid, 128);
                if (pt == 0) {
                    // W = [T diag(beta 2^G2); junk] K  (M=128, N=128 keys, K=64 tokens)
                    tc::tc_after_sync();
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc::mma_bf16(tcol, tc::sdesc_sw128(kq + 8192 + kk * 32, 16, 1024),
                                     tc::sdesc_sw128(kq + kk * 2048, 16384, 1024), idW, kk > 0);
                    tc::mma_commit(mW);
                }
                wait(mW, n & 1, abort_flag);
                tc::tc_after_sync();
                if (pw < 2) {
                    // W row r (keys 0..127) -> bf16 slot image, over K half 0 / the A tile
                    const int r = pt;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        float xw[32];
                        tc::tmem_ld32(tcol + ((uint32_t)(32 * pw) << 16) + 32 * q4, xw);
                        tc::tmem_wait_ld();
                        const int hf = q4 >> 1;
#pragma unroll
                        for (int cc = 0; cc < 4; ++cc) {
                            const int ch = 4 * (q4 & 1) + cc;
                            tc::st_shared_v4(kq + SL_W + hf * 8192 + tc::sw128_off(r, ch),
                                             pack2(xw[8 * cc + 0], xw[8 * cc + 1]),
                                             pack2(xw[8 * cc + 2], xw[8 * cc + 3]),
                                             pack2(xw[8 * cc + 4], xw[8 * cc + 5]),
                                             pack2(xw[8 * cc + 6], xw[8 * cc + 7]));
                        }
                    }
                }
                {
                    // Tb over K half 1 (W has read it)
                    const int r = pt >> 1, hf = pt & 1;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        tc::st_shared_v4(kq + SL_TB + tc::sw128_off(r, 4 * hf + q4),
                                         tb_words[4 * q4], tb_words[4 * q4 + 1],
                                         tb_words[4 * q4 + 2], tb_words[4 * q4 + 3]);
                }
                tc::fence_async_smem();
                tc::tc_before_sync();
                tc::named_bar(bid, 128);
                const bool more = job_at(n + 1, jn);
                if (pt == 0) {
                    // hand the slot image on (to the chain CTA, or to global memory),
                    // then reuse the stage
                    if constexpr (MODE == kFused) {
                        if (n >= 1) wait(sfree, (n - 1) & 1, abort_flag, true);
                        tc::bulk_s2cluster(r_sl, kq, SZ_SLOT, r_tpf);
                        tc::bulk_s2cluster(r_sc, cst_u32, kScalBytes, r_tpf);
                    } else {
                        const int64_t ii = jb.gi * H + hd;
                        tc::bulk_s2g(p.img + ii * SZ_SLOT, kq, SZ_SLOT);
                        tc::bulk_s2g(p.img + p.n_img * SZ_SLOT + ii * kScalBytes, cst_u32,
                                     kScalBytes);
                    }
                    tc::bulk_commit();
                    tc::bulk_wait_read0();
                    if (more && !*abort_flag) {
                        issue_load(jn);
                        ++loads;
                    }
                    if constexpr (MODE == kPersist) {
                        // publish: the image's writes complete, then the ready flag
                        tc::bulk_wait0();
                        tc::fence_proxy_async_global();
                        tc::st_release_gpu_u32(p.ready + jb.gi * H + hd, 1u);
                    }
                }
                jb = jn;
                have = more;
            }
            if (pt == 0) {
                // never leave with a copy or an MMA in flight
                tc::bulk_wait0();
                if (loads > 0) drain_wait(full, (loads - 1) & 1);
                if (*abort_flag) {
                    tc::mma_commit(&bars[B_DRAINP]);
                    drain_wait(&bars[B_DRAINP], 0);
                }
            }
        }
    } else {
        // =============================================================== chain
        // warps 0-15: four warpgroups, warpgroup wg owns key columns 32wg.. of S and
        // tokens 16wg.. of the per-chunk tiles; warp 16: MMA and TMA issue
        uint64_t* mA = &bars[B_MA];
        uint64_t* mD = &bars[B_MD];
        uint64_t* mO = &bars[B_MO];
        uint64_t* s2 = &bars[B_S2];
        uint64_t* s4 = &bars[B_S4];
        constexpr uint32_t kSlotTx = SZ_SLOT + (uint32_t)sizeof(ChainScal);
        if (warp == 17) {
            if (lane == 0) {
                // TMA warp: K, V and Q tiles (two buffers each, buffer c & 1) as their
                // buffers fall free, and the slots back to the prep CTA once consumed
                const uint32_t r_free0 = MODE == kFused ? tc::mapa(smem_u32(&bars[B_FREE]), 0) : 0u;
                // persistent form: this chain's images in global memory
                const int64_t gi0 = MODE == kFused ? 0 : (int64_t)seq * p.nch_dense;
                int last_img = -1;
                auto load_img = [&](int c) {
                    if (*abort_flag) return;
                    const int j = c % NPREP;
                    const int64_t ii = (gi0 + c) * H + head;
                    if constexpr (MODE == kPersist) {
                        // wait (bounded) for the prep CTAs to publish this image
                        uint32_t i = 0;
                        while (tc::ld_acquire_gpu_u32(p.ready + ii) == 0u) {
                            if (++i == kPolls || *abort_flag) {
                                if (!*abort_flag) {
                                    *abort_flag = 1u;
                                    record_status(GDN_ERR_TIMEOUT);
                                }
                                return;
                            }
                        }
                        tc::fence_proxy_async_global();
                    }
                    tc::mbar_arrive_expect_tx(&bars[B_TPF + j], kSlotTx);
                    tc::bulk_g2s(sbase + C_OFF_SL + j * SZ_SLOT, p.img + ii * SZ_SLOT, SZ_SLOT,
                                 &bars[B_TPF + j]);
                    tc::bulk_g2s(sbase + C_OFF_SC + j * kScalBytes,
                                 p.img + p.n_img * SZ_SLOT + ii * kScalBytes, kScalBytes,
                                 &bars[B_TPF + j]);
                    last_img = c;
                };
                int last[3] = {-1, -1, -1};
                auto load = [&](int kind, int c) {
                    if (*abort_flag) return;  // at most one copy in flight per buffer
                    const int y = (int)(cs + (int64_t)C * c);
                    const uint32_t off = (kind == 0 ? C_OFF_K : kind == 1 ? C_OFF_V : C_OFF_Q) +
                                         (c & 1) * SZ_T;
                    uint64_t* bar = &bars[(kind == 0 ? B_FULL : kind == 1 ? B_VF : B_QF) + (c & 1)];
                    const CUtensorMap* m = kind == 0 ? &p.tm_k : kind == 1 ? &p.tm_v : &p.tm_q;
                    const int x0 = head * (kind == 1 ? VD : KD);
                    tc::mbar_arrive_expect_tx(bar, SZ_T);
                    tc::tma_load_2d(base + off, m, x0, y, bar);
                    tc::tma_load_2d(base + off + 8192, m, x0 + 64, y, bar);
                    last[kind] = c;
                };
                tc::prefetch_tmap(&p.tm_k);
                tc::prefetch_tmap(&p.tm_v);
                tc::prefetch_tmap(&p.tm_q);
                for (int c = 0; c < 2 && c < nch; ++c) {
                    load(1, c);
                    load(0, c);
                    load(2, c);
                }
                if (MODE == kPersist)
                    for (int c = 0; c < NPREP && c < nch; ++c) load_img(c);
                for (int c = 0; c < nch; ++c) {
                    const uint32_t ph = (c >> 1) & 1;
                    if (c + 2 < nch) {
                        if (wait(&bars[B_VFREE + (c & 1)], ph, abort_flag)) load(1, c + 2);
                        if (wait(&bars[B_QFREE + (c & 1)], ph, abort_flag)) load(2, c + 2);
                        if (wait(&bars[B_KFREE + (c & 1)], ph, abort_flag)) load(0, c + 2);
                    }
                    if (c + NPREP < nch) {
                        // re-arm the slot's barrier for the next image, then hand the
                        // slot back to the prep CTA (or fetch that image)
                        const int j = c % NPREP;
                        if (wait(&bars[B_SLOTDONE + j], (c / NPREP) & 1, abort_flag)) {
                            if constexpr (MODE == kFused) {
                                tc::mbar_arrive_expect_tx(&bars[B_TPF + j], kSlotTx);
                                tc::mbar_arrive_cluster(r_free0 + 8 * j);
                            } else {
                                load_img(c + NPREP);
                            }
                        }
                    }
                }
                for (int c = last_img - NPREP + 1; c <= last_img; ++c)
                    if (c >= 0) drain_wait(&bars[B_TPF + c % NPREP], (c / NPREP) & 1);
                // never leave with a copy in flight
                for (int kind = 0; kind < 3; ++kind) {
                    uint64_t* b0 = &bars[kind == 0 ? B_FULL : kind == 1 ? B_VF : B_QF];
                    for (int c = last[kind] - 1; c <= last[kind]; ++c)
                        if (c >= 0) drain_wait(b0 + (c & 1), (c >> 1) & 1);
                }
            }
        } else if (warp == 16) {
            {
                // MMA warp: the dependent products (U, dS) are issued as soon as their
                // inputs are written; the output products fill the gaps.  All 32 lanes
                // run it and one elected lane issues each product (warp-uniform
                // operands give a shorter issue sequence than a lone lane).
                const uint32_t idU0 = tc::idesc_bf16(128, 64, 1, 0);
                const uint32_t id1 = tc::idesc_bf16(128, 64, 0, 0) | tc::kNegateA;
                const uint32_t idO = tc::idesc_bf16(128, 64, 0, 0);
                const uint32_t id2 = tc::idesc_bf16(128, 128, 0, 1);
                // U0 for chunk c: D_U = V^T Tb^T  (A = V tile MN-major, B = Tb K-major)
                auto issue_u0 = [&](int c) {
                    wait(&bars[B_VF + (c & 1)], (c >> 1) & 1, abort_flag);
                    __syncwarp();
                    wait(&bars[B_TPF + c % NPREP], (c / NPREP) & 1, abort_flag);
                    __syncwarp();
                    tc::tc_after_sync();
                    const uint32_t vt = sbase + C_OFF_V + (c & 1) * SZ_T;
                    const uint32_t tb = sbase + C_OFF_SL + (c % NPREP) * SZ_SLOT + SL_TB;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc::mma_bf16_w(tmem + C_COL_U, tc::sdesc_sw128(vt + kk * 2048, 8192, 1024),
                                     tc::sdesc_sw128(tb + kk * 32, 16, 1024), idU0, kk > 0);
                    tc::mma_commit_w(&bars[B_VFREE + (c & 1)]);
                };
                if (nch > 0) issue_u0(0);
                for (int c = 0; c < nch; ++c) {
                    const uint32_t sl = sbase + C_OFF_SL + (c % NPREP) * SZ_SLOT;
                    wait(s4, c & 1, abort_flag);  // bf16 S of this chunk written
                    __syncwarp();
                    tc::tc_after_sync();
                    // Ut^T = V^T Tb^T - S W^T
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        tc::mma_bf16_ts_w(tmem + C_COL_U, tmem + C_COL_SB + 8 * kk,
                                        tc::sdesc_sw128(sl + SL_W + (kk >> 2) * 8192 + (kk & 3) * 32,
                                                        16, 1024),
                                        id1, 1);
                    tc::mma_commit_w(mA);
                    // S Q^T for the output
                    wait(&bars[B_QF + (c & 1)], (c >> 1) & 1, abort_flag);
                    __syncwarp();
                    tc::tc_after_sync();
                    const uint32_t qt = sbase + C_OFF_Q + (c & 1) * SZ_T;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        tc::mma_bf16_ts_w(tmem + C_COL_O1 + 64u * (c & 1), tmem + C_COL_SB + 8 * kk,
                                        tc::sdesc_sw128(qt + (kk >> 2) * 8192 + (kk & 3) * 32, 16,
                                                        1024),
                                        idO, kk > 0);
                    tc::mma_commit_w(&bars[B_QFREE + (c & 1)]);
                    wait(s2, c & 1, abort_flag);  // Ut^T, (w Ut)^T written; output(c-1) done
                    __syncwarp();
                    wait(&bars[B_FULL + (c & 1)], (c >> 1) & 1, abort_flag);
                    __syncwarp();
                    tc::tc_after_sync();
                    // dS = (w Ut)^T K
                    const uint32_t kt = sbase + C_OFF_K + (c & 1) * SZ_T;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc::mma_bf16_ts_w(tmem + C_COL_DS, tmem + C_COL_WB + 8 * kk,
                                        tc::sdesc_sw128(kt + kk * 2048, 8192, 1024), id2, kk > 0);
                    tc::mma_commit_w(mD);
                    tc::mma_commit_w(&bars[B_KFREE + (c & 1)]);
                    // Ut^T P^T
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc::mma_bf16_ts_w(tmem + C_COL_O2, tmem + C_COL_UB + 8 * kk,
                                        tc::sdesc_sw128(sl + SL_P + kk * 32, 16, 1024), idO,
                                        kk > 0);
                    tc::mma_commit_w(mO);
                    tc::mma_commit_w(&bars[B_SLOTDONE + c % NPREP]);
                    // next chunk's U0 (D_U was read before s2)
                    if (c + 1 < nch) issue_u0(c + 1);
                }
                // never leave with an MMA in flight
                tc::mma_commit_w(&bars[B_DRAIN]);
                drain_wait(&bars[B_DRAIN], 0);
                __syncwarp();
            }
        } else {
            const int wg = warp >> 2, q = warp & 3;
            const int vr = 32 * q + lane;  // value row of S = tensor-memory lane
            const uint32_t lane_base = (uint32_t)(32 * q) << 16;
            const int k0 = 32 * wg;        // this warpgroup's 32 key columns of S
            const int64_t hb0 = (int64_t)(seq * H + head) * KD * VD;
            // S[vr][k0 .. k0+31] = h[k][vr]
            float S[32];
#pragma unroll
            for (int jj = 0; jj < 32; ++jj)
                S[jj] = p.h0 ? p.h0[hb0 + (int64_t)(k0 + jj) * VD + vr] : 0.f;
            auto store_sb = [&]() {
                uint32_t w16[16];
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) w16[jj] = pack2(S[2 * jj], S[2 * jj + 1]);
                tc::tmem_st16(tmem + lane_base + C_COL_SB + 16u * wg, w16);
                tc::tmem_wait_st();
                tc::tc_before_sync();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(s4);
            };
            store_sb();
            const bool issuer = (wg == 0 && lane == 0);  // one thread per value quarter
            auto output = [&](int c) {
                // o_t = scale (2^G2_t (S Q^T)[vr][t] + (Ut^T P^T)[vr][t]) for 16 tokens
                const int64_t t0 = cs + (int64_t)C * c;
                const int len = (int)((ce - t0) < C ? (ce - t0) : C);
                const ChainScal* scp =
                    reinterpret_cast<const ChainScal*>(base + C_OFF_SC) + (c % NPREP);
                wait(mO, c & 1, abort_flag);
                tc::tc_after_sync();
                float o1[16], o2[16];
                tc::tmem_ld16(tmem + lane_base + C_COL_O1 + 64u * (c & 1) + 16u * wg, o1);
                tc::tmem_ld16(tmem + lane_base + C_COL_O2 + 16u * wg, o2);
                tc::tmem_wait_ld();
                const float scl = p.scale;
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) o1[jj] = scl * fmaf(scp->gam[16 * wg + jj], o1[jj], o2[jj]);
                if (!OBF16 && len == C) {
                    // stage the 64 x 32 block of this value quarter (128-byte swizzle),
                    // then one TMA store per quarter
                    const uint32_t stg = sbase + C_OFF_OS + q * 8192;
                    if (issuer) tc::bulk_wait_read0();  // previous chunk's store read the stage
                    tc::named_bar(1 + q, 128);
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj) {
                        const int t = 16 * wg + jj;
                        asm volatile("st.shared.f32 [%0], %1;" ::"r"(stg + tc::sw128_off(t, lane >> 2) +
                                                                    4 * (lane & 3)),
                                     "f"(o1[jj])
                                     : "memory");
                    }
                    tc::fence_async_smem();
                    tc::named_bar(1 + q, 128);
                    if (issuer) {
                        tc::tma_store_2d(&p.tm_o, stg, head * VD + 32 * q, (int)t0);
                        tc::bulk_commit();
                    }
                } else {
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj) {
                        const int t = 16 * wg + jj;
                        if (t < len) {
                            const int64_t oi = ((t0 + t) * H + head) * VD + vr;
                            if constexpr (OBF16)
                                static_cast<__nv_bfloat16*>(p.o)[oi] = __float2bfloat16_rn(o1[jj]);
                            else
                                static_cast<float*>(p.o)[oi] = o1[jj];
                        }
                    }
                }
            };
            // this warp is done with the gate factors of chunk c
            auto slot_consumed = [&](int c) {
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&bars[B_SLOTDONE + c % NPREP]);
            };
            for (int c = 0; c < nch; ++c) {
                const int j = c % NPREP;
                const ChainScal* sc = reinterpret_cast<const ChainScal*>(base + C_OFF_SC) + j;
                wait(&bars[B_TPF + j], (c / NPREP) & 1, abort_flag);
                if (c >= 1) output(c - 1);  // overlaps this chunk's MMA latency
                if (c >= 1) slot_consumed(c - 1);
                wait(mA, c & 1, abort_flag);
                tc::tc_after_sync();
                {
                    // Ut^T columns 16wg..16wg+15 -> bf16 Ut^T and (w Ut)^T in tensor memory
                    float u[16];
                    tc::tmem_ld16(tmem + lane_base + C_COL_U + 16u * wg, u);
                    tc::tmem_wait_ld();
                    uint32_t ub[8], wb[8];
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj) {
                        const float w0 = sc->w[16 * wg + 2 * jj], w1 = sc->w[16 * wg + 2 * jj + 1];
                        ub[jj] = pack2(u[2 * jj], u[2 * jj + 1]);
                        wb[jj] = pack2(w0 * u[2 * jj], w1 * u[2 * jj + 1]);
                    }
                    tc::tmem_st8(tmem + lane_base + C_COL_UB + 8u * wg, ub);
                    tc::tmem_st8(tmem + lane_base + C_COL_WB + 8u * wg, wb);
                    tc::tmem_wait_st();
                    tc::tc_before_sync();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(s2);
                }
                wait(mD, c & 1, abort_flag);
                tc::tc_after_sync();
                {
                    // S <- 2^G2_L S + dS, and its bf16 copy for the next chunk
                    const float e = sc->eGL;
                    float d[32];
                    tc::tmem_ld32(tmem + lane_base + C_COL_DS + 32u * wg, d);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) S[jj] = fmaf(e, S[jj], d[jj]);
                    store_sb();  // S Q^T and MMA_1 of this chunk completed before dS
                }
            }
            if (nch >= 1) {
                output(nch - 1);
                slot_consumed(nch - 1);
            }
            if (issuer) tc::bulk_wait0();  // output stores complete
            if (p.hT) {
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) p.hT[hb0 + (int64_t)(k0 + jj) * VD + vr] = S[jj];
            }
        }
    }
    tc::tc_before_sync();
    __syncthreads();
    if (MODE == kFused) tc::cluster_sync();  // no CTA leaves while the other may still touch its memory
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

// Launches the kernel: with `img` null, one cluster of two CTAs per (sequence,
// head); otherwise (a dense batch) the persistent form, one cooperative launch
// of one CTA per SM, with the slot images and their ready flags in `img` /
// `ready` (n_img of each).  Returns 0 on success, 1 when the tensor maps could
// not be built, 2 on a launch error.
inline int launch_chunk_tc(const ChunkArgs& a, int64_t T_total, bool obf16, cudaStream_t st,
                           uint8_t* img = nullptr, uint32_t* ready = nullptr, int64_t n_img = 0,
                           int n_sms = 148) {
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
    p.img = img;
    p.nch_dense = a.cu_seqlens ? 0 : (int)((a.T + tcf::C - 1) / tcf::C);
    p.n_seq = a.n_seq;
    p.n_img = n_img;
    p.ready = ready;
    const bool persist = img && ready && !a.cu_seqlens;
    using KernFn = void (*)(tcf::Params);
    KernFn kern = persist ? (obf16 ? tcf::chunk_fwd_tc_kernel<true, tcf::kPersist>
                                   : tcf::chunk_fwd_tc_kernel<false, tcf::kPersist>)
                          : (obf16 ? tcf::chunk_fwd_tc_kernel<true, tcf::kFused>
                                   : tcf::chunk_fwd_tc_kernel<false, tcf::kFused>);
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)tcf::SMEM_BYTES) != cudaSuccess)
        return 2;
    const int64_t chains = (int64_t)a.n_seq * a.H;
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.blockDim = dim3(tcf::kThreads, 1, 1);
    cfg.dynamicSmemBytes = tcf::SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    if (persist) {
        // the chains on CTAs [0, chains), the prep on every other SM; all CTAs
        // resident at once (cooperative), since chain CTAs wait on prep CTAs
        p.n_chain = (int)chains;
        if (cudaMemsetAsync(ready, 0, (size_t)n_img * 4, st) != cudaSuccess) return 2;
        cfg.gridDim = dim3((unsigned)n_sms, 1, 1);
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
    } else {
        cfg.gridDim = dim3((unsigned)(chains * 2), 1, 1);
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
    }
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, p) != cudaSuccess) return 2;
    return 0;
}

}  // namespace gdn
