// chunk_tc.cuh -- fused tensor-core chunked forward of the gated delta rule
// (bf16 q/k/v, K = V = 128, fp32 state, fp32 accumulation), sm_100a.
//
// The three GDN steps of ZzCompute (PyTorch Helion Hackathon gallery entry 11)
// -- item 4 "Recompute W/U" (in-chunk cumsum, A, T = (I+A)^-1, W, U), item 2
// "Chunk Forward H" (state recurrence) and item 3 "Chunk Forward O" (chunk
// output) -- run in one launch, so q/k/v/g/beta are read from HBM once and
// o/h_T written once.  The state is carried transposed, S = h^T (value rows,
// key columns, the rule's own orientation).  Per chunk (64 tokens, G2 =
// log2-scaled in-chunk cumsum of g, gam_t = 2^G2_t, w_t = 2^(G2_L - G2_t)):
//   A    = strictly-lower beta_r 2^(G2_r-G2_s) (K K^T)_rs,  T = (I + A)^-1
//   P    = lower-incl 2^(G2_r-G2_s) (Q K^T)_rs
//   Tb   = T diag(beta),  T' = T diag(beta gam),  W = T' K
//   Ut^T = V^T Tb^T - S W^T                      ( = (U - W h)^T of the WY form)
//   S'   = 2^G2_L S + (w Ut)^T K
//   o_t  = scale (gam_t (S Q^T)_{:,t} + (Ut^T P^T)_{:,t})
// Each (sequence, head) runs on a cluster of R + 1 CTAs, one per SM (R = 1, or
// 2-3 when the chains leave SMs idle):
//  * ranks 0..R-1, "prep": three warpgroups each; prep CTA r takes the chunks
//    c with (c / 3) % R == r, its warpgroup j those with c % 3 == j, each
//    warpgroup with its own K/Q stage and image buffer.  S_kk = [K; Q] K^T on
//    tcgen05; the A and P rows from it; T by 16x16 blocks (substitution on the
//    diagonal, warp-level tf32 MMAs off it).  The image [T' | Tb | P] (bf16)
//    and the gate factors go to the chain CTA's slot c % 3 with bulk copies
//    that complete on the chain's mbarrier.  The K/Q stage is refilled as soon
//    as S_kk has read it, so the warpgroup's next chunk loads during this
//    chunk's inverse.
//  * rank R, "chain": four warpgroups carry S in fp32 registers (value row =
//    tensor-memory lane, 32 key columns per warpgroup) and keep its bf16 copy
//    in tensor memory, where it is the A operand of the chain's MMAs, so the
//    serial part is two tcgen05 products per chunk (Ut^T, then dS) with no
//    shared-memory round trip of the state.  W^T = K^T T'^T is formed on
//    this SM one chunk ahead, from the K tile it loads anyway.  The output is
//    staged in a swizzled fp32 tile that a store warp writes with TMA while
//    the next chunk runs.  A loader thread keeps K, V, Q tiles in flight
//    (three, two and one buffers) and hands each slot back to the prep CTA
//    that fills it next; it never blocks on one resource while another is
//    ready.
// Every wait is bounded: a wait that gives up sets the CTA's abort flag (later
// waits fall through, so every barrier is still reached), records
// GDN_ERR_TIMEOUT, and the issuing threads drain their copies and MMAs before
// tensor memory is released.
#pragma once

#include <cudaTypedefs.h>

#include <mutex>
#include <utility>

#include "chunk_simt.cuh"
#include "tc_ptx.cuh"

namespace gdn {

constexpr bool kTcAvailable = true;

namespace tcf {

constexpr int C = 64;    // chunk
constexpr int KD = 128;  // key dim
constexpr int VD = 128;  // value dim
constexpr int kThreads = 608;  // chain CTA: 16 state warps, MMA, loader and store warps
constexpr int NPREP = 3;       // prep warpgroups = image slots
// chain CTA warp roles: state warps 0-15 (four warpgroups; they also stage the
// output), then the MMA, loader and output-store warps
constexpr int NSW = 16;  // state warps
constexpr int W_MMA = 16, W_LOAD = 17, W_STORE = 18;
constexpr uint32_t kPolls = 1u << 22;
constexpr uint32_t kIdleLimit = 1u << 27;  // loader: polls without progress before giving up
constexpr float kLog2e = 1.4426950408889634f;

// ---- the image of one chunk: three 64 x 64 bf16 tiles in the 128-byte swizzle
// (each 1024-byte aligned) [T' | Tb | P], and the gate factors (528 bytes), which
// the chain keeps in a ring of NFAC entries so that a slot can take the next
// image as soon as its tiles are spent, while the factors are still read.
constexpr uint32_t SL_TP = 0;       // T'  = T diag(beta gam)   [row r][col s]
constexpr uint32_t SL_TB = 8192;    // Tb  = T diag(beta)
constexpr uint32_t SL_P = 16384;    // P' = scale P
constexpr uint32_t SZ_TILES = 24576;
constexpr int NFAC = 2 * 3;         // gate-factor ring (two images per slot)
struct ChainScal {
    float w[64];    // 2^(G2_L - G2)
    float gam[64];  // scale * 2^G2 (the output's inter-chunk factor)
    float eGL;      // 2^G2_L
    float pad[3];
};
constexpr uint32_t kScalBytes = (uint32_t)sizeof(ChainScal);
static_assert(kScalBytes == 528, "gate-factor image size");
constexpr uint32_t kImgTx = SZ_TILES + kScalBytes;  // bytes one image delivers

// ---- shared memory, prep CTA: per warpgroup a K/Q stage [K h0 | Q h0 | K h1 | Q h1]
// (8 KB each, h = key half), an image buffer, the fp32 A / T^T matrix and scalars
constexpr uint32_t SZ_KQ = 32768;
constexpr int AP = 68;        // fp32 row pitch of A / T^T
constexpr int XP = 20;        // pitch of the 16x16 scratch blocks of the inverse
constexpr uint32_t SZ_AT = 64 * AP * 4;
struct PrepScal {
    float G2[64];    // in-chunk inclusive cumsum of g, log2 units
    float gam[64];   // 2^G2
    float beta[64];
    float ginv[64];  // 2^-G2 (used only when the chunk's total decay stays above 2^-126)
    float tmp[4];
};
constexpr uint32_t P_OFF_KQ = 0;
constexpr uint32_t P_OFF_IMG = P_OFF_KQ + NPREP * SZ_KQ;
constexpr uint32_t P_OFF_AT = P_OFF_IMG + NPREP * SZ_TILES;
constexpr uint32_t P_OFF_SC = P_OFF_AT + NPREP * SZ_AT;
constexpr uint32_t P_OFF_PS = P_OFF_SC + NPREP * kScalBytes;
constexpr uint32_t P_END = P_OFF_PS + NPREP * (uint32_t)sizeof(PrepScal);
static_assert(10 * 16 * XP * 4 <= SL_P, "inverse scratch fits below the P tile");

// ---- shared memory, chain CTA
constexpr uint32_t SZ_T = 16384;  // one K, V or Q tile: [2 halves][64 tokens][128 B]
constexpr int NKB = 3, NVB = 2, NQB = 1;
constexpr uint32_t C_OFF_K = 0;
constexpr uint32_t C_OFF_V = C_OFF_K + NKB * SZ_T;
constexpr uint32_t C_OFF_Q = C_OFF_V + NVB * SZ_T;
constexpr uint32_t C_OFF_SL = C_OFF_Q + NQB * SZ_T;    // NPREP image slots
constexpr uint32_t C_OFF_WT = C_OFF_SL + NPREP * SZ_TILES;  // W^T bf16 [128 keys][64 tokens]
constexpr uint32_t C_OFF_OUT = C_OFF_WT + 16384;           // fp32 output stage: 4 x [64][32]
constexpr uint32_t C_OFF_SC = C_OFF_OUT + 32768;           // NFAC x gate factors
constexpr uint32_t C_END = C_OFF_SC + NFAC * kScalBytes;

constexpr uint32_t BODY = (P_END > C_END ? P_END : C_END);
constexpr uint32_t OFF_BAR = (BODY + 15) & ~15u;
constexpr int NBARS = 44;
constexpr uint32_t OFF_MISC = OFF_BAR + NBARS * 8;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 64 + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// ---- tensor memory columns
constexpr uint32_t P_TMEM_COLS = 256;  // prep: S_kk of warpgroup g at 64 g
constexpr uint32_t C_COL_SB = 0;       // chain: bf16 S (128 keys packed in 64 columns)
constexpr uint32_t C_COL_U = 64;       // Ut^T fp32 (64 tokens)
constexpr uint32_t C_COL_UB = 128;     // Ut^T bf16 (32)
constexpr uint32_t C_COL_WB = 160;     // (w Ut)^T bf16 (32)
constexpr uint32_t C_COL_DS = 192;     // dS fp32 (128 keys)
constexpr uint32_t C_COL_O1 = 320;     // S Q^T fp32 (64)
constexpr uint32_t C_COL_O2 = 384;     // Ut^T P^T fp32 (64)
constexpr uint32_t C_COL_WT = 448;     // W^T fp32 (lane = key, 64 tokens)
constexpr uint32_t C_TMEM_COLS = 512;

// barrier slots (each array sized by its buffer count)
enum : int {
    P_FULL = 0,                    // [NPREP] prep: K/Q stage loaded
    P_MS = P_FULL + NPREP,         // [NPREP] prep: S_kk ready
    P_FREE = P_MS + NPREP,         // [NPREP] prep: chain slot free (remote arrivals)
    P_DRAIN = P_FREE + NPREP,
    C_KF = P_DRAIN + 1,            // [NKB] chain: K tile loaded
    C_VF = C_KF + NKB,             // [NVB] V tile loaded
    C_QF = C_VF + NVB,             // [NQB] Q tile loaded
    C_KFREE = C_QF + NQB,          // [NKB] K buffer read (W^T and dS done)
    C_VFREE = C_KFREE + NKB,       // [NVB] V buffer read (U0 done)
    C_QFREE = C_VFREE + NVB,       // [NQB] Q buffer read (S Q^T done)
    C_TPF = C_QFREE + NQB,         // [NPREP] slot filled (bulk-copy transactions from the prep CTA)
    C_SLOTDONE = C_TPF + NPREP,    // [NPREP] slot's tiles consumed (U^T P'^T commit)
    C_OUTRDY = C_SLOTDONE + NPREP, // chunk output staged (state-warp arrivals)
    C_STGFREE,                     // output stage read out by the TMA stores
    C_MA,                          // Ut^T ready
    C_MD,                          // dS ready
    C_MO,                          // S Q^T and Ut^T P^T ready
    C_MW,                          // W^T ready
    C_S2,                          // bf16 Ut^T, (w Ut)^T written (state-warp arrivals)
    C_S4,                          // bf16 S and bf16 W^T written (state-warp arrivals)
    C_OFREE,                       // output accumulators read (state-warp arrivals)
    C_DRAIN,
    NBAR_USED
};
static_assert(NBAR_USED <= NBARS, "barrier slots");

struct Params {
    CUtensorMap tm_q, tm_k, tm_v, tm_o;  // tm_o: fp32 output, 32-column x 64-row boxes
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
    int R;  // prep CTAs per cluster (ranks 0..R-1); the chain is rank R
};

// Bounded wait that honours the CTA's abort flag.  `cluster` selects acquire at
// cluster scope (arrivals from the other CTA).  Small enough to inline at every
// wait of the hot loops: the abort flag is checked every 256 polls, and a wait
// that gives up only raises the flag (the kernel records GDN_ERR_TIMEOUT once,
// on its way out).
__device__ __forceinline__ bool wait(uint64_t* bar, uint32_t phase, volatile uint32_t* abort,
                                     bool cluster = false) {
    const uint32_t a = smem_u32(bar);
    uint32_t i = 0;
#pragma unroll 1
    while (!(cluster ? tc::mbar_try_wait_cluster(a, phase) : mbar_try_wait(a, phase))) {
        if ((++i & 255u) == 0u && (*abort || i >= kPolls)) {
            *abort = 1u;
            return false;
        }
    }
    return true;
}
// The same for a whole converged warp: it leaves the loop only by warp votes, so
// the code after it is warp-uniform (the tcgen05 issue sequences that follow
// need uniform operands and stay short when the compiler can see that).
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t phase, volatile uint32_t* abort,
                                          bool cluster = false) {
    const uint32_t a = smem_u32(bar);
    uint32_t i = 0;
#pragma unroll 1
    while (!__all_sync(0xffffffffu,
                       cluster ? tc::mbar_try_wait_cluster(a, phase) : mbar_try_wait(a, phase))) {
        if ((++i & 255u) == 0u && __any_sync(0xffffffffu, *abort != 0u || i >= kPolls)) {
            *abort = 1u;
            return false;
        }
    }
    return true;
}

// Bounded wait that ignores the abort flag (used to drain on the way out).
__device__ __noinline__ void drain_wait(uint64_t* bar, uint32_t phase) {
    const uint32_t a = smem_u32(bar);
    for (uint32_t i = 0; i < kPolls && !mbar_try_wait(a, phase); ++i) {
    }
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) { return tc::pack_bf16(lo, hi); }

// 16 consecutive floats from shared memory (16-byte aligned) in four vector loads.
__device__ __forceinline__ void lds16(uint32_t addr, float (&v)[16]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint4 x = tc::ld_shared_v4(addr + 16 * i);
        v[4 * i + 0] = __uint_as_float(x.x);
        v[4 * i + 1] = __uint_as_float(x.y);
        v[4 * i + 2] = __uint_as_float(x.z);
        v[4 * i + 3] = __uint_as_float(x.w);
    }
}
// Shared-memory store at a register address plus a compile-time offset.
template <int OFF>
__device__ __forceinline__ void sts_f32_imm(uint32_t addr, float v) {
    asm volatile("st.shared.f32 [%0+%1], %2;" ::"r"(addr), "n"(OFF), "f"(v) : "memory");
}
// Rows T0 + J (J = 0..N-1) of a 128-byte-swizzled fp32 staging tile: the address is
// ak[row & 7] (holding the swizzled column of this lane) plus a constant row offset.
template <int T0, int N, int... J>
__device__ __forceinline__ void stage_out(const uint32_t (&ak)[8], const float (&gm)[N],
                                          const float (&o1)[N], const float (&o2)[N],
                                          std::integer_sequence<int, J...>) {
    (sts_f32_imm<((T0 + J) >> 3) * 1024 + ((T0 + J) & 7) * 128>(ak[(T0 + J) & 7],
                                                                 fmaf(gm[J], o1[J], o2[J])),
     ...);
}

// ------------------------------------------------ triangular inverse (prep)

// Warp-level tf32 tensor-core MMA (m16n8k8, fp32 accumulate).  tcgen05's
// smallest tile is 64 rows, so the 16x16 blocks of the inverse use this form.
// Fragment layout (PTX ISA, mma.m16n8k8 .tf32): g = lane/4, t = lane%4;
// A: (g,t) (g+8,t) (g,t+4) (g+8,t+4); B: (t,g) (t+4,g); C: (g,2t) (g,2t+1)
// (g+8,2t) (g+8,2t+1).
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
// A 16x16 fp32 operand block in shared memory: element (r, c) at p[r * rs + c * cs].
struct Blk {
    float* p;
    int rs, cs;
};
// acc (+)= X Y for 16x16 blocks (one code path for every operand layout).
__device__ __forceinline__ void mm16(float (&acc)[2][4], Blk x, Blk y, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
        const int k0 = 8 * kk;
        uint32_t a[4] = {to_tf32(x.p[g * x.rs + (k0 + t) * x.cs]),
                         to_tf32(x.p[(g + 8) * x.rs + (k0 + t) * x.cs]),
                         to_tf32(x.p[g * x.rs + (k0 + t + 4) * x.cs]),
                         to_tf32(x.p[(g + 8) * x.rs + (k0 + t + 4) * x.cs])};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
            mma_tf32(acc[nt], a, to_tf32(y.p[(k0 + t) * y.rs + (8 * nt + g) * y.cs]),
                     to_tf32(y.p[(k0 + t + 4) * y.rs + (8 * nt + g) * y.cs]));
    }
}
// Stores sign * acc into the block z.
__device__ __forceinline__ void mm16_out(const float (&acc)[2][4], Blk z, float sign, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        const int c = 8 * nt + 2 * t;
        z.p[g * z.rs + c * z.cs] = sign * acc[nt][0];
        z.p[g * z.rs + (c + 1) * z.cs] = sign * acc[nt][1];
        z.p[(g + 8) * z.rs + c * z.cs] = sign * acc[nt][2];
        z.p[(g + 8) * z.rs + (c + 1) * z.cs] = sign * acc[nt][3];
    }
}

// T = (I + A)^-1 for the strictly lower 64x64 A held in AT (fp32, pitch AP).
// T is unit lower triangular; its strictly lower part is written transposed
// into AT's strictly upper triangle (T[r][s] at AT[s][r], s < r), so A and T
// share one buffer.  By 16x16 blocks: the diagonal blocks D_i = (I+A_ii)^-1
// by substitution, then the two 32x32 halves (T_10 = -D_1 A_10 D_0, T_32
// likewise), then the lower-left 32x32 quarter T_BA = -T_BB (A_BA T_AA).
// Called by the 128 threads of one prep warpgroup (warp pw); Xs is scratch for
// ten 16x16 blocks (the dense D_i, then six products); named barrier `bid`.
__device__ __forceinline__ void invert_unit_lower(float* AT, float* Xs, int pw, int lane, int bid) {
    auto Ab = [AT](int i, int j) { return Blk{AT + 16 * i * AP + 16 * j, AP, 1}; };
    auto Tb = [AT](int i, int j) { return Blk{AT + 16 * j * AP + 16 * i, 1, AP}; };  // i > j
    auto Sb = [Xs](int b) { return Blk{Xs + b * 16 * XP, XP, 1}; };  // D_i = block i, X_k = 4 + k
    // 1. D_pw by substitution, lanes 0..15 one column each: x_r = -sum_{s<r} A_rs x_s
    if (lane < 16) {
        const int o = 16 * pw, j = lane;
        float t[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
            for (int s = 0; s < r; s += 2) {
                acc0 = fmaf(AT[(o + r) * AP + o + s], t[s], acc0);
                if (s + 1 < r) acc1 = fmaf(AT[(o + r) * AP + o + s + 1], t[s + 1], acc1);
            }
            t[r] = (r < j) ? 0.f : ((r == j) ? 1.f : -(acc0 + acc1));
        }
        float* dcol = Xs + pw * 16 * XP + j;
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            dcol[r * XP] = t[r];
            if (r > j) AT[(o + j) * AP + o + r] = t[r];
        }
    }
    tc::named_bar(bid, 128);
    // 2. X_pw = A * D: (A_10 D_0), (A_32 D_2), (A_21 D_1), (A_31 D_1);
    //    then T_10 = -D_1 X_0 (warp 0), T_32 = -D_3 X_1 (warp 1)
    {
        const int ai = pw == 0 ? 1 : (pw == 1 ? 3 : pw), aj = pw == 0 ? 0 : (pw == 1 ? 2 : 1);
        const int dj = pw == 0 ? 0 : (pw == 1 ? 2 : 1);
        float c[2][4] = {};
        mm16(c, Ab(ai, aj), Sb(dj), lane);
        mm16_out(c, Sb(4 + pw), 1.f, lane);
        if (pw < 2) {
            __syncwarp();
            const int i = pw == 0 ? 1 : 3;
            float c2[2][4] = {};
            mm16(c2, Sb(i), Sb(4 + pw), lane);
            mm16_out(c2, Tb(i, i - 1), -1.f, lane);
        }
    }
    tc::named_bar(bid, 128);
    // 3. warps 0, 1: X_{4+pw} = A_i0 D_0 + A_i1 T_10 (i = 2 + pw)
    //    warp 2: T_21 = -D_2 X_2;  warp 3: T_31 = -(T_32 X_2 + D_3 X_3)
    {
        float c[2][4] = {};
        if (pw < 2) {
            mm16(c, Ab(2 + pw, 0), Sb(0), lane);
            mm16(c, Ab(2 + pw, 1), Tb(1, 0), lane);
            mm16_out(c, Sb(8 + pw), 1.f, lane);
        } else {
            mm16(c, pw == 2 ? Sb(2) : Tb(3, 2), Sb(6), lane);
            if (pw == 3) mm16(c, Sb(3), Sb(7), lane);
            mm16_out(c, Tb(pw, 1), -1.f, lane);
        }
    }
    tc::named_bar(bid, 128);
    // 4. warp 0: T_20 = -D_2 X_8;  warp 1: T_30 = -(T_32 X_8 + D_3 X_9)
    if (pw < 2) {
        float c[2][4] = {};
        mm16(c, pw == 0 ? Sb(2) : Tb(3, 2), Sb(8), lane);
        if (pw == 1) mm16(c, Sb(3), Sb(9), lane);
        mm16_out(c, Tb(2 + pw, 0), -1.f, lane);
    }
    tc::named_bar(bid, 128);
}

// Non-blocking test of an mbarrier phase (local arrivals / cluster acquire).
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t phase) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n"
        " mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(phase)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_test_cluster(uint64_t* bar, uint32_t phase) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n"
        " mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(phase)
        : "memory");
    return ok != 0;
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
    const uint32_t R = (uint32_t)p.R;  // prep CTAs of the cluster; the chain is rank R
    const bool is_chain = rank == R;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int H = p.H;
    // the (sequence, head) of this cluster
    const int sh = (int)(blockIdx.x / (R + 1u));
    const int head = sh % H;
    const int seq = p.order ? p.order[sh / H] : sh / H;
    int64_t cs, ce;
    if (p.cu) {
        cs = p.cu[seq];
        ce = p.cu[seq + 1];
    } else {
        cs = (int64_t)seq * p.T;
        ce = cs + p.T;
    }
    // per-CTA constants, made warp-uniform (lane-0 broadcast, warp reduction) so the
    // compiler can keep the loop bounds and tcgen05 operands derived from them uniform
    cs = __shfl_sync(0xffffffffu, cs, 0);
    ce = __shfl_sync(0xffffffffu, ce, 0);
    const int nch = (int)__reduce_max_sync(0xffffffffu, (uint32_t)((ce - cs + C - 1) / C));

    if (threadIdx.x == 0) {
        for (int i = 0; i < NBARS; ++i) {
            uint32_t cnt = 1u;
            if (i == C_S2 || i == C_S4) cnt = (uint32_t)NSW;  // the state warps
            if (i == C_OFREE || i == C_OUTRDY) cnt = (uint32_t)NSW;
            mbar_init(&bars[i], cnt);
        }
        misc[1] = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        // chain: arm the slot barriers for the first images before the prep CTA
        // can start a copy (it waits at the cluster barrier below)
        if (is_chain)
            for (int i = 0; i < NPREP; ++i) tc::mbar_arrive_expect_tx(&bars[C_TPF + i], kImgTx);
    }
    const uint32_t ncols = is_chain ? C_TMEM_COLS : P_TMEM_COLS;
    if (warp == 0) tc::tmem_alloc(&misc[0], ncols);
    tc::tc_before_sync();
    __syncthreads();
    tc::cluster_sync();  // every CTA's barriers initialised before any remote arrive
    tc::tc_after_sync();
    // read through a warp reduction so the compiler treats it as warp-uniform (the
    // tcgen05 operands it feeds must be uniform)
    const uint32_t tmem = __reduce_max_sync(0xffffffffu, misc[0]);

    if (!is_chain) {
        // ================================================================ prep
        // prep CTA `rank` takes the chunks c with (c / NPREP) % R == rank; its
        // warpgroup pg those with c % NPREP == pg, i.e. c = pg + NPREP (rank + R n)
        const int pg = warp >> 2;
        if (pg < NPREP) {
            const int pt = threadIdx.x - 128 * pg, pw = warp & 3;
            const int bid = 1 + pg;
            uint8_t* kq_p = base + P_OFF_KQ + pg * SZ_KQ;
            const uint32_t kq = sbase + P_OFF_KQ + pg * SZ_KQ;
            const uint32_t im = sbase + P_OFF_IMG + pg * SZ_TILES;
            float* Xs = reinterpret_cast<float*>(base + P_OFF_IMG + pg * SZ_TILES);
            float* AT = reinterpret_cast<float*>(base + P_OFF_AT + pg * SZ_AT);
            PrepScal* ps = reinterpret_cast<PrepScal*>(base + P_OFF_PS) + pg;
            ChainScal* cst = reinterpret_cast<ChainScal*>(base + P_OFF_SC + pg * kScalBytes);
            const uint32_t cst_u32 = sbase + P_OFF_SC + pg * kScalBytes;
            uint64_t* full = &bars[P_FULL + pg];
            uint64_t* mS = &bars[P_MS + pg];
            uint64_t* sfree = &bars[P_FREE + pg];
            const uint32_t tcol = tmem + 64u * pg;
            // this warpgroup's slot in the chain CTA
            const uint32_t r_sl = tc::mapa(sbase + C_OFF_SL + pg * SZ_TILES, R);
            const uint32_t r_sc0 = tc::mapa(sbase + C_OFF_SC, R);  // gate-factor ring
            const uint32_t r_tpf = tc::mapa(smem_u32(&bars[C_TPF + pg]), R);
            const int c0 = pg + NPREP * (int)rank, cstep = NPREP * (int)R;
            const uint32_t idS = tc::idesc_bf16(128, 64, 0, 0);
            auto issue_load = [&](int c) {
                const int y = (int)(cs + (int64_t)C * c);
                tc::mbar_arrive_expect_tx(full, SZ_KQ);
                tc::tma_load_2d(kq_p + 0, &p.tm_k, head * KD + 0, y, full);
                tc::tma_load_2d(kq_p + 8192, &p.tm_q, head * KD + 0, y, full);
                tc::tma_load_2d(kq_p + 16384, &p.tm_k, head * KD + 64, y, full);
                tc::tma_load_2d(kq_p + 24576, &p.tm_q, head * KD + 64, y, full);
            };
            int loads = 0;
            if (pt == 0 && c0 < nch) {
                tc::prefetch_tmap(&p.tm_q);
                tc::prefetch_tmap(&p.tm_k);
                issue_load(c0);
                loads = 1;
            }
            int n = 0;
            // g and beta of a chunk's 64 tokens (thread pt < 64 holds token pt), fetched
            // one job ahead so their latency overlaps the previous chunk's work
            auto load_gb = [&](int c, float& gv, float& bv) {
                const int64_t t0 = cs + (int64_t)C * c;
                gv = 0.f;
                bv = 0.f;
                if (c < nch && pt < 64 && t0 + pt < ce) {
                    gv = p.g[(t0 + pt) * H + head];
                    bv = p.beta[(t0 + pt) * H + head];
                }
            };
            float gv_next, bv_next;
            load_gb(c0, gv_next, bv_next);
            for (int c = c0; c < nch; c += cstep, ++n) {
                const float gv = gv_next, bv = bv_next;
                load_gb(c + cstep, gv_next, bv_next);
                wait(full, n & 1, abort_flag);
                __syncwarp();
                if (pw == 0) {
                    // S_kk = [K; Q] K^T, issued by one elected lane of warp 0
                    tc::tc_after_sync();
                    if (tc::elect_one()) {
                        const uint32_t lk = tc::desc_lo(kq, 16);
                        tc::mma_ss<0>(tcol, tc::desc(lk), tc::desc(lk), idS);
#pragma unroll
                        for (int kk = 1; kk < 8; ++kk) {
                            const uint32_t off = (kk >> 2) * 1024 + (kk & 3) * 2;  // 16-byte units
                            tc::mma_ss<1>(tcol, tc::desc(lk + off), tc::desc(lk + off), idS);
                        }
                        tc::mma_commit(mS);
                    }
                    __syncwarp();
                }
                // in-chunk inclusive cumsum of g (log2 units) on warps 0-1
                float x = gv * kLog2e;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, x, off);
                    if (lane >= off) x += y;
                }
                if (pt == 31) ps->tmp[0] = x;
                if (pt == 0) tc::bulk_wait_read0();  // the previous image has left im / cst
                tc::named_bar(bid, 128);
                if (pw == 1) x += ps->tmp[0];
                if (pt < 64) ps->G2[pt] = x;
                tc::named_bar(bid, 128);
                const float G2L = ps->G2[63];
                if (pt < 64) {
                    const float gm = exp2f(x);
                    ps->gam[pt] = gm;
                    ps->ginv[pt] = exp2f(-x);
                    ps->beta[pt] = bv;
                    cst->w[pt] = exp2f(G2L - x);
                    cst->gam[pt] = p.scale * gm;
                    if (pt == 0) cst->eGL = exp2f(G2L);
                }
                wait(mS, n & 1, abort_flag);
                tc::tc_after_sync();
                // the stage has been read by S_kk: this warpgroup's next chunk may load into it
                if (pt == 0 && c + cstep < nch && !*abort_flag) {
                    issue_load(c + cstep);
                    ++loads;
                }
                tc::named_bar(bid, 128);  // gam / beta visible
                {
                    // row of S_kk: rows 0-63 = K K^T (-> A row), rows 64-127 = Q K^T (-> P row).
                    // The decay 2^(G2_r - G2_s) is factored as 2^G2_r * 2^-G2_s when the
                    // chunk's total decay stays above 2^-126 (no factor overflows or
                    // underflows), else taken per element (masked entries may overflow to
                    // inf there before the select discards them).
                    const uint32_t ta = tcol + ((uint32_t)(32 * pw) << 16);
                    const int r = pt & 63;
                    const float g2r = ps->G2[r];
                    const float coef = pt < 64 ? bv : p.scale;  // P rows carry the output scale
                    const float cg = coef * ps->gam[r];
                    const int lim = pt < 64 ? r : r + 1;  // columns s < lim are kept
                    const bool factored = G2L > -126.f;
#pragma unroll 1
                    for (int h = 0; h < 2; ++h) {
                        float sv[32];
                        tc::tmem_ld32(ta + 32 * h, sv);
                        tc::tmem_wait_ld();
                        if (factored) {
                            float gi[16];
#pragma unroll
                            for (int hh = 0; hh < 2; ++hh) {
                                lds16(smem_u32(ps->ginv + 32 * h + 16 * hh), gi);
#pragma unroll
                                for (int j = 0; j < 16; ++j) {
                                    const int s = 32 * h + 16 * hh + j;
                                    sv[16 * hh + j] = s < lim ? (cg * gi[j]) * sv[16 * hh + j] : 0.f;
                                }
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < 32; ++j) {
                                const int s = 32 * h + j;
                                const float f = coef * exp2f(g2r - ps->G2[s]);
                                sv[j] = s < lim ? f * sv[j] : 0.f;
                            }
                        }
                        if (pt < 64) {
                            float* arow = AT + r * AP + 32 * h;
#pragma unroll
                            for (int j = 0; j < 32; j += 4)
                                *reinterpret_cast<float4*>(arow + j) =
                                    make_float4(sv[j], sv[j + 1], sv[j + 2], sv[j + 3]);
                        } else {
                            tc::store_half_row_bf16(im + SL_P, r, h, sv);
                        }
                    }
                }
                tc::tc_before_sync();     // S_kk read before the next S_kk overwrites it
                tc::named_bar(bid, 128);  // A rows complete
                invert_unit_lower(AT, Xs, pw, lane, bid);
                {
                    // T' = T diag(beta gam), Tb = T diag(beta): row r, 32 columns per thread
                    const int r = pt >> 1, hf = pt & 1;
#pragma unroll 1
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const int ch = 4 * hf + q4;
                        float tb[8], tp[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int s = 8 * ch + e;
                            const float tv = s < r ? AT[s * AP + r] : (s == r ? 1.f : 0.f);
                            tb[e] = tv * ps->beta[s];
                            tp[e] = tb[e] * ps->gam[s];
                        }
                        const uint32_t off = tc::sw128_off(r, ch);
                        tc::st_shared_v4(im + SL_TB + off, pack2(tb[0], tb[1]), pack2(tb[2], tb[3]),
                                         pack2(tb[4], tb[5]), pack2(tb[6], tb[7]));
                        tc::st_shared_v4(im + SL_TP + off, pack2(tp[0], tp[1]), pack2(tp[2], tp[3]),
                                         pack2(tp[4], tp[5]), pack2(tp[6], tp[7]));
                    }
                }
                tc::fence_async_smem();
                tc::named_bar(bid, 128);
                if (pt == 0) {
                    // ship the image once the chain has released the slot (after its last
                    // product of chunk c - NPREP; handed back to this warpgroup once per
                    // job of it from chunk NPREP on)
                    if (c >= NPREP) wait(sfree, (uint32_t)(n - (rank == 0 ? 1 : 0)) & 1u, abort_flag, true);
                    tc::bulk_s2cluster(r_sl, im, SZ_TILES, r_tpf);
                    tc::bulk_s2cluster(r_sc0 + (uint32_t)(c % NFAC) * kScalBytes, cst_u32, kScalBytes,
                                       r_tpf);
                    tc::bulk_commit();
                }
            }
            if (pt == 0) {
                // never leave with a copy or an MMA in flight
                tc::bulk_wait0();
                if (loads > n) drain_wait(full, n & 1);
                if (*abort_flag) {
                    tc::mma_commit(&bars[P_DRAIN]);
                    drain_wait(&bars[P_DRAIN], 0);
                }
            }
        }
    } else {
        // =============================================================== chain
        uint64_t* mA = &bars[C_MA];
        uint64_t* mD = &bars[C_MD];
        uint64_t* mO = &bars[C_MO];
        uint64_t* mW = &bars[C_MW];
        uint64_t* s2 = &bars[C_S2];
        uint64_t* s4 = &bars[C_S4];
        uint64_t* ofree = &bars[C_OFREE];
        auto kbuf = [&](int c) { return sbase + C_OFF_K + (uint32_t)(c % NKB) * SZ_T; };
        auto vbuf = [&](int c) { return sbase + C_OFF_V + (uint32_t)(c % NVB) * SZ_T; };
        auto qbuf = [&](int c) { return sbase + C_OFF_Q + (uint32_t)(c % NQB) * SZ_T; };
        auto slot = [&](int c) { return sbase + C_OFF_SL + (uint32_t)(c % NPREP) * SZ_TILES; };
        const uint32_t wt = sbase + C_OFF_WT;
        const uint32_t ostg = sbase + C_OFF_OUT;
        if (warp == W_LOAD) {
            if (lane == 0) {
                // loader: K, V and Q tiles as their buffers fall free, and the slots
                // back to the prep CTA once consumed; polls every resource in turn
                const uint32_t l_free0 = smem_u32(&bars[P_FREE]);
                tc::prefetch_tmap(&p.tm_k);
                tc::prefetch_tmap(&p.tm_v);
                tc::prefetch_tmap(&p.tm_q);
                auto load = [&](const CUtensorMap* m, uint32_t dst, uint64_t* bar, int c) {
                    const int y = (int)(cs + (int64_t)C * c);
                    tc::mbar_arrive_expect_tx(bar, SZ_T);
                    tc::tma_load_2d(base + (dst - sbase), m, head * 128, y, bar);
                    tc::tma_load_2d(base + (dst - sbase) + 8192, m, head * 128 + 64, y, bar);
                };
                int nk = 0, nv = 0, nq = 0, ns = 0;
                uint32_t idle = 0;
                while (!*abort_flag) {
                    bool prog = false;
                    if (ns + NPREP < nch && mbar_test(&bars[C_SLOTDONE + ns % NPREP], (ns / NPREP) & 1)) {
                        // re-arm the slot's barrier for its next image, then hand it back
                        const int j = ns % NPREP;
                        tc::mbar_arrive_expect_tx(&bars[C_TPF + j], kImgTx);
                        // to the prep CTA that builds chunk ns + NPREP
                        const uint32_t tr = (uint32_t)((ns + NPREP) / NPREP) % R;
                        tc::mbar_arrive_cluster(tc::mapa(l_free0 + 8u * (uint32_t)j, tr));
                        ++ns;
                        prog = true;
                    }
                    if (nk < nch && (nk < NKB || mbar_test(&bars[C_KFREE + nk % NKB], ((nk / NKB) - 1) & 1))) {
                        load(&p.tm_k, kbuf(nk), &bars[C_KF + nk % NKB], nk);
                        ++nk;
                        prog = true;
                    }
                    if (nv < nch && (nv < NVB || mbar_test(&bars[C_VFREE + nv % NVB], ((nv / NVB) - 1) & 1))) {
                        load(&p.tm_v, vbuf(nv), &bars[C_VF + nv % NVB], nv);
                        ++nv;
                        prog = true;
                    }
                    if (nq < nch && (nq < NQB || mbar_test(&bars[C_QFREE + nq % NQB], ((nq / NQB) - 1) & 1))) {
                        load(&p.tm_q, qbuf(nq), &bars[C_QF + nq % NQB], nq);
                        ++nq;
                        prog = true;
                    }
                    if (nk == nch && nv == nch && nq == nch && ns + NPREP >= nch) break;
                    if (prog) {
                        idle = 0;
                    } else if (++idle == kIdleLimit) {
                        *abort_flag = 1u;
                        record_status(GDN_ERR_TIMEOUT);
                    }
                }
                // never leave with a copy in flight
                for (int c = nk - NKB; c < nk; ++c)
                    if (c >= 0) drain_wait(&bars[C_KF + c % NKB], (c / NKB) & 1);
                for (int c = nv - NVB; c < nv; ++c)
                    if (c >= 0) drain_wait(&bars[C_VF + c % NVB], (c / NVB) & 1);
                for (int c = nq - NQB; c < nq; ++c)
                    if (c >= 0) drain_wait(&bars[C_QF + c % NQB], (c / NQB) & 1);
            }
        } else if (warp == W_MMA) {
            // MMA warp: all 32 lanes run it, converged, and one elected lane issues
            // every product and commit (a commit tracks the products of its own
            // thread).  Descriptors are precomputed words plus constant offsets, so
            // each issue is a few instructions.  The dependent products (Ut^T, dS) go out as soon as
            // their inputs are written; W^T of the next chunk goes ahead of dS when
            // its tiles are in.
            const uint32_t idWT = tc::idesc_bf16(128, 64, 1, 0);
            const uint32_t idU0 = tc::idesc_bf16(128, 64, 1, 0);
            const uint32_t idUt = tc::idesc_bf16(128, 64, 0, 1) | tc::kNegateA;
            const uint32_t idSQ = tc::idesc_bf16(128, 64, 0, 0);
            const uint32_t idDS = tc::idesc_bf16(128, 128, 0, 1);
            const uint32_t idUP = tc::idesc_bf16(128, 64, 0, 0);
            // low descriptor words (start address, leading offset) of each buffer
            auto lo = [](uint32_t addr, uint32_t lbo) { return tc::desc_lo(addr, lbo); };
            auto issue_wt_mmas = [&](int c) {  // W^T(c) = K^T T'^T  (A = K tile MN-major, B = T' K-major)
                tc::tc_after_sync();
                if (tc::elect_one()) {
                    const uint32_t la = lo(kbuf(c), 8192), lb = lo(slot(c) + SL_TP, 16);
                    tc::mma_ss<0>(tmem + C_COL_WT, tc::desc(la), tc::desc(lb), idWT);
#pragma unroll
                    for (int kk = 1; kk < 4; ++kk)
                        tc::mma_ss<1>(tmem + C_COL_WT, tc::desc(la + 128 * kk), tc::desc(lb + 2 * kk), idWT);
                    tc::mma_commit(mW);
                }
            };
            auto issue_wt = [&](int c) {
                wait_warp(&bars[C_KF + c % NKB], (c / NKB) & 1, abort_flag);
                wait_warp(&bars[C_TPF + c % NPREP], (c / NPREP) & 1, abort_flag, true);
                __syncwarp();
                issue_wt_mmas(c);
            };
            auto issue_u0 = [&](int c) {  // U0(c) = V^T Tb^T
                wait_warp(&bars[C_VF + c % NVB], (c / NVB) & 1, abort_flag);
                wait_warp(&bars[C_TPF + c % NPREP], (c / NPREP) & 1, abort_flag, true);
                __syncwarp();
                tc::tc_after_sync();
                if (tc::elect_one()) {
                    const uint32_t la = lo(vbuf(c), 8192), lb = lo(slot(c) + SL_TB, 16);
                    tc::mma_ss<0>(tmem + C_COL_U, tc::desc(la), tc::desc(lb), idU0);
#pragma unroll
                    for (int kk = 1; kk < 4; ++kk)
                        tc::mma_ss<1>(tmem + C_COL_U, tc::desc(la + 128 * kk), tc::desc(lb + 2 * kk), idU0);
                    tc::mma_commit(&bars[C_VFREE + c % NVB]);
                }
            };
            if (nch > 0) {
                issue_wt(0);
                issue_u0(0);
            }
            for (int c = 0; c < nch; ++c) {
                wait_warp(s4, c & 1, abort_flag);  // bf16 S and W^T of this chunk written
                __syncwarp();
                tc::tc_after_sync();
                if (tc::elect_one()) {
                    // Ut^T = V^T Tb^T - S W^T
                    const uint32_t lwt = lo(wt, 8192);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        tc::mma_ts<1>(tmem + C_COL_U, tmem + C_COL_SB + 8 * kk, tc::desc(lwt + 128 * kk), idUt);
                    tc::mma_commit(mA);
                }
                // S Q^T for the output, once the previous output has been read out
                wait_warp(&bars[C_QF + c % NQB], (c / NQB) & 1, abort_flag);
                if (c >= 1) wait_warp(ofree, (c - 1) & 1, abort_flag);
                __syncwarp();
                tc::tc_after_sync();
                if (tc::elect_one()) {
                    const uint32_t lq = lo(qbuf(c), 16);
                    tc::mma_ts<0>(tmem + C_COL_O1, tmem + C_COL_SB, tc::desc(lq), idSQ);
#pragma unroll
                    for (int kk = 1; kk < 8; ++kk)
                        tc::mma_ts<1>(tmem + C_COL_O1, tmem + C_COL_SB + 8 * kk,
                                      tc::desc(lq + (kk >> 2) * 512 + (kk & 3) * 2), idSQ);
                    tc::mma_commit(&bars[C_QFREE + c % NQB]);
                }
                // W^T of the next chunk ahead of dS when its K tile and image are in
                bool early = false;
                if (c + 1 < nch) {
                    // every lane must have observed both completions
                    const bool ok =
                        mbar_test(&bars[C_KF + (c + 1) % NKB], ((c + 1) / NKB) & 1) &&
                        mbar_test_cluster(&bars[C_TPF + (c + 1) % NPREP], ((c + 1) / NPREP) & 1);
                    early = __all_sync(0xffffffffu, ok) && !*abort_flag;
                    if (early) issue_wt_mmas(c + 1);
                }
                wait_warp(s2, c & 1, abort_flag);  // Ut^T and (w Ut)^T written in bf16
                __syncwarp();
                tc::tc_after_sync();
                if (tc::elect_one()) {
                    // dS = (w Ut)^T K
                    const uint32_t lk = lo(kbuf(c), 8192);
                    tc::mma_ts<0>(tmem + C_COL_DS, tmem + C_COL_WB, tc::desc(lk), idDS);
#pragma unroll
                    for (int kk = 1; kk < 4; ++kk)
                        tc::mma_ts<1>(tmem + C_COL_DS, tmem + C_COL_WB + 8 * kk, tc::desc(lk + 128 * kk), idDS);
                    tc::mma_commit(mD);
                    tc::mma_commit(&bars[C_KFREE + c % NKB]);
                    // Ut^T P^T
                    const uint32_t lp = lo(slot(c) + SL_P, 16);
                    tc::mma_ts<0>(tmem + C_COL_O2, tmem + C_COL_UB, tc::desc(lp), idUP);
#pragma unroll
                    for (int kk = 1; kk < 4; ++kk)
                        tc::mma_ts<1>(tmem + C_COL_O2, tmem + C_COL_UB + 8 * kk, tc::desc(lp + 2 * kk), idUP);
                    tc::mma_commit(mO);
                    tc::mma_commit(&bars[C_SLOTDONE + c % NPREP]);  // the slot's tiles are spent
                }
                if (c + 1 < nch) {
                    if (!early) issue_wt(c + 1);
                    issue_u0(c + 1);  // D_U was read before s2
                }
            }
            // never leave with an MMA in flight
            if (tc::elect_one()) {
                tc::mma_commit(&bars[C_DRAIN]);
                drain_wait(&bars[C_DRAIN], 0);
            }
            __syncwarp();
        } else if (warp == W_STORE) {
            if (lane == 0) {
                // output store warp: sends each full chunk's staged fp32 output out with
                // four TMA stores (one per value quarter) and frees the stage once the
                // stores have read it; ragged or bf16 chunks were stored directly
                tc::prefetch_tmap(&p.tm_o);
                for (int c = 0; c < nch; ++c) {
                    wait(&bars[C_OUTRDY], c & 1, abort_flag);
                    const int64_t t0 = cs + (int64_t)C * c;
                    if (!OBF16 && ce - t0 >= C && !*abort_flag) {
#pragma unroll
                        for (int qq = 0; qq < 4; ++qq)
                            tc::tma_store_2d(&p.tm_o, ostg + (uint32_t)qq * 8192u, head * VD + 32 * qq,
                                             (int)t0);
                        tc::bulk_commit();
                        tc::bulk_wait_read0();
                    }
                    tc::mbar_arrive(&bars[C_STGFREE]);
                }
                tc::bulk_wait0();  // the output is in global memory before the CTA leaves
            }
        } else if (warp < NSW) {
            // state warps: warpgroup wg owns key columns 32wg.. of S and tokens
            // 16wg.. of the per-chunk tiles; warp q of it the value rows 32q..
            const int wg = warp >> 2, q = warp & 3;
            const int vr = 32 * q + lane;  // value row of S = tensor-memory lane
            const uint32_t lane_base = (uint32_t)(32 * q) << 16;
            const int k0 = 32 * wg;
            const int64_t hb0 = (int64_t)(seq * H + head) * KD * VD;
            float S[32];  // S[vr][k0 .. k0+31] = h[k][vr]
            if (p.h0) {
                const float* hp = p.h0 + hb0 + (int64_t)k0 * VD + vr;
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) S[jj] = hp[jj * VD];
            } else {
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) S[jj] = 0.f;
            }
            // W^T (lane = key 32q + lane) tokens 16wg.. -> bf16 row of the MN-major B tile
            // (Ut^T of the previous chunk has read the buffer)
            auto conv_wt = [&]() {
                float x[16];
                tc::tmem_ld16(tmem + lane_base + C_COL_WT + 16u * wg, x);
                tc::tmem_wait_ld();
                tc::st_shared_v4(wt + tc::sw128_off(vr, 2 * wg), pack2(x[0], x[1]), pack2(x[2], x[3]),
                                 pack2(x[4], x[5]), pack2(x[6], x[7]));
                tc::st_shared_v4(wt + tc::sw128_off(vr, 2 * wg + 1), pack2(x[8], x[9]),
                                 pack2(x[10], x[11]), pack2(x[12], x[13]), pack2(x[14], x[15]));
                tc::fence_async_smem();
            };
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
            if (nch > 0) {
                wait(mW, 0, abort_flag);
                tc::tc_after_sync();
                conv_wt();
                store_sb();
            }
            for (int c = 0; c < nch; ++c) {
                const int j = c % NPREP;
                const ChainScal* sc = reinterpret_cast<const ChainScal*>(base + C_OFF_SC) + (c % NFAC);
                wait(&bars[C_TPF + j], (c / NPREP) & 1, abort_flag, true);
                wait(mA, c & 1, abort_flag);
                tc::tc_after_sync();
                {
                    // Ut^T columns 16wg..16wg+15 -> bf16 Ut^T and (w Ut)^T in tensor memory
                    float u[16];
                    tc::tmem_ld16(tmem + lane_base + C_COL_U + 16u * wg, u);
                    tc::tmem_wait_ld();
                    float wv[16];
                    lds16(smem_u32(sc->w + 16 * wg), wv);
                    uint32_t ub[8], wb[8];
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj) {
                        ub[jj] = pack2(u[2 * jj], u[2 * jj + 1]);
                        wb[jj] = pack2(wv[2 * jj] * u[2 * jj], wv[2 * jj + 1] * u[2 * jj + 1]);
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
                    // S <- 2^G2_L S + dS
                    const float e = sc->eGL;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        float d[16];
                        tc::tmem_ld16(tmem + lane_base + C_COL_DS + 32u * wg + 16u * h, d);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj) S[16 * h + jj] = fmaf(e, S[16 * h + jj], d[jj]);
                    }
                }
                if (c + 1 < nch) {
                    // next chunk's W^T (Ut^T of this chunk has read the tile), then the bf16
                    // copy of S (S Q^T and Ut^T of this chunk completed before dS)
                    wait(mW, (c + 1) & 1, abort_flag);
                    tc::tc_after_sync();
                    conv_wt();
                    store_sb();
                }
                {
                    // o_t = scale gam_t (S Q^T)[vr][t] + (Ut^T P'^T)[vr][t] (P' = scale P) for
                    // this warpgroup's 16 tokens, staged in the spent slot for the store warp
                    // (full fp32 chunks) or stored directly (ragged chunks, bf16 output)
                    const int64_t t0 = cs + (int64_t)C * c;
                    const int len = (int)((ce - t0) < C ? (ce - t0) : C);
                    wait(mO, c & 1, abort_flag);
                    tc::tc_after_sync();
                    float o1[16], o2[16];
                    tc::tmem_ld16(tmem + lane_base + C_COL_O1 + 16u * wg, o1);
                    tc::tmem_ld16(tmem + lane_base + C_COL_O2 + 16u * wg, o2);
                    tc::tmem_wait_ld();
                    tc::tc_before_sync();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(ofree);
                    float gm[16];
                    lds16(smem_u32(sc->gam + 16 * wg), gm);
                    // one output in flight: the previous chunk's has left the stage
                    if (c >= 1) wait(&bars[C_STGFREE], (c - 1) & 1, abort_flag);
                    if (!OBF16 && len == C) {
                        // 128-byte swizzle: 16-byte chunk lane/4 of row t sits at (lane/4) ^ (t & 7)
                        const uint32_t a0 = ostg + (uint32_t)q * 8192u + 4u * (uint32_t)(lane & 3);
                        const uint32_t ch = (uint32_t)(lane >> 2);
                        uint32_t ak[8];
#pragma unroll
                        for (int k = 0; k < 8; ++k) ak[k] = a0 + ((ch ^ (uint32_t)k) << 4) + (uint32_t)(2 * wg) * 1024u;
                        stage_out<0>(ak, gm, o1, o2, std::make_integer_sequence<int, 16>{});
                        tc::fence_async_smem();
                    } else {
                        const int64_t stride = (int64_t)H * VD;
                        const int64_t ob = ((t0 + 16 * wg) * H + head) * VD + vr;
                        const int nv = len - 16 * wg;  // valid tokens of this warpgroup's 16
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj) {
                            const float ov = fmaf(gm[jj], o1[jj], o2[jj]);
                            if (jj < nv) {
                                if constexpr (OBF16)
                                    static_cast<__nv_bfloat16*>(p.o)[ob + jj * stride] =
                                        __float2bfloat16_rn(ov);
                                else
                                    static_cast<float*>(p.o)[ob + jj * stride] = ov;
                            }
                        }
                    }
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(&bars[C_OUTRDY]);  // output staged (or stored)
                }
            }
            if (p.hT) {
                float* hp = p.hT + hb0 + (int64_t)k0 * VD + vr;
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) hp[jj * VD] = S[jj];
            }
        }
    }
    tc::tc_before_sync();
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) record_status(GDN_ERR_TIMEOUT);
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

// [rows, cols] row-major, 128-byte swizzle: bf16 inputs in 64 x 64 boxes, the
// fp32 output in 32-column x 64-row boxes.
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

// Prep CTAs per cluster for `chains` clusters: 1, or 2-3 when the chains leave SMs
// idle and every cluster of that size is resident at once (the chain then waits
// less for its images).  The resident-cluster count is queried once per device,
// output type and cluster size.
template <class KernFn>
inline int pick_prep_ctas(KernFn kern, bool obf16, int64_t chains) {
    static std::mutex mu;
    static int cache[64][2][4];  // [device][obf16][R]: resident clusters + 1 (0 = unknown)
    int dev = 0, n_sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 1;
    if (cudaDeviceGetAttribute(&n_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 1;
    for (int R = 3; R >= 2; --R) {
        if (chains * (R + 1) > n_sms) continue;
        int ncl;
        {
            std::lock_guard<std::mutex> lock(mu);
            ncl = cache[dev][obf16][R] - 1;
        }
        if (ncl < 0) {
            cudaLaunchConfig_t cfg;
            memset(&cfg, 0, sizeof(cfg));
            cfg.blockDim = dim3(tcf::kThreads, 1, 1);
            cfg.dynamicSmemBytes = tcf::SMEM_BYTES;
            cfg.gridDim = dim3((unsigned)(R + 1), 1, 1);
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = (unsigned)(R + 1);
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            ncl = 0;
            if (cudaOccupancyMaxActiveClusters(&ncl, kern, &cfg) != cudaSuccess) {
                (void)cudaGetLastError();
                ncl = 0;
            }
            std::lock_guard<std::mutex> lock(mu);
            cache[dev][obf16][R] = ncl + 1;
        }
        if (ncl >= chains) return R;
    }
    return 1;
}

// Launches the kernel: one cluster per (sequence, head), R prep CTAs and the
// chain CTA.  Returns 0 on success, 1 when the tensor maps could not be built,
// 2 on a launch error.
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
    using KernFn = void (*)(tcf::Params);
    KernFn kern = obf16 ? tcf::chunk_fwd_tc_kernel<true> : tcf::chunk_fwd_tc_kernel<false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)tcf::SMEM_BYTES) != cudaSuccess)
        return 2;
    const int64_t chains = (int64_t)a.n_seq * a.H;
    const int R = pick_prep_ctas(kern, obf16, chains);
    p.R = R;
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.blockDim = dim3(tcf::kThreads, 1, 1);
    cfg.dynamicSmemBytes = tcf::SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    cfg.gridDim = dim3((unsigned)(chains * (R + 1)), 1, 1);
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)(R + 1);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, p) != cudaSuccess) return 2;
    return 0;
}

}  // namespace gdn
