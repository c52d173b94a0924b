// chunk_gdn.cuh — gated delta rule, chunked prefill: two kernels (the main pass
// is templated: KDA runs it on its own prep kernel's outputs, gdn_main_kernel<true>).
//
// gdn_prep_kernel (fully parallel over (batch, head, chunk)): for each 64-token
//   chunk, the state-independent parts, from one M=128 MMA [Q ; K] K^T:
//     P = Q K^T o Gamma o M                            (the Q rows),
//     A = diag(beta) (K K^T o Gamma o strict-lower)    (the K rows),
//     T = (I + A)^-1   (16x16 diagonal blocks by substitution, then two levels of
//                       block merges on mma.sync tf32),
//     U = T diag(beta gamma) K                         (one M=64, N=128 MMA),
//   and writes T diag(beta), P and -U as bf16 operand images (128-byte
//   swizzled, exactly as the main kernel's shared memory wants them) to the
//   workspace: 32 KB per (batch, head, chunk).
//
// gdn_main_kernel (one CTA per (batch, head, 32-column value slab), 9 warps):
//   with W = T diag(beta) (V - diag(gamma) K S0) = T diag(beta) V - U S0,
//     [X2 ; W] = [0 ; T diag(beta)] V + [Q ; -U] S0   (one accumulator; the first
//                                                     product off the recurrence),
//     dS = K^T diag(gamma_C/gamma) W,  S <- gamma_C S + dS   (fp32, one state row
//                                                     per thread),
//     O = diag(gamma) X2 + [P ; K0] W   (rows 0-63).
//   Two MMA round trips per chunk on the recurrence ([Q ; -U] S0, then dS).
// The derivation of the WY / UT form is in chunk_tc.cuh's header.
//
// Pairwise decays Gamma_ti = gamma_t / gamma_i (i <= t) are products of
// gamma_t = exp2(b_t) and 1/gamma_i = exp2(-b_i) when the chunk's cumulative
// log2-decay b_63 is >= -120 (both factors finite in fp32), otherwise
// exp2(b_t - b_i) per element.  No factor overflows either way.
//
// Hand-offs use mbarriers (TMA transactions, tcgen05.commit, thread arrivals)
// and named barriers inside a group; every wait is bounded.
#pragma once

#include <cstddef>

#include "device.cuh"

namespace la {
namespace ck {
namespace gdn {

constexpr int NTHREADS = 288;   // the main pass: producer, output group, state group

constexpr uint32_t TT_BYTES = 8192;                  // T, bf16 [64][64]
// Workspace item per (batch, head, chunk), written by the prep kernel: operand
// images, bf16, 128-byte swizzled exactly as the main kernel's shared memory
// wants them: T diag(beta) [64][64], P [64][64] and -U = -T diag(beta gamma) K as
// two [64][64] blocks (key columns 0-63, 64-127).  KDA's item (chunk_kda.cuh)
// has the same three images (its U is T diag(beta) (K o Gamma)) and appends
// Gamma_C.
constexpr uint32_t ITEM_T = 0;
constexpr uint32_t ITEM_P = 8192;
constexpr uint32_t ITEM_U = 16384;
constexpr uint32_t ITEM_BYTES = 32768;

constexpr uint32_t QK_ACS = 128 * 128;               // one atom column: Q rows 0-63, K rows 64-127

}  // namespace gdn

// KDA workspace item per (batch, head, chunk), written by kda_prep_kernel
// (chunk_kda.cuh) and read by gdn_main_kernel<true>: the gated delta rule's
// item, then Gamma_C.
namespace kda {
constexpr uint32_t ITEM_T = gdn::ITEM_T;      // T diag(beta) image
constexpr uint32_t ITEM_P = gdn::ITEM_P;      // P image
constexpr uint32_t ITEM_U = gdn::ITEM_U;      // -U = -T diag(beta) (K o Gamma), two [64][64] blocks
constexpr uint32_t ITEM_GC = 32768;           // Gamma_C, fp32 [128]
constexpr uint32_t ITEM_BYTES = 32768 + 512;
}  // namespace kda

namespace gdn {
// Prep-kernel shared memory: [Q ; K] as two atom columns of 128 rows (Q rows
// 0-63, K rows 64-127), one M=128 operand.  The next item's Q is loaded once
// this item's [Q ; K] K^T has read it, its K once the -U MMA has.
constexpr int AF_LD = 68;
constexpr int TMP_LD = 36;
constexpr uint32_t P_ACS = QK_ACS;                   // atom column: Q | K
constexpr uint32_t P_K = 8192;                       // K block within an atom column
constexpr uint32_t P_AF = 2 * P_ACS;                 // A, then T, fp32 [64][AF_LD]; then the
                                                     // T diag(beta gamma) operand image (bf16)
constexpr uint32_t P_TMP = P_AF + 64 * AF_LD * 4;    // fp32 scratch [32][TMP_LD]
constexpr uint32_t P_END = P_TMP + 32 * TMP_LD * 4;   // the control block follows
static_assert(P_END % 16 == 0, "the prep kernel's control block must be 16-byte aligned");
static_assert(P_AF % 1024 == 0, "the operand image in AF must be 1 KB aligned");
constexpr int PREP_THREADS = 128;
constexpr uint32_t PREP_TMEM_COLS = 128;
constexpr int PREP_CTAS_PER_SM = 4;

struct PCtl {
    uint64_t qfull, kfull, mma, mma_u, drain;
    uint32_t tmem_base;
    int abort, stop, fast;
    // read as float4 (the block itself starts 16-byte aligned)
    alignas(16) float alpha[64], beta[64];
    float gam[64], ginv[64], b2[64];
};
static_assert(offsetof(PCtl, alpha) % 16 == 0, "PCtl's gate arrays are read as float4");


// ---- mma.sync m16n8k8 tf32 (fp32 accumulate) used for the block merges ----
__device__ __forceinline__ uint32_t tf32(float x) {
    uint32_t u;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(u) : "f"(x));
    return u;
}
// A fragment: rows r0..r0+15, cols k0..k0+7 of a row-major fp32 matrix.
__device__ __forceinline__ void lda(uint32_t a[4], const float *M, int ld, int r0, int k0, int lane) {
    const int g = lane >> 2, t = lane & 3;
    a[0] = tf32(M[(r0 + g) * ld + k0 + t]);
    a[1] = tf32(M[(r0 + g + 8) * ld + k0 + t]);
    a[2] = tf32(M[(r0 + g) * ld + k0 + t + 4]);
    a[3] = tf32(M[(r0 + g + 8) * ld + k0 + t + 4]);
}
// B fragment: rows (k) k0..k0+7, cols (n) n0..n0+7 of a row-major fp32 matrix.
__device__ __forceinline__ void ldb(uint32_t b[2], const float *M, int ld, int k0, int n0, int lane) {
    const int g = lane >> 2, t = lane & 3;
    b[0] = tf32(M[(k0 + t) * ld + n0 + g]);
    b[1] = tf32(M[(k0 + t + 4) * ld + n0 + g]);
}
__device__ __forceinline__ void mma_tf32(float c[4], const uint32_t a[4], const uint32_t b[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// Store a 16 x 16 result held as two 16x8 accumulators (scaled by s).
__device__ __forceinline__ void stc(float *M, int ld, int r0, int c0, const float c[2][4], float s,
                                    int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        const int col = c0 + 8 * nt + 2 * t;
        M[(r0 + g) * ld + col] = s * c[nt][0];
        M[(r0 + g) * ld + col + 1] = s * c[nt][1];
        M[(r0 + g + 8) * ld + col] = s * c[nt][2];
        M[(r0 + g + 8) * ld + col + 1] = s * c[nt][3];
    }
}

// Row r of a [rows][32] bf16 tile with the 64-byte swizzle (16-byte chunk c of
// row r at chunk c ^ ((r >> 1) & 3)).
__device__ __forceinline__ void store_row64(uint8_t *tile, int r, const float *x32) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint4 u;
        u.x = pack_bf16x2(x32[8 * c + 0], x32[8 * c + 1]);
        u.y = pack_bf16x2(x32[8 * c + 2], x32[8 * c + 3]);
        u.z = pack_bf16x2(x32[8 * c + 4], x32[8 * c + 5]);
        u.w = pack_bf16x2(x32[8 * c + 6], x32[8 * c + 7]);
        *reinterpret_cast<uint4 *>(tile + r * 64 + (((c ^ (r >> 1)) & 3) << 4)) = u;
    }
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}


__device__ __forceinline__ void bulk_load(void *smem_dst, const void *gsrc, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(gsrc)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// log2 of the cumulative product of the chunk's 64 alphas (inclusive prefix),
// with gamma = 2^b and 1/gamma = 2^-b.  One warp, two tokens per lane.
// Returns the fast-path flag (b_63 >= -120).
// `al` holds this lane's two alphas (tokens 2*lane and 2*lane+1).
__device__ __forceinline__ int gate_scan(const float *al, const float *beta, float *b2,
                                         float *gam, float *ginv, float *bg, int lane) {
    const float a0 = log2f(al[0]), a1 = log2f(al[1]);
    const float x1 = a0 + a1;
    float inc = x1;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, inc, off);
        if (lane >= off) inc += y;
    }
    const float e0 = inc - x1 + a0, e1 = inc;
    if (b2) {
        b2[2 * lane] = e0;
        b2[2 * lane + 1] = e1;
    }
    const float g0 = exp2f(e0), g1 = exp2f(e1);
    gam[2 * lane] = g0;
    gam[2 * lane + 1] = g1;
    ginv[2 * lane] = exp2f(-e0);
    ginv[2 * lane + 1] = exp2f(-e1);
    if (bg) {
        bg[2 * lane] = beta[2 * lane] * g0;
        bg[2 * lane + 1] = beta[2 * lane + 1] * g1;
    }
    const float last = __shfl_sync(0xffffffffu, e1, 31);
    return last >= -120.f ? 1 : 0;
}

// Row t of the decayed, masked score matrix from 64 raw scores x (in place):
//   x_i <- x_i * rowf * gamma_t / gamma_i  for i <= t (i < t if strict), else 0.
// ncols = 32 when only the first 32 columns can be unmasked (t < 32).  gam, ginv
// and b2 are 16-byte aligned shared arrays, read four at a time.
template <bool STRICT>
__device__ __forceinline__ void decay_mask_row(float *x, int t, int ncols, float rowf, bool fast,
                                               const float *gam, const float *ginv, const float *b2) {
    if (fast) {
        const float rs = rowf * gam[t];
        const float4 *g4 = reinterpret_cast<const float4 *>(ginv);
#pragma unroll
        for (int i4 = 0; i4 < 16; ++i4) {
            if (4 * i4 >= ncols) {
#pragma unroll
                for (int e = 0; e < 4; ++e) x[4 * i4 + e] = 0.f;
                continue;
            }
            const float4 g = g4[i4];
            const float gv[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int i = 4 * i4 + e;
                const bool keep = STRICT ? (i < t) : (i <= t);
                x[i] = keep ? x[i] * (rs * gv[e]) : 0.f;
            }
        }
    } else {
        const float bt = b2[t];
        const float4 *b4 = reinterpret_cast<const float4 *>(b2);
#pragma unroll
        for (int i4 = 0; i4 < 16; ++i4) {
            if (4 * i4 >= ncols) {
#pragma unroll
                for (int e = 0; e < 4; ++e) x[4 * i4 + e] = 0.f;
                continue;
            }
            const float4 g = b4[i4];
            const float gv[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int i = 4 * i4 + e;
                const bool keep = STRICT ? (i < t) : (i <= t);
                x[i] = keep ? x[i] * (rowf * exp2f(bt - gv[e])) : 0.f;
            }
        }
    }
}

// T = (I + A)^-1 for a strictly lower triangular 64x64 fp32 A held in AF
// (row stride AF_LD), in place; 128 threads (lt = 0..127) with named barriers
// `bar` (128 threads) and `bar64` (the first 64 threads).  TMP: fp32 scratch.
__device__ __forceinline__ void invert_unit_lower64(float *AF, float *TMP, int lt, int lane, int bar,
                                                    int bar64) {
    const int lw = lt >> 5;
    // (1) 16x16 diagonal blocks by substitution, one column per thread
    if (lt < 64) {
        const int I = lt >> 4, jj = lt & 15;
        const float *Ab = AF + (16 * I) * AF_LD + 16 * I;
        float acc[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) acc[t] = (t == jj) ? 1.f : 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float ti = acc[i];
#pragma unroll
            for (int tt = i + 1; tt < 16; ++tt) acc[tt] = fmaf(-Ab[tt * AF_LD + i], ti, acc[tt]);
        }
        bar_named(bar64, 64);   // every read of the diagonal A blocks is done
        float *Tb = AF + (16 * I) * AF_LD + 16 * I + jj;
#pragma unroll
        for (int t = 0; t < 16; ++t) Tb[t * AF_LD] = acc[t];
    }
    bar_named(bar, 128);
    // (2) T_10 = -D_1 A_10 D_0 and T_32 = -D_3 A_32 D_2 (two warps)
    if (lw < 2) {
        const int I = 2 * lw + 1, J = 2 * lw;
        float *tw = TMP + lw * 16 * 20;
        float y[2][4] = {};
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            uint32_t a[4];
            lda(a, AF, AF_LD, 16 * I, 16 * J + 8 * ks, lane);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                uint32_t bb[2];
                ldb(bb, AF, AF_LD, 16 * J + 8 * ks, 16 * J + 8 * nt, lane);
                mma_tf32(y[nt], a, bb);
            }
        }
        stc(tw, 20, 0, 0, y, 1.f, lane);
        __syncwarp();
        float z[2][4] = {};
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            uint32_t a[4];
            lda(a, AF, AF_LD, 16 * I, 16 * I + 8 * ks, lane);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                uint32_t bb[2];
                ldb(bb, tw, 20, 8 * ks, 8 * nt, lane);
                mma_tf32(z[nt], a, bb);
            }
        }
        stc(AF, AF_LD, 16 * I, 16 * J, z, -1.f, lane);
    }
    bar_named(bar, 128);
    // (3) bottom-left 32x32: Z = -Y' (A_[23][01] X'), X' = T[0:32,0:32], Y' = T[32:64,32:64]
    const int mt = lw >> 1, nh = lw & 1;
    float m[2][4] = {};
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
        if (nh == 1 && ks < 2) continue;   // X'[k][16..31] = 0 for k < 16
        uint32_t a[4];
        lda(a, AF, AF_LD, 32 + 16 * mt, 8 * ks, lane);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            uint32_t bb[2];
            ldb(bb, AF, AF_LD, 8 * ks, 16 * nh + 8 * nt, lane);
            mma_tf32(m[nt], a, bb);
        }
    }
    stc(TMP, TMP_LD, 16 * mt, 16 * nh, m, 1.f, lane);
    bar_named(bar, 128);
    float z[2][4] = {};
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
        if (ks >= 2 * (mt + 1)) continue;   // Y'[16mt+r][k] = 0 for k >= 16(mt+1)
        uint32_t a[4];
        lda(a, AF, AF_LD, 32 + 16 * mt, 32 + 8 * ks, lane);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            uint32_t bb[2];
            ldb(bb, TMP, TMP_LD, 8 * ks, 16 * nh + 8 * nt, lane);
            mma_tf32(z[nt], a, bb);
        }
    }
    bar_named(bar, 128);   // all reads of A_[23][01] are done before it is overwritten
    stc(AF, AF_LD, 32 + 16 * mt, 16 * nh, z, -1.f, lane);
    bar_named(bar, 128);
}

}  // namespace gdn

struct GdnPrepParams {
    int64_t B, T, H;
    int nchunks;                  // chunks per (batch, head): ceil(max_seqlen / 64)
    const float *alpha, *beta;
    uint8_t *ws;                  // [B*H*nchunks][ITEM_BYTES]
    const int64_t *cu_seqlens;    // packed sequences, or nullptr (dense)
    int64_t max_seqlen;           // = T for the dense layout
};

// One CTA handles (batch, head, chunk) items in a grid-stride loop.  The next
// item's Q is loaded (TMA) as soon as this item's [Q ; K] K^T MMA has read it,
// its alpha and beta are fetched into registers at the same point, and its K
// once this item's -U MMA has read K.  The grid is sized to the CTAs that are
// resident at once (4 per SM: 55 KB of shared memory, 128 TMEM columns), so
// that the other CTAs of an SM cover a load still in flight.
//
// Per item: [Q ; K] K^T -> P (to the item) and A; T = (I + A)^-1; the item's
// T diag(beta) image; then -U = -(T diag(beta gamma)) K as one M=64, N=128 MMA
// whose A operand is written over AF, and its image.
__global__ void __launch_bounds__(gdn::PREP_THREADS, gdn::PREP_CTAS_PER_SM)
gdn_prep_kernel(const __grid_constant__ CUtensorMap mapq, const __grid_constant__ CUtensorMap mapk,
                const GdnPrepParams p) {
    using namespace gdn;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *tiles = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);   // 1 KB aligned
    PCtl *ctl = reinterpret_cast<PCtl *>(tiles + P_END);
    const uint32_t tb = smem_u32(tiles);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t items = p.B * p.H * (int64_t)p.nchunks;
    float *AF = reinterpret_cast<float *>(tiles + P_AF);
    float *TMP = reinterpret_cast<float *>(tiles + P_TMP);

    if (tid == 0) {
        mbar_init(&ctl->qfull, 1);
        mbar_init(&ctl->kfull, 1);
        mbar_init(&ctl->mma, 1);
        mbar_init(&ctl->mma_u, 1);
        mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        fence_barrier_init();
        tma_prefetch_desc(&mapq);
        tma_prefetch_desc(&mapk);
    }
    if (warp == 0) {
        tmem_alloc(&ctl->tmem_base, PREP_TMEM_COLS);
        tc_fence_before_sync();
    }
    __syncthreads();
    tc_fence_after_sync();
    // the main pass, launched as a programmatic dependent, may be scheduled now: it
    // waits for this grid's completion before it reads anything written here
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const uint32_t tmem = ctl->tmem_base;
    const uint32_t tq = tmem + ((uint32_t)(32 * warp) << 16);

    // item w -> (batch, head, chunk); item counts stay below 2^32 (a workspace of
    // 32 KB per item could not exist otherwise), so 32-bit divisions suffice
    struct ItemPos { int64_t b, h; int c; };
    auto item_pos = [&](int64_t w) {
        const uint32_t wu = (uint32_t)w, nch = (uint32_t)p.nchunks, H = (uint32_t)p.H;
        const uint32_t bh = wu / nch;
        return ItemPos{(int64_t)(bh / H), (int64_t)(bh % H), (int)(wu - bh * nch)};
    };
    // warp 2, lane 0: TMA of item w's Q (kq = 0) or K (kq = 1)
    auto load_half = [&](int64_t w, int kq) {
        const ItemPos ip = item_pos(w);
        const SeqSpan sq = seq_span(p.cu_seqlens, ip.b, p.T, p.max_seqlen, false);
        uint64_t *bar = kq ? &ctl->kfull : &ctl->qfull;
        mbar_arrive_expect_tx(bar, KA * C * 128u);
        for (int a = 0; a < KA; ++a)
            tma_load_4d(tiles + a * P_ACS + (kq ? P_K : 0u), kq ? &mapk : &mapq, bar, 64 * a, (int)ip.h,
                        sq.t0 + ip.c * C, sq.b0);
    };
    // warp 2: item w's alpha, beta for tokens 2*lane, 2*lane+1, loaded unconditionally
    // (a clamped index) so that nothing waits for them before their use one item
    // later, where tokens past T take alpha = 1 and beta = 0
    float al[2] = {1.f, 1.f}, be[2] = {0.f, 0.f};
    bool gin[2] = {false, false};
    auto fetch_gates = [&](int64_t w) {
        const ItemPos ip = item_pos(w);
        const int64_t h = ip.h;
        const int c = ip.c;
        const SeqSpan sq = seq_span(p.cu_seqlens, ip.b, p.T, p.max_seqlen, false);
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int64_t tt = (int64_t)c * C + 2 * lane + e;   // position in the sequence
            gin[e] = tt < sq.len;
            const int64_t idx = gin[e] ? (sq.row0 + tt) * p.H + h : 0;   // element 0 always exists
            al[e] = __ldg(p.alpha + idx);
            be[e] = __ldg(p.beta + idx);
        }
    };

    constexpr uint32_t ID_QK = idesc_bf16(128, 64, false, false);
    constexpr uint32_t ID_U = idesc_bf16(64, 128, false, true);
    // packed sequences: items are enumerated up to the longest sequence, and the
    // chunks past a shorter sequence's end are skipped (nothing reads them).  The
    // next item of this CTA is the first of its stride with a chunk to do; every
    // thread computes it the same way.
    auto next_item = [&](int64_t w) {
        if (p.cu_seqlens)
            for (; w < items; w += gridDim.x) {
                const ItemPos ip = item_pos(w);
                const SeqSpan sq = seq_span(p.cu_seqlens, ip.b, p.T, p.max_seqlen, false);
                if ((int64_t)ip.c * C < sq.len) break;
            }
        return w;
    };
    int it = 0;
    const int64_t w0 = next_item(blockIdx.x);
    if (warp == 2 && w0 < items) {
        if (lane == 0) {
            load_half(w0, 0);
            load_half(w0, 1);
        }
        fetch_gates(w0);
    }
    // copies in flight (thread 64's view)
    bool q_pending = w0 < items, k_pending = q_pending;
    const uint32_t kb = tb + P_K;   // the K rows (atom column 0)
    for (int64_t w = w0, wn = next_item(w0 + gridDim.x); w < items; w = wn, wn = next_item(wn + gridDim.x), ++it) {
        if (warp == 2) {   // this item's gates (fetched one item ahead) into shared memory
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                ctl->alpha[2 * lane + e] = gin[e] ? al[e] : 1.f;
                ctl->beta[2 * lane + e] = gin[e] ? be[e] : 0.f;
            }
        }
        if (tid == 0) ctl->stop = ctl->abort;   // one thread decides, everyone reads after the barrier
        bar_named(1, 128);
        if (ctl->stop) break;
        bool landed = mbar_wait(&ctl->qfull, (uint32_t)it & 1u);
        landed = mbar_wait(&ctl->kfull, (uint32_t)it & 1u) && landed;
        if (!landed) ctl->abort = 1;
        if (tid == 64) q_pending = k_pending = false;
        if (warp == 0)
            ctl->fast = gate_scan(&ctl->alpha[2 * lane], ctl->beta, ctl->b2, ctl->gam, ctl->ginv, nullptr, lane);
        if (tid == 32) {   // [Q ; K] K^T: rows 0-63 Q K^T, rows 64-127 K K^T
            tc_fence_after_sync();
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk)
                umma_bf16(tmem, desc_k(tb, P_ACS, kk), desc_k(kb, P_ACS, kk), ID_QK, kk > 0);
            umma_commit(&ctl->mma);
        }
        bar_named(1, 128);
        if (!mbar_wait(&ctl->mma, (uint32_t)it & 1u)) ctl->abort = 1;
        tc_fence_after_sync();
        // Q is free: start the next item's Q and gates
        if (warp == 2 && wn < items) {
            if (lane == 0 && !ctl->abort) {
                load_half(wn, 0);
                q_pending = true;
            }
            fetch_gates(wn);
        }
        {   // row r = tid of the M=128 accumulator: warps 0-1 the P row of token r
            // (inclusive mask, to the item's P image), warps 2-3 the A row of token
            // r - 64 (strict mask, times beta, to AF)
            const int t = tid & 63;
            const bool prow = warp < 2;
            float x[64];
            tmem_ld32(tq, *reinterpret_cast<float(*)[32]>(x));
            tmem_ld32(tq + 32u, *reinterpret_cast<float(*)[32]>(x + 32));
            tmem_wait_ld();
            if (prow) {
                decay_mask_row<false>(x, t, t < 32 ? 32 : 64, 1.f, ctl->fast != 0, ctl->gam, ctl->ginv, ctl->b2);
                uint8_t *dst = p.ws + w * (int64_t)ITEM_BYTES + ITEM_P + (uint32_t)t * 128u;
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) {
                    uint4 u;
                    u.x = pack_bf16x2(x[8 * cc + 0], x[8 * cc + 1]);
                    u.y = pack_bf16x2(x[8 * cc + 2], x[8 * cc + 3]);
                    u.z = pack_bf16x2(x[8 * cc + 4], x[8 * cc + 5]);
                    u.w = pack_bf16x2(x[8 * cc + 6], x[8 * cc + 7]);
                    *reinterpret_cast<uint4 *>(dst + (uint32_t)(((cc ^ t) & 7) << 4)) = u;
                }
            } else {
                decay_mask_row<true>(x, t, t < 32 ? 32 : 64, ctl->beta[t], ctl->fast != 0, ctl->gam, ctl->ginv,
                                     ctl->b2);
                float *arow = AF + t * AF_LD;
#pragma unroll
                for (int i = 0; i < 64; i += 4)
                    *reinterpret_cast<float4 *>(arow + i) = make_float4(x[i], x[i + 1], x[i + 2], x[i + 3]);
            }
        }
        tc_fence_before_sync();
        bar_named(1, 128);
        invert_unit_lower64(AF, TMP, tid, lane, 1, 2);
        {   // T diag(beta) -> the item; T diag(beta gamma) -> the -U MMA's A operand,
            // written over AF once every thread has read its part of T
            const int t = tid >> 1, hh = tid & 1;
            const float4 *Trow = reinterpret_cast<const float4 *>(AF + t * AF_LD + 32 * hh);
            const float4 *be4 = reinterpret_cast<const float4 *>(ctl->beta + 32 * hh);
            const float4 *ga4 = reinterpret_cast<const float4 *>(ctl->gam + 32 * hh);
            uint8_t *dst = p.ws + w * (int64_t)ITEM_BYTES + ITEM_T;
            uint4 ug[4];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                float tv[8], bv[8], gv[8];
#pragma unroll
                for (int hq = 0; hq < 2; ++hq) {
                    const float4 a = Trow[2 * cc + hq], bb = be4[2 * cc + hq], g = ga4[2 * cc + hq];
                    tv[4 * hq] = a.x; tv[4 * hq + 1] = a.y; tv[4 * hq + 2] = a.z; tv[4 * hq + 3] = a.w;
                    bv[4 * hq] = bb.x; bv[4 * hq + 1] = bb.y; bv[4 * hq + 2] = bb.z; bv[4 * hq + 3] = bb.w;
                    gv[4 * hq] = g.x; gv[4 * hq + 1] = g.y; gv[4 * hq + 2] = g.z; gv[4 * hq + 3] = g.w;
                }
                uint4 u;
                uint32_t *pu = &u.x, *pg = &ug[cc].x;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    pu[e] = pack_bf16x2(tv[2 * e] * bv[2 * e], tv[2 * e + 1] * bv[2 * e + 1]);
                    pg[e] = pack_bf16x2(tv[2 * e] * (bv[2 * e] * gv[2 * e]),
                                        tv[2 * e + 1] * (bv[2 * e + 1] * gv[2 * e + 1]));
                }
                const int chunk = 4 * hh + cc;
                *reinterpret_cast<uint4 *>(dst + (uint32_t)t * 128u + (uint32_t)(((chunk ^ t) & 7) << 4)) = u;
            }
            bar_named(1, 128);   // every read of T is done
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                const int chunk = 4 * hh + cc;
                *reinterpret_cast<uint4 *>(tiles + P_AF + (uint32_t)t * 128u + (uint32_t)(((chunk ^ t) & 7) << 4)) =
                    ug[cc];
            }
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        bar_named(1, 128);
        if (tid == 32) {   // U = (T diag(beta gamma)) K: M=64 tokens, N=128 key columns, K=64 tokens
            tc_fence_after_sync();
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk)
                umma_bf16(tmem, desc_k(tb + P_AF, C * 128, kk), desc_mn128(kb, P_ACS, kk), ID_U, kk > 0);
            umma_commit(&ctl->mma_u);
        }
        if (!mbar_wait(&ctl->mma_u, (uint32_t)it & 1u)) ctl->abort = 1;
        tc_fence_after_sync();
        // K is free: the next item's K
        if (tid == 64 && wn < items && !ctl->abort) {
            load_half(wn, 1);
            k_pending = true;
        }
        {   // -U -> the item: row tr = 16 warp + (lane & 15) of the M=64 accumulator,
            // key columns 64 hf .. 64 hf + 63 = block hf of the image
            const int tr = 16 * warp + (lane & 15), hf = lane >> 4;
            float x[64];
            tmem_ld16x2_32<64>(tq, *reinterpret_cast<float(*)[32]>(x));
            tmem_ld16x2_32<64>(tq + 32u, *reinterpret_cast<float(*)[32]>(x + 32));
            tmem_wait_ld();
            uint8_t *dst = p.ws + w * (int64_t)ITEM_BYTES + ITEM_U + (uint32_t)hf * 8192u + (uint32_t)tr * 128u;
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
                uint4 u;
                u.x = pack_bf16x2(-x[8 * cc + 0], -x[8 * cc + 1]);
                u.y = pack_bf16x2(-x[8 * cc + 2], -x[8 * cc + 3]);
                u.z = pack_bf16x2(-x[8 * cc + 4], -x[8 * cc + 5]);
                u.w = pack_bf16x2(-x[8 * cc + 6], -x[8 * cc + 7]);
                *reinterpret_cast<uint4 *>(dst + (uint32_t)(((cc ^ tr) & 7) << 4)) = u;
            }
        }
        tc_fence_before_sync();
        bar_named(1, 128);   // AF, TMEM and the gates are reused by the next item
    }
    // let a prefetched copy land and every MMA finish before the CTA frees TMEM
    // and exits (these two waits keep the long limit even after a timeout)
    if (tid == 64 && q_pending) (void)mbar_drain(&ctl->qfull, (uint32_t)it & 1u);
    if (tid == 64 && k_pending) (void)mbar_drain(&ctl->kfull, (uint32_t)it & 1u);
    if (tid == 32) {
        umma_commit(&ctl->drain);
        (void)mbar_drain(&ctl->drain, 0u);
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 0) tmem_dealloc(tmem, PREP_TMEM_COLS);
}



namespace gdn {
// Shared memory of gdn_main_kernel (byte offsets from a 1 KB aligned base).
//   ring A, 2 stages: [Q ; -U] as two atom columns of 128 rows (Q rows 0-63 from
//     q by TMA, -U rows 64-127 from the item), the A operand of
//     [X2 ; W] += [Q ; -U] S0;
//   ring B, 3 stages: Z | T diag(beta) | P | K | V, where [Z ; T diag(beta)] is
//     the A operand of [X2 ; W] = [0 ; T diag(beta)] V (Z stays zero), [P ; K0]
//     that of PW (rows 64-127, the first K block, give rows of the accumulator
//     that are never read) and K that of dS = K^T diag(gamma_C / gamma) W;
//   W (2 buffers) and diag(gamma_C / gamma) W, bf16 [64][32], and S0, bf16
//     [128][32], all with the 64-byte swizzle.
template <bool KDA>
struct ML {
    static constexpr int NA = 2, NB = 3;
    static constexpr uint32_t A_BYTES = 2 * QK_ACS;
    static constexpr uint32_t B_Z = 0, B_T = 8192, B_P = 16384, B_K = 24576, B_V = 40960;
    static constexpr uint32_t B_GC = 45056;                     // KDA: Gamma_C, fp32 [128]
    static constexpr uint32_t B_BYTES = KDA ? 46080 : 45056;    // stages stay 1 KB aligned
    static constexpr uint32_t SA = 0;
    static constexpr uint32_t SB = SA + NA * A_BYTES;
    static constexpr uint32_t TWS = SB + NB * B_BYTES;
    static constexpr uint32_t TWGS = TWS + 2 * 4096;
    static constexpr uint32_t TSS = TWGS + 4096;
    static constexpr uint32_t TEND = TSS + 8192;
};
// TMEM columns of gdn_main_kernel
constexpr uint32_t M_TMEM_COLS = 256;
constexpr uint32_t M_XW = 0;    // 2 x 32, M=128 [X2 ; W] (chunk c in buffer c & 1)
constexpr uint32_t M_DS = 64;   // 32,     M=128 dS
constexpr uint32_t M_PW = 96;   // 2 x 32, M=128 [P ; K0] W (rows 0-63)

struct MCtl {
    uint64_t fullA[2], emptyA[2], fullB[3], emptyB[3];
    uint64_t wready[2], pw_done[2], w0_done[2], xk_done, ds_done, drain;
    uint32_t tmem_base;
    int abort, stopS, stopL[2];
    // the gated delta rule, per ring-B stage: b = log2 of the inclusive cumulative
    // alpha, gamma = 2^b, 1/gamma and gamma_C / gamma (written by the producer)
    float b2[3][64], gam[3][64], ginv[3][64], gct[3][64];
};
static_assert(ML<false>::NA == 2 && ML<false>::NB == 3, "MCtl's barrier arrays follow the rings");
}  // namespace gdn

// The gated delta rule's main pass (one CTA per (batch, head, 32-column value
// slab), 9 warps).  With the item's T diag(beta) and -U, the state enters a
// chunk's work through one MMA chain whose accumulator already holds the
// state-independent part:
//   [X2 ; W] = [0 ; T diag(beta)] V + [Q ; -U] S0      (X2 = Q S0)
//   dS = K^T diag(gamma_C / gamma) W,   S <- gamma_C S + dS   (fp32 carry)
//   O  = diag(gamma) X2 + P W.
//   warp 0      producer: ring A (Q by TMA, -U from the item) and ring B (K, V
//               by TMA; T diag(beta), P from the item; the decay factors);
//   warps 1-4   output group: PW = [P ; K0] W and O, then the accumulator of
//               the chunk after next: [0 ; T diag(beta)] V;
//   warps 5-8   state group: W -> bf16 (and diag(gamma_C / gamma) W), dS, the
//               state update, and [Q ; -U] S0 of the next chunk.
// KDA = true: the KDA main pass on kda_prep_kernel's outputs (chunk_kda.cuh has
// the algebra): maps.q and maps.kc cover its Qp = Q o Gamma and Kc = K o
// Gamma_C / Gamma, and its items hold T diag(beta), P, -U = -T diag(beta)(K o
// Gamma) and Gamma_C.  Then X2 = Qp S0 already carries the decay, dS = Kc^T W,
// and the state row d decays by Gamma_C[d].
template <bool KDA>
__global__ void __launch_bounds__(gdn::NTHREADS, 1)
gdn_main_kernel(const __grid_constant__ Maps maps, const ChunkParams p, const uint8_t *ws) {
    using namespace gdn;
    using L = ML<KDA>;
    constexpr uint32_t ITEM = KDA ? kda::ITEM_BYTES : ITEM_BYTES;   // workspace bytes per chunk
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    MCtl *ctl = reinterpret_cast<MCtl *>(smem_raw);
    uint8_t *tiles = smem_raw + align1k((uint32_t)sizeof(MCtl) + (smem_u32(smem_raw) & 1023u)) -
                     (smem_u32(smem_raw) & 1023u);
    const uint32_t tb = smem_u32(tiles);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3;
    const int nslab = (int)(p.dv / DVT);
    const int dvt = (int)(blockIdx.x % nslab);
    const int64_t bh = blockIdx.x / nslab;
    const int64_t b = bh / p.H, h = bh % p.H;
    // this sequence's tokens (dense: all T of batch b); items are stored for
    // ceil(max_seqlen / 64) chunks per (batch, head)
    const SeqSpan sq = seq_span(p.cu_seqlens, b, p.T, p.max_seqlen, tid == 0 && h == 0 && dvt == 0);
    const int nchunks = (int)((sq.len + C - 1) / C);
    const int64_t ws_chunks = (p.max_seqlen + C - 1) / C;

    if (tid == 0) {
        for (int s = 0; s < L::NA; ++s) {
            mbar_init(&ctl->fullA[s], 1);
            mbar_init(&ctl->emptyA[s], 1);   // [Q ; -U] S0 has read the stage
        }
        for (int s = 0; s < L::NB; ++s) {
            mbar_init(&ctl->fullB[s], 32);
            mbar_init(&ctl->emptyB[s], 2);   // dS and PW have read the stage
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&ctl->wready[i], 128);
            mbar_init(&ctl->pw_done[i], 1);
            mbar_init(&ctl->w0_done[i], 1);
        }
        mbar_init(&ctl->xk_done, 1);
        mbar_init(&ctl->ds_done, 1);
        mbar_init(&ctl->drain, 2);   // one commit from each MMA-issuing thread
        ctl->abort = 0;
        fence_barrier_init();
        tma_prefetch_desc(&maps.q);
        tma_prefetch_desc(KDA ? &maps.kc : &maps.k);
        tma_prefetch_desc(&maps.v);
    }
    if (warp == 0) {
        tmem_alloc(&ctl->tmem_base, M_TMEM_COLS);
        tc_fence_before_sync();
    }
    for (int i = tid; i < L::NB * 8192 / 16; i += NTHREADS) {   // the Z blocks stay zero
        const int st = i / 512, off = (i % 512) * 16;
        *reinterpret_cast<uint4 *>(tiles + L::SB + st * L::B_BYTES + L::B_Z + off) = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = ctl->tmem_base;
    const uint32_t tq = tmem + ((uint32_t)(32 * quad) << 16);   // this warp's TMEM lanes

    constexpr uint32_t ID_XW = idesc_bf16(128, DVT, false, true);
    constexpr uint32_t ID_DS = idesc_bf16(128, DVT, true, true);
    auto stage_a = [&](int c) { return L::SA + (uint32_t)(c & 1) * L::A_BYTES; };
    auto stage_b = [&](int c) { return L::SB + (uint32_t)(c % L::NB) * L::B_BYTES; };

    if (warp == 0) {
        // ------------------------------------------------------------------ producer
        // launched as a programmatic dependent of the prep kernel: its items (and,
        // for KDA, Qp and Kc) are complete and visible once this returns; nothing
        // else in this kernel reads them but through the producer's copies
        asm volatile("griddepcontrol.wait;" ::: "memory");
        float al[2] = {1.f, 1.f};   // the alphas of the chunk to be issued next
        auto fetch = [&](int c) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int64_t tt = (int64_t)c * C + 2 * lane + e;
                al[e] = tt < sq.len ? p.g[(sq.row0 + tt) * p.H + h] : 1.f;
            }
        };
        // whole warp: wait (if `need`) until the slot's last readers are done; false
        // once the CTA is aborting (lane 0 decides, so the warp leaves together)
        auto acquire = [&](uint64_t *bar, uint32_t parity, bool need) {
            if (need) {
                int ok = 1;
                if (lane == 0) ok = mbar_wait(bar, parity);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok && lane == 0) ctl->abort = 1;
            }
            const int stop = (lane == 0) ? ctl->abort : 0;
            return __shfl_sync(0xffffffffu, stop, 0) == 0;
        };
        if (!KDA && nchunks > 0) fetch(0);
        int issuedA = 0, issuedB = 0;
        for (int c = 0; c < nchunks; ++c) {
            const int tm = sq.t0 + c * C;   // tensor-map coordinate of the chunk's first token
            // KDA: the prep's Qp, Kc (one row block per sequence, even when packed)
            const int tqk = KDA ? c * C : tm, bqk = KDA ? (int)b : sq.b0;
            const uint8_t *item = ws + (bh * ws_chunks + c) * (int64_t)ITEM;
            const int a = c & 1, s = c % L::NB;
            if (!acquire(&ctl->emptyA[a], (uint32_t)((c >> 1) - 1) & 1u, c >= L::NA)) break;
            if (lane == 0) {
                uint8_t *qa = tiles + stage_a(c);
                mbar_arrive_expect_tx(&ctl->fullA[a], 2u * KA * C * 128u);
#pragma unroll
                for (int ka = 0; ka < KA; ++ka) {
                    tma_load_4d(qa + ka * QK_ACS, &maps.q, &ctl->fullA[a], 64 * ka, (int)h, tqk, bqk);
                    bulk_load(qa + ka * QK_ACS + 64 * 128, item + ITEM_U + ka * 8192, 8192, &ctl->fullA[a]);
                }
            }
            issuedA = c + 1;
            if (!acquire(&ctl->emptyB[s], (uint32_t)((c / L::NB) - 1) & 1u, c >= L::NB)) break;
            if (lane == 0) {
                uint8_t *sb = tiles + stage_b(c);
                mbar_expect_tx(&ctl->fullB[s], KA * C * 128u + C * DVT * 2u + 2u * TT_BYTES + (KDA ? 512u : 0u));
#pragma unroll
                for (int ka = 0; ka < KA; ++ka)
                    tma_load_4d(sb + L::B_K + ka * 8192, KDA ? &maps.kc : &maps.k, &ctl->fullB[s], 64 * ka, (int)h,
                                tqk, bqk);
                tma_load_4d(sb + L::B_V, &maps.v, &ctl->fullB[s], dvt * DVT, (int)h, tm, sq.b0);
                bulk_load(sb + L::B_T, item + ITEM_T, TT_BYTES, &ctl->fullB[s]);
                bulk_load(sb + L::B_P, item + ITEM_P, TT_BYTES, &ctl->fullB[s]);
                if (KDA) bulk_load(sb + L::B_GC, item + kda::ITEM_GC, 512, &ctl->fullB[s]);
            }
            if constexpr (!KDA) {
                // the chunk's decay factors: gamma = 2^b, gamma_C / gamma = 2^(b_63 - b)
                (void)gate_scan(al, nullptr, ctl->b2[s], ctl->gam[s], ctl->ginv[s], nullptr, lane);
                const float blast = __shfl_sync(0xffffffffu, ctl->b2[s][2 * lane + 1], 31);
                __syncwarp();
                ctl->gct[s][2 * lane] = exp2f(blast - ctl->b2[s][2 * lane]);
                ctl->gct[s][2 * lane + 1] = exp2f(blast - ctl->b2[s][2 * lane + 1]);
                if (c + 1 < nchunks) fetch(c + 1);   // in flight while the next slots free up
            }
            mbar_arrive(&ctl->fullB[s]);
            issuedB = c + 1;
        }
        // let copies still in flight land before the CTA can exit
        if (lane == 0) {
            for (int c = (issuedA > L::NA ? issuedA - L::NA : 0); c < issuedA; ++c)
                (void)mbar_drain(&ctl->fullA[c & 1], (uint32_t)(c >> 1) & 1u);
            for (int c = (issuedB > L::NB ? issuedB - L::NB : 0); c < issuedB; ++c)
                (void)mbar_drain(&ctl->fullB[c % L::NB], (uint32_t)(c / L::NB) & 1u);
        }
    } else if (warp < 5) {
        // ------------------------------------------------------------------ output group
        const int lt = tid - 32;
        const bool leader = (lt == 0);
        const int ro = 32 * quad + lane;   // M=128 row: output rows 0-63 in quads 0, 1
        // [X2 ; W] = [0 ; T diag(beta)] V of chunk c
        auto issue_w0 = [&](int c) {
            const uint32_t zb = tb + stage_b(c) + L::B_Z, vb = tb + stage_b(c) + L::B_V;
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk)
                umma_bf16(tmem + M_XW + 32u * (uint32_t)(c & 1), desc_k(zb, 16384, kk), desc_mn64(vb, kk), ID_XW,
                          kk > 0);
            umma_commit(&ctl->w0_done[c & 1]);
        };
        if (leader)   // chunks 0 and 1 into the two accumulator buffers
            for (int c = 0; c < 2 && c < nchunks; ++c) {
                if (!mbar_wait(&ctl->fullB[c], 0u)) ctl->abort = 1;
                tc_fence_after_sync();
                issue_w0(c);
            }
        // PW = [P ; K0] W and O = diag(gamma) X2 + PW of chunk j (a failed wait sets
        // the abort flag; every thread still takes every barrier)
        auto finish = [&](int j) {
            const int sj = j % L::NB, jb = j & 1;
            const int64_t tj = (int64_t)j * C;
            const int nvalid = (int)min((int64_t)C, sq.len - tj);
            if (!mbar_wait(&ctl->wready[jb], (uint32_t)(j >> 1) & 1u)) ctl->abort = 1;
            // read before the stage can be refilled (KDA: X2 = Qp S0 already decays)
            const float gam_o = KDA ? 1.f : ctl->gam[sj][ro & 63];
            bar_named(1, 128);
            if (leader) {
                // stage j landed long ago (the state group has its W); the wait makes the
                // copy's completion visible to this thread
                if (!mbar_wait(&ctl->fullB[sj], (uint32_t)(j / L::NB) & 1u)) ctl->abort = 1;
                tc_fence_after_sync();
                const uint32_t ps = tb + stage_b(j) + L::B_P;
                const uint32_t wsb = tb + L::TWS + (uint32_t)jb * 4096u;
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    umma_bf16(tmem + M_PW + 32u * jb, desc_k(ps, 16384, kk), desc_mn64(wsb, kk), ID_XW, kk > 0);
                umma_commit(&ctl->pw_done[jb]);
                umma_commit(&ctl->emptyB[sj]);
            }
            if (!mbar_wait(&ctl->pw_done[jb], (uint32_t)(j >> 1) & 1u)) ctl->abort = 1;
            tc_fence_after_sync();
            if (quad < 2) {
                float x2[32], pw[32];
                tmem_ld32(tq + M_XW + 32u * jb, x2);
                tmem_ld32(tq + M_PW + 32u * jb, pw);
                tmem_wait_ld();
                if (ro < nvalid) {
                    __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(p.o) +
                                         ((sq.row0 + tj + ro) * p.H + h) * p.dv + dvt * DVT;
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
                        uint4 u;
                        u.x = pack_bf16x2(fmaf(gam_o, x2[8 * cc + 0], pw[8 * cc + 0]),
                                          fmaf(gam_o, x2[8 * cc + 1], pw[8 * cc + 1]));
                        u.y = pack_bf16x2(fmaf(gam_o, x2[8 * cc + 2], pw[8 * cc + 2]),
                                          fmaf(gam_o, x2[8 * cc + 3], pw[8 * cc + 3]));
                        u.z = pack_bf16x2(fmaf(gam_o, x2[8 * cc + 4], pw[8 * cc + 4]),
                                          fmaf(gam_o, x2[8 * cc + 5], pw[8 * cc + 5]));
                        u.w = pack_bf16x2(fmaf(gam_o, x2[8 * cc + 6], pw[8 * cc + 6]),
                                          fmaf(gam_o, x2[8 * cc + 7], pw[8 * cc + 7]));
                        reinterpret_cast<uint4 *>(dst)[cc] = u;
                    }
                }
            }
            tc_fence_before_sync();
            bar_named(1, 128);   // X2 and PW of buffer jb are read
            if (leader && j + 2 < nchunks) {
                // chunk j+2's [0 ; T diag(beta)] V into the buffer just read (the state
                // group read W of chunk j from it before wready)
                if (!mbar_wait(&ctl->fullB[(j + 2) % L::NB], (uint32_t)((j + 2) / L::NB) & 1u)) ctl->abort = 1;
                tc_fence_after_sync();
                issue_w0(j + 2);
            }
        };
        for (int j = 0; j < nchunks; ++j) {
            const int pb = j & 1;
            if (leader) ctl->stopL[pb] = ctl->abort;
            bar_named(1, 128);
            if (ctl->stopL[pb]) break;
            finish(j);
        }
        if (leader) umma_commit(&ctl->drain);
    } else {
        // ------------------------------------------------------------------ state group
        const int st = tid - 160;
        const bool leader = (st == 0);
        const int d = 32 * quad + lane;   // state row
        float S[DVT];
        {
            const float *src = p.S0 ? p.S0 + ((bh * DK + d) * p.dv + dvt * DVT) : nullptr;
#pragma unroll
            for (int j = 0; j < DVT; j += 4) {
                float4 x = src ? *reinterpret_cast<const float4 *>(src + j) : make_float4(0, 0, 0, 0);
                S[j] = x.x; S[j + 1] = x.y; S[j + 2] = x.z; S[j + 3] = x.w;
            }
            store_row64(tiles + L::TSS, d, S);
        }
        fence_proxy_async_smem();
        bar_named(2, 128);
        // [X2 ; W] += [Q ; -U] S0 of chunk c, once [0 ; T diag(beta)] V of chunk c is
        // in the accumulator and the ring-A stage has landed
        auto issue_xk = [&](int c) {
            bool ok = mbar_wait(&ctl->w0_done[c & 1], (uint32_t)(c >> 1) & 1u);
            ok = mbar_wait(&ctl->fullA[c & 1], (uint32_t)(c >> 1) & 1u) && ok;
            if (!ok) ctl->abort = 1;
            tc_fence_after_sync();
            const uint32_t qa = tb + stage_a(c);
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk)
                umma_bf16(tmem + M_XW + 32u * (uint32_t)(c & 1), desc_k(qa, QK_ACS, kk),
                          desc_mn64(tb + L::TSS, kk), ID_XW, 1u);
            umma_commit(&ctl->xk_done);
            umma_commit(&ctl->emptyA[c & 1]);
        };
        if (leader && nchunks > 0) issue_xk(0);
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % L::NB, pb = c & 1;
            if (leader) ctl->stopS = ctl->abort;
            bar_named(2, 128);
            if (ctl->stopS) break;
            bool ok = mbar_wait(&ctl->fullB[s], (uint32_t)(c / L::NB) & 1u);
            ok = mbar_wait(&ctl->xk_done, (uint32_t)c & 1u) && ok;
            if (!ok) ctl->abort = 1;
            tc_fence_after_sync();
            // decay of state row d over the chunk, read before the stage can be refilled
            const float gC = KDA ? reinterpret_cast<const float *>(tiles + stage_b(c) + L::B_GC)[d]
                                 : ctl->gam[s][C - 1];
            if (quad >= 2) {   // W row t -> bf16 W (for PW) and diag(gamma_C / gamma) W (for dS;
                               // KDA: Kc carries Gamma_C / Gamma and dS reads W itself)
                const int t = d - 64;
                // PW of chunk c-2 has read W buffer pb
                if (c >= 2 && !mbar_wait(&ctl->pw_done[pb], (uint32_t)((c - 2) >> 1) & 1u)) ctl->abort = 1;
                float w[32];
                tmem_ld32(tq + M_XW + 32u * pb, w);
                const float g = KDA ? 1.f : ctl->gct[s][t];
                tmem_wait_ld();
                store_row64(tiles + L::TWS + (uint32_t)pb * 4096u, t, w);
                if (!KDA) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) w[j] *= g;
                    store_row64(tiles + L::TWGS, t, w);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            mbar_arrive(&ctl->wready[pb]);   // the output group may issue PW(c)
            bar_named(2, 128);
            if (leader) {   // dS = K^T diag(gamma_C / gamma) W (KDA: Kc^T W), K = tokens
                tc_fence_after_sync();
                const uint32_t kb = tb + stage_b(c) + L::B_K;
                const uint32_t wb = KDA ? tb + L::TWS + (uint32_t)pb * 4096u : tb + L::TWGS;
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    umma_bf16(tmem + M_DS, desc_mn128(kb, C * 128, kk), desc_mn64(wb, kk), ID_DS, kk > 0);
                umma_commit(&ctl->ds_done);
                umma_commit(&ctl->emptyB[s]);
            }
            if (!mbar_wait(&ctl->ds_done, (uint32_t)c & 1u)) ctl->abort = 1;
            tc_fence_after_sync();
            {   // S <- gamma_C S + dS, then its bf16 copy for chunk c+1 ([Q ; -U] S0 of
                // chunk c has finished: xk_done)
                float ds[DVT];
                tmem_ld32(tq + M_DS, ds);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < DVT; ++j) S[j] = fmaf(gC, S[j], ds[j]);
                store_row64(tiles + L::TSS, d, S);
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            bar_named(2, 128);
            if (leader && c + 1 < nchunks) issue_xk(c + 1);
        }
        if (leader) {   // every MMA issued by either group has finished before TMEM is released
            umma_commit(&ctl->drain);
            (void)mbar_drain(&ctl->drain, 0u);
        }
        if (!ctl->abort && p.S_out) {
            float *dst = p.S_out + ((bh * DK + d) * p.dv + dvt * DVT);
#pragma unroll
            for (int j = 0; j < DVT; j += 4)
                *reinterpret_cast<float4 *>(dst + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 0) tmem_dealloc(tmem, M_TMEM_COLS);
}

}  // namespace ck
}  // namespace la
