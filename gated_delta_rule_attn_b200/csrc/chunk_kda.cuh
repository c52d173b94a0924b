// chunk_kda.cuh — KDA (per-key-channel retention with the delta rule), chunked
// prefill: a parallel prep kernel here, then gdn_main_kernel<true> (chunk_gdn.cuh).
//
// Rule (page "状态空间与线性注意力", KDA：逐通道遗忘与误差写入), per token:
//   S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,  o_t = S_t^T q_t,
// alpha_t in (0, 1]^dk.  Inside a 64-token chunk, with Gamma_t = prod_{s<=t} alpha_s
// (per key channel) and S0 the state entering the chunk, unrolling the update as
// for the gated delta rule gives S_t = Diag(Gamma_t) S0 + sum_{i<=t}
// Diag(Gamma_t / Gamma_i) k_i w_i^T, hence
//   A  = diag(beta) (((K o Gamma)(K / Gamma)^T) o strict-lower),  T = (I + A)^-1,
//   W  = T diag(beta) (V - (K o Gamma) S0),
//   O  = (Q o Gamma) S0 + P W,   P = ((Q o Gamma)(K / Gamma)^T) o M,
//   S <- Diag(Gamma_C) S0 + (K o Gamma_C / Gamma)^T W.
// The state-independent parts (P, T) need the pairwise factors Gamma_t / Gamma_i,
// which a 64-token chunk cannot write as a product of per-token factors in fp32
// (the page bounds log alpha to (-5, 0): e^-320 over a chunk).  The page's
// remedy is short sub-tiles; here each 16-token sub-chunk s takes its middle
// token m_s (the 8th) as reference: with G_t = Gamma_t / Gamma_{m_s} and
// H_t = 1 / G_t for t in s (both within 2^(+-58) under the page's bound), a query
// row t of sub-chunk a against key row i of sub-chunk s <= a is
//   (q_t o G_t) . (k_i o H_i o Gamma_{m_a} / Gamma_{m_s}),
// the last factor a product of sub-chunk gate products (<= 1).  So for each of
// the 4 query sub-chunks one MMA [Qs ; Ks] Kr_a^T (M = 128, N = 64, K = 128) gives
// that sub-chunk's rows of P and A; Kr_a holds the keys of sub-chunks <= a scaled
// for reference m_a.  Every factor is a product of alphas or the reciprocal of
// one (one rcp per element, no exp/log).  The products across sub-chunks are
// formed with a 2^64 prescale and met by G or H times 2^-64, so every product
// that can reach the result stays a normal fp32 number.  The kernel raises
// kErrRange outside the domain where every 8-token retention product is
// >= 2^-60 (which the page's bound log alpha > -5 satisfies).
//
// kda_prep_kernel, one (batch, head, chunk) item per CTA iteration (grid-stride,
// 4 warps, 2 CTAs per SM), writes to the workspace:
//   per item: the images of T diag(beta), P and -U = -T diag(beta) (K o Gamma)
//   (bf16, 128-byte swizzled, the shared-memory operand layout of
//   gdn_main_kernel; U by one M=64, N=128 MMA) and Gamma_C (fp32 [128]);
//   per token: Qp = q o Gamma and Kc = k o Gamma_C / Gamma as bf16 [B,Ls,H,128]
//   tensors, which gdn_main_kernel<true> loads by TMA in place of q and k.
// With W = T diag(beta) (V - (K o Gamma) S0) = T diag(beta) V - U S0 the main
// pass runs the gated delta rule's chain unchanged.
//   Dense layout: Ls = T.  Packed sequences: one row block per sequence,
//   Ls = 64 ceil(max_seqlen / 64), so a sequence's tail chunk owns its padding
//   rows, which are written as zeros (the next sequence's tokens never appear
//   in its chunks).
// Warp w owns sub-chunk w: lane l holds key channels 4l..4l+3 of its 16 tokens.
#pragma once

#include "device.cuh"

namespace la {
namespace ck {
namespace kda {

constexpr int PREP_THREADS = 128;
// (the per-chunk item layout, ITEM_*, is in chunk_gdn.cuh beside its reader)
constexpr uint32_t QS_ACS = 128 * 128;         // [Qs ; Ks] atom column: 128 rows x 128 B
// Kr_a holds the keys of sub-chunks 0..a: 16 (a + 1) rows, two atom columns
__host__ __device__ constexpr uint32_t kr_acs(int a) { return 2048u * (uint32_t)(a + 1); }
__host__ __device__ constexpr uint32_t kr_off(int a) { return 2048u * (uint32_t)(a * (a + 1)); }
constexpr uint32_t P_QS = 0;                   // [Qs ; Ks], rows 32w..32w+15 = Qs of sub-chunk w,
                                               // rows 32w+16..32w+31 = Ks of sub-chunk w
constexpr uint32_t P_KR = 2 * QS_ACS;          // Kr_a, a = 0..3 (40 KB)
constexpr uint32_t P_KP = P_KR + kr_off(4);    // K o Gamma, [64][128], two atom columns of 8 KB
constexpr uint32_t P_END = P_KP + 16384;
// A, then T (fp32 [64][AF_LD]), and the merge scratch reuse [Qs ; Ks] once the
// MMAs that read it are done
constexpr uint32_t P_AF = P_QS;
constexpr uint32_t P_TMP = P_AF + 64 * gdn::AF_LD * 4;
static_assert(P_TMP + 32 * gdn::TMP_LD * 4 <= P_KR, "A/T scratch must fit in the [Qs ; Ks] tile");
constexpr float kMinFactor = 8.673617379884035e-19f;   // 2^-60
constexpr float kUp = 18446744073709551616.f;          // 2^64
constexpr float kDown = 5.421010862427522e-20f;        // 2^-64

}  // namespace kda

struct KCtl {
    uint64_t mma, mma_u, drain;
    uint32_t tmem_base;
    int abort, stop;
    // per sub-chunk and key channel: the product of alpha over its tokens up to
    // and including the middle one (D) and over the tokens after it (U)
    alignas(16) float D[4][128];
    alignas(16) float U[4][128];
    alignas(16) float beta[64];   // read as float4
};

struct KdaPrepParams {
    int64_t B, T, H;
    int nchunks;                      // chunks per (sequence, head): ceil(max_seqlen / 64)
    int64_t Ls;                       // token extent of qp, kc: T, or 64 nchunks when packed
    const __nv_bfloat16 *q, *k;       // [B,T,H,128] (packed: [1,T,H,128])
    const float *alpha, *beta;        // [B,T,H,128], [B,T,H] (packed: [1,T,H,*])
    uint8_t *items;                   // [B*H*nchunks][ITEM_BYTES]
    __nv_bfloat16 *qp, *kc;           // [B,Ls,H,128]
    const int64_t *cu_seqlens;        // packed sequences, or nullptr (dense)
    int64_t max_seqlen;               // = T for the dense layout
};

// Four products as two packed fp32x2 multiplies.
__device__ __forceinline__ float4 mul4(float4 a, float4 b) {
    const float2 lo = __fmul2_rn(make_float2(a.x, a.y), make_float2(b.x, b.y));
    const float2 hi = __fmul2_rn(make_float2(a.z, a.w), make_float2(b.z, b.w));
    return make_float4(lo.x, lo.y, hi.x, hi.y);
}
__device__ __forceinline__ float4 rcp4(float4 a) {
    return make_float4(rcp_approx(a.x), rcp_approx(a.y), rcp_approx(a.z), rcp_approx(a.w));
}
__device__ __forceinline__ float min4(float4 a) { return fminf(fminf(a.x, a.y), fminf(a.z, a.w)); }
__device__ __forceinline__ float4 bf16x4_to_f32(uint2 u) {
    const float2 a = unpack_bf16x2(u.x), b = unpack_bf16x2(u.y);
    return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ uint2 f32_to_bf16x4(float4 x) {
    return make_uint2(pack_bf16x2(x.x, x.y), pack_bf16x2(x.z, x.w));
}
// 4 channels d..d+3 (d % 4 == 0) of row r of a K-major 128-byte swizzled tile
// with `acs` bytes per 64-channel atom column.
__device__ __forceinline__ void st4_sw128(uint8_t *tile, uint32_t acs, int r, int d, float4 x) {
    *reinterpret_cast<uint2 *>(tile + (uint32_t)(d >> 6) * acs + (uint32_t)r * 128u +
                               ((((uint32_t)(d & 63) >> 3) ^ ((uint32_t)r & 7u)) << 4) +
                               ((uint32_t)(d & 7) << 1)) = f32_to_bf16x4(x);
}

__global__ void __launch_bounds__(kda::PREP_THREADS, 2) kda_prep_kernel(const KdaPrepParams p) {
    using namespace kda;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    KCtl *ctl = reinterpret_cast<KCtl *>(smem_raw);
    uint8_t *tiles = smem_raw + align1k((uint32_t)sizeof(KCtl) + (smem_u32(smem_raw) & 1023u)) -
                     (smem_u32(smem_raw) & 1023u);
    const uint32_t tb = smem_u32(tiles);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int sc = warp;          // this warp's sub-chunk: tokens 16 sc .. 16 sc + 15
    const int d0 = 4 * lane;      // this lane's key channels d0 .. d0 + 3
    const int64_t items = p.B * p.H * (int64_t)p.nchunks;
    float *AF = reinterpret_cast<float *>(tiles + P_AF);
    float *TMP = reinterpret_cast<float *>(tiles + P_TMP);

    if (tid == 0) {
        mbar_init(&ctl->mma, 1);
        mbar_init(&ctl->mma_u, 1);
        mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&ctl->tmem_base, 256);
        tc_fence_before_sync();
    }
    __syncthreads();
    tc_fence_after_sync();
    // the main pass, launched as a programmatic dependent, may be scheduled now: it
    // waits for this grid's completion before it reads anything written here
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const uint32_t tmem = ctl->tmem_base;
    const uint32_t tw = tmem + ((uint32_t)(32 * warp) << 16);   // this warp's TMEM lanes
    constexpr uint32_t ID_U = idesc_bf16(64, 128, false, true);

    int it = 0;   // items processed (one MMA commit each): the mbarrier phase
    for (int64_t w = blockIdx.x; w < items; w += gridDim.x) {
        const int64_t bh = w / p.nchunks;
        const int c = (int)(w % p.nchunks);
        const int64_t b = bh / p.H, h = bh % p.H;
        const int64_t t0 = (int64_t)c * C;   // position in the sequence
        const SeqSpan sq = seq_span(p.cu_seqlens, b, p.T, p.max_seqlen, false);
        if (tid == 0) ctl->stop = ctl->abort;   // one thread decides, everyone reads after the barrier
        bar_named(1, 128);
        if (ctl->stop) break;
        if (t0 >= sq.len) continue;   // past this packed sequence's last chunk (uniform over the CTA)
        // rows of qp, kc this item writes: the sequence's tokens, plus (packed)
        // the padding rows of its tail chunk, as zeros
        const int64_t wlen = p.cu_seqlens ? p.Ls : sq.len;

        // (1) loads: alpha (1 past T), q and k (0 past T) of this thread's 16 tokens x 4 channels
        float4 g[16];
        uint2 qr[16], kr[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int64_t t = t0 + 16 * sc + j;
            const bool valid = t < sq.len;
            const int64_t row = ((sq.row0 + (valid ? t : 0)) * p.H + h) * DK + d0;
            g[j] = valid ? __ldg(reinterpret_cast<const float4 *>(p.alpha + row)) : make_float4(1.f, 1.f, 1.f, 1.f);
            qr[j] = valid ? __ldg(reinterpret_cast<const uint2 *>(p.q + row)) : make_uint2(0u, 0u);
            kr[j] = valid ? __ldg(reinterpret_cast<const uint2 *>(p.k + row)) : make_uint2(0u, 0u);
        }
        if (tid < 64) {
            const int64_t t = t0 + tid;
            ctl->beta[tid] = t < sq.len ? p.beta[(sq.row0 + t) * p.H + h] : 0.f;
        }
        {   // bring the next item's rows into L2 while this one is worked on: thread
            // i < 64 the alpha row (512 B) of token i, thread 64 + i its q and k rows
            const int64_t wn = w + gridDim.x;
            if (wn < items) {
                const int64_t bhn = wn / p.nchunks, bn = bhn / p.H, hn = bhn % p.H;
                const SeqSpan sn = seq_span(p.cu_seqlens, bn, p.T, p.max_seqlen, false);
                const int64_t tn = (int64_t)(wn % p.nchunks) * C + (tid & 63);
                if (tn < sn.len) {
                    const int64_t row = ((sn.row0 + tn) * p.H + hn) * DK;
                    if (tid < 64) {
                        bulk_prefetch_l2(p.alpha + row, DK * 4);
                    } else {
                        bulk_prefetch_l2(p.q + row, DK * 2);
                        bulk_prefetch_l2(p.k + row, DK * 2);
                    }
                }
            }
        }
        // G_j = Gamma_t / Gamma_middle, in place of alpha: 1 / prod_{j+1..7} alpha
        // for j <= 7, prod_{8..j} alpha for j >= 8
        float4 suf = make_float4(1.f, 1.f, 1.f, 1.f);
#pragma unroll
        for (int j = 7; j >= 0; --j) {
            const float4 a = g[j];
            g[j] = rcp4(suf);
            suf = mul4(suf, a);
        }
        float4 run = make_float4(1.f, 1.f, 1.f, 1.f);
#pragma unroll
        for (int j = 8; j < 16; ++j) {
            run = mul4(run, g[j]);
            g[j] = run;
        }
        // the smallest 8-token products (suf: tokens 0..7, run: 8..15) bound G and 1/G
        bool bad = !(fminf(min4(suf), min4(run)) >= kMinFactor);
        *reinterpret_cast<float4 *>(&ctl->D[sc][d0]) = suf;
        *reinterpret_cast<float4 *>(&ctl->U[sc][d0]) = run;
        bar_named(1, 128);

        // (2) per-channel factors from the sub-chunk products (unrolled selects:
        // no register array is indexed by the warp's sub-chunk)
        // gm = Gamma at this sub-chunk's middle; cm = Gamma_C / gm;
        // mk[a] = Gamma_{m_a} / gm for a > sc (the Kr_a scale of this sub-chunk's
        // keys; 1 for a = sc), each times 2^64; gc = Gamma_C
        const float4 up = make_float4(kUp, kUp, kUp, kUp);
        float4 gm = up, cm = up, acc = up, gc = make_float4(1.f, 1.f, 1.f, 1.f), mk[4];
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const float4 Ds = *reinterpret_cast<const float4 *>(&ctl->D[s][d0]);
            const float4 Us = *reinterpret_cast<const float4 *>(&ctl->U[s][d0]);
            const float4 Ls = mul4(Ds, Us);
            gc = mul4(gc, Ls);
            if (s < sc) gm = mul4(gm, Ls);
            if (s == sc) {
                gm = mul4(gm, Ds);
                cm = mul4(cm, Us);
                acc = cm;
            }
            if (s > sc) {
                cm = mul4(cm, Ls);
                mk[s] = mul4(acc, Ds);
                acc = mul4(acc, Ls);
            }
        }
        uint8_t *item = p.items + w * (int64_t)ITEM_BYTES;
        if (sc == 0) *reinterpret_cast<float4 *>(item + ITEM_GC + 4 * d0) = gc;

        // (3) scaled operand rows
        uint8_t *qs = tiles + P_QS;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int64_t t = t0 + 16 * sc + j;
            const float4 qf = bf16x4_to_f32(qr[j]), kf = bf16x4_to_f32(kr[j]);
            const float4 G = g[j], Hf = rcp4(G);
            const float4 down = make_float4(kDown, kDown, kDown, kDown);
            const float4 Gd = mul4(G, down), Hd = mul4(Hf, down);
            const float4 Gg = mul4(Gd, gm);   // Gamma_t
            st4_sw128(qs, QS_ACS, 32 * sc + j, d0, mul4(qf, G));
            st4_sw128(qs, QS_ACS, 32 * sc + 16 + j, d0, mul4(kf, G));
            st4_sw128(tiles + P_KR + kr_off(sc), kr_acs(sc), 16 * sc + j, d0, mul4(kf, Hf));
#pragma unroll
            for (int a = 0; a < 4; ++a)
                if (a > sc) st4_sw128(tiles + P_KR + kr_off(a), kr_acs(a), 16 * sc + j, d0, mul4(kf, mul4(Hd, mk[a])));
            st4_sw128(tiles + P_KP, 8192u, 16 * sc + j, d0, mul4(kf, Gg));   // 0 past T (k is)
            if (t < wlen) {
                const int64_t row = ((b * p.Ls + t) * p.H + h) * DK + d0;
                const bool in = t < sq.len;
                *reinterpret_cast<uint2 *>(p.qp + row) = in ? f32_to_bf16x4(mul4(qf, Gg)) : make_uint2(0u, 0u);
                *reinterpret_cast<uint2 *>(p.kc + row) =   // Gamma_C / Gamma_t
                    in ? f32_to_bf16x4(mul4(kf, mul4(Hd, cm))) : make_uint2(0u, 0u);
            }
        }
        if (__any_sync(0xffffffffu, bad) && lane == 0) raise_error(kErrRange);
        fence_proxy_async_smem();
        tc_fence_before_sync();
        bar_named(1, 128);

        // (4) four MMAs: rows of [Qs ; Ks] against Kr_a (N = 16 (a + 1) keys), into
        // TMEM columns 64a (columns past 16 (a + 1) are masked on readout)
        if (tid == 0) {
            tc_fence_after_sync();
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int kk = 0; kk < DK / 16; ++kk)
                    umma_bf16(tmem + 64u * a, desc_k(tb + P_QS, QS_ACS, kk),
                              desc_k(tb + P_KR + kr_off(a), kr_acs(a), kk), idesc_bf16(128, 16 * (a + 1), false, false),
                              kk > 0);
            umma_commit(&ctl->mma);
        }
        if (!mbar_wait(&ctl->mma, (uint32_t)it & 1u)) ctl->abort = 1;
        tc_fence_after_sync();

        // (5) lane l < 16: P row of token 16w + l; lane l >= 16: A row of token 16w + l - 16.
        // Both come from accumulator w; only columns < 16(w+1) can be unmasked.
        {
            const int t = 16 * warp + (lane & 15);
            float x0[32], x1[32];
            tmem_ld32(tw + 64u * warp, x0);
            if (warp >= 2) tmem_ld32(tw + 64u * warp + 32u, x1);
            tmem_wait_ld();
            if (warp < 2) {
#pragma unroll
                for (int i = 0; i < 32; ++i) x1[i] = 0.f;
            }
            if (lane < 16) {
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    x0[i] = i <= t ? x0[i] : 0.f;
                    x1[i] = 32 + i <= t ? x1[i] : 0.f;
                }
                uint8_t *dst = item + ITEM_P + (uint32_t)t * 128u;
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) {
                    const float *x = cc < 4 ? x0 + 8 * cc : x1 + 8 * (cc - 4);
                    uint4 u;
                    u.x = pack_bf16x2(x[0], x[1]);
                    u.y = pack_bf16x2(x[2], x[3]);
                    u.z = pack_bf16x2(x[4], x[5]);
                    u.w = pack_bf16x2(x[6], x[7]);
                    *reinterpret_cast<uint4 *>(dst + (uint32_t)(((cc ^ t) & 7) << 4)) = u;
                }
            } else {
                const float be = ctl->beta[t];
                float *arow = AF + t * gdn::AF_LD;
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    *reinterpret_cast<float4 *>(arow + i) =
                        make_float4(i < t ? be * x0[i] : 0.f, i + 1 < t ? be * x0[i + 1] : 0.f,
                                    i + 2 < t ? be * x0[i + 2] : 0.f, i + 3 < t ? be * x0[i + 3] : 0.f);
                    *reinterpret_cast<float4 *>(arow + 32 + i) =
                        make_float4(32 + i < t ? be * x1[i] : 0.f, 33 + i < t ? be * x1[i + 1] : 0.f,
                                    34 + i < t ? be * x1[i + 2] : 0.f, 35 + i < t ? be * x1[i + 3] : 0.f);
                }
            }
        }
        tc_fence_before_sync();
        bar_named(1, 128);
        gdn::invert_unit_lower64(AF, TMP, tid, lane, 1, 2);
        {   // T diag(beta) -> the item's image (128-byte swizzled [64][64] bf16), and the
            // same image over AF (once every thread has read its part of T) as the
            // A operand of U = T diag(beta) (K o Gamma)
            const int t = tid >> 1, hh = tid & 1;
            const float4 *Trow = reinterpret_cast<const float4 *>(AF + t * gdn::AF_LD + 32 * hh);
            const float4 *be4 = reinterpret_cast<const float4 *>(ctl->beta + 32 * hh);
            uint8_t *dst = item + ITEM_T;
            uint4 img[4];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                const float4 t0 = Trow[2 * cc], t1 = Trow[2 * cc + 1], b0 = be4[2 * cc], b1 = be4[2 * cc + 1];
                img[cc] = make_uint4(pack_bf16x2(t0.x * b0.x, t0.y * b0.y), pack_bf16x2(t0.z * b0.z, t0.w * b0.w),
                                     pack_bf16x2(t1.x * b1.x, t1.y * b1.y), pack_bf16x2(t1.z * b1.z, t1.w * b1.w));
                const int chunk = 4 * hh + cc;
                *reinterpret_cast<uint4 *>(dst + (uint32_t)t * 128u + (uint32_t)(((chunk ^ t) & 7) << 4)) = img[cc];
            }
            bar_named(1, 128);   // every read of T is done
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                const int chunk = 4 * hh + cc;
                *reinterpret_cast<uint4 *>(tiles + P_AF + (uint32_t)t * 128u + (uint32_t)(((chunk ^ t) & 7) << 4)) =
                    img[cc];
            }
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        bar_named(1, 128);
        if (tid == 0) {   // U: M=64 tokens, N=128 key channels, K=64 tokens
            tc_fence_after_sync();
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk)
                umma_bf16(tmem, desc_k(tb + P_AF, C * 128, kk), desc_mn128(tb + P_KP, 8192u, kk), ID_U, kk > 0);
            umma_commit(&ctl->mma_u);
        }
        if (!mbar_wait(&ctl->mma_u, (uint32_t)it & 1u)) ctl->abort = 1;
        ++it;
        tc_fence_after_sync();
        {   // -U -> the item: row tr = 16 warp + (lane & 15) of the M=64 accumulator,
            // key channels 64 hf .. 64 hf + 63 = block hf of the image
            const int tr = 16 * warp + (lane & 15), hf = lane >> 4;
            float x[64];
            tmem_ld16x2_32<64>(tw, *reinterpret_cast<float(*)[32]>(x));
            tmem_ld16x2_32<64>(tw + 32u, *reinterpret_cast<float(*)[32]>(x + 32));
            tmem_wait_ld();
            uint8_t *dst = item + ITEM_U + (uint32_t)hf * 8192u + (uint32_t)tr * 128u;
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
        bar_named(1, 128);   // AF aliases [Qs ; Ks], which the next item rewrites; TMEM too
    }
    // every MMA has finished before TMEM is released (a long wait even after a
    // timeout ended the loop)
    if (tid == 0) {
        umma_commit(&ctl->drain);
        (void)mbar_drain(&ctl->drain, 0u);
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

}  // namespace ck
}  // namespace la
