// chunk_tc.cuh — chunked prefill on the 5th-generation tensor cores (tcgen05,
// accumulators in TMEM, operands staged in shared memory by TMA).
//
// Work split: one CTA per (batch b, head h, 32-wide slab of value columns).
// The CTA walks the sequence in chunks of C = 64 tokens.  Inside a chunk every
// token-pair interaction is a dense bf16 x bf16 -> fp32 MMA; across chunks the
// dk x 32 state slab is carried in fp32 registers (thread d owns row d) and a
// bf16 copy of it is the MMA operand of the next chunk's inter-chunk read.
// "Parallel inside a chunk, linear accumulation across chunks" is the tiling of
// page "线性注意力与状态空间前沿论文" §1 (Lightning Attention-2); the gate
// products inside a chunk are kept as differences of cumulative log-gates
// (page "Linear / RNN 路线" §2.2: chunk-wise parallel GLA needs the gate
// cumulative product handled with care).
//
// Notation for one chunk (positions t, i in [0, 64), S0 = state entering it):
//   ELU+1 (page "Linear / RNN 路线" §2.1):
//     P = (phiQ phiK^T) o M,   O = phiQ S0 + P V,   den = phiQ z0 + P 1 + eps
//     S <- S0 + phiK^T V,  z <- z0 + phiK^T 1
//   GLA (§2.2): gamma_t = prod_{s<=t} g_s (per key dim, reference = chunk start)
//     Qt = Q o gamma,  Kt = K / gamma,  Kh = Kt o gamma_C
//     P = (Qt Kt^T) o M,  O = Qt S0 + P V,  S <- diag(gamma_C) S0 + Kh^T V
//   Gated delta rule (page "线性注意力与 SSM", GDN box): gamma_t = prod alpha,
//     Gamma_ti = gamma_t / gamma_i (computed as exp2 of log2 differences <= 0),
//     A = diag(beta) (K K^T o Gamma o strict-lower), T = (I + A)^-1,
//     U = T diag(beta) V,  W_k = T diag(beta gamma) K,   (state independent)
//     W = U - W_k S0,  O = diag(gamma) Q S0 + P W,  P = (Q K^T) o Gamma o M,
//     S <- gamma_C S0 + K^T diag(gamma_C / gamma) W.
//   This is the WY / UT form of the delta rule's intra-chunk dependence (named
//   on page "线性注意力速览" for DeltaNet and page "状态空间与线性注意力" for
//   KDA): unrolling S_t = alpha_t S_{t-1} + beta_t k_t (v_t - alpha_t S_{t-1}^T
//   k_t)^T inside a chunk gives S_t = gamma_t S0 + sum_{i<=t} (gamma_t/gamma_i)
//   k_i w_i^T with w_t = beta_t (v_t - gamma_t S0^T k_t) - beta_t sum_{i<t}
//   (gamma_t/gamma_i)(k_t.k_i) w_i, i.e. (I + A) W = diag(beta) V -
//   diag(beta gamma) K S0.
//
// Tail chunk: TMA zero-fills rows past T; padded rows get g = 1 (GLA),
// alpha = 1 and beta = 0 (GDN) and phi(k) = 0 (ELU), so they change nothing.
//
// Operand tiles in shared memory are "128-byte swizzled" rows of 64 bf16
// (see sw128_off); a [rows][64] atom column is both the K-major layout of a
// (rows x 64) operand and the MN-major layout of a (64 x rows) operand.
// V is loaded with the 64-byte swizzle (32 columns = 64 bytes per row).
//
// Every wait is bounded (mbar_wait); on a timeout the CTA records the error,
// stops issuing work, waits for its copies in flight and frees its TMEM.
#pragma once

#include <algorithm>
#include <string>

#include "device.cuh"
#include "recurrent.cuh"

namespace la {

bool make_map_4d(CUtensorMap *map, const void *base, CUtensorMapDataType dtype, int esize,
                 int64_t B, int64_t T, int64_t H, int64_t D, int box_d, int box_t,
                 CUtensorMapSwizzle swz);
cudaError_t allow_smem(const void *kernel, int bytes);

struct ChunkParams {
    int64_t B, T, H, dv;
    const void *q, *k, *v;
    const float *g, *beta, *S0, *z0;
    float *S_out, *z_out;
    void *o;
    float eps;
};

namespace ck {

constexpr int C = 64;         // chunk length (tokens)
constexpr int DK = 128;       // key dim handled by these kernels
constexpr int DVT = 32;       // value columns per CTA
constexpr int NT = 128;       // threads per CTA
constexpr int KA = DK / 64;   // 64-wide atom columns along dk
constexpr uint32_t TM_COLS = 256;

// --- descriptors --------------------------------------------------------------
// A descriptor is built once per operand (k-step 0) and advanced per k-step by
// adding the byte offset >> 4 to its start-address field (the tiles live below
// 256 KB, so the 14-bit field never carries).
__device__ __forceinline__ uint64_t dk0(uint32_t base) { return smem_desc(base, 16u, 1024u, kSwizzle128); }
__device__ __forceinline__ uint64_t dmn128_0(uint32_t base, uint32_t lbo) {
    return smem_desc(base, lbo, 1024u, kSwizzle128);
}
__device__ __forceinline__ uint64_t dmn64_0(uint32_t base) { return smem_desc(base, 4096u, 512u, kSwizzle64); }
// K-major, 128-byte swizzle: rows of 64 elements, `acs` bytes between atom
// columns, k-step kk covers K elements [16kk, 16kk+16).
__device__ __forceinline__ uint64_t kstep_k(uint64_t d0, uint32_t acs, int kk) {
    return d0 + (uint64_t)(((uint32_t)(kk >> 2) * acs + (uint32_t)(kk & 3) * 32u) >> 4);
}
// MN-major, 128-byte swizzle: K runs down 128-byte rows, 16 rows per k-step.
__device__ __forceinline__ uint64_t kstep_mn128(uint64_t d0, int kk) { return d0 + (uint64_t)(kk * 128); }
// MN-major, 64-byte swizzle (32 MN elements per 64-byte row), 16 rows per k-step.
__device__ __forceinline__ uint64_t kstep_mn64(uint64_t d0, int kk) { return d0 + (uint64_t)(kk * 64); }

__device__ __forceinline__ uint64_t desc_k(uint32_t base, uint32_t acs, int kk) {
    return kstep_k(dk0(base), acs, kk);
}
__device__ __forceinline__ uint64_t desc_mn128(uint32_t base, uint32_t lbo, int kk) {
    return kstep_mn128(dmn128_0(base, lbo), kk);
}
__device__ __forceinline__ uint64_t desc_mn64(uint32_t base, int kk) { return kstep_mn64(dmn64_0(base), kk); }

__device__ __forceinline__ void store_row_bf16(uint8_t *tile, int r, const float *x64) {
    // row r of a [rows][64] SW128 tile from 64 floats (16-byte stores)
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        uint4 u;
        u.x = pack_bf16x2(x64[8 * c + 0], x64[8 * c + 1]);
        u.y = pack_bf16x2(x64[8 * c + 2], x64[8 * c + 3]);
        u.z = pack_bf16x2(x64[8 * c + 4], x64[8 * c + 5]);
        u.w = pack_bf16x2(x64[8 * c + 6], x64[8 * c + 7]);
        *reinterpret_cast<uint4 *>(tile + r * 128 + (((c ^ r) & 7) << 4)) = u;
    }
}

__device__ __forceinline__ __nv_bfloat16 *elem(uint8_t *tile, int r, int col) {
    return reinterpret_cast<__nv_bfloat16 *>(tile + sw128_off((uint32_t)r, (uint32_t)col));
}

// Output rows of an M=64 accumulator: warp w, lanes 0..15 hold rows 16w+lane.
__device__ __forceinline__ void store_out_row(void *o, const ChunkParams &p, int64_t b, int64_t h,
                                              int64_t t, int dvt, const float *x) {
    __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(o) +
                         ((b * p.T + t) * p.H + h) * p.dv + (int64_t)dvt * DVT;
#pragma unroll
    for (int c = 0; c < DVT / 8; ++c) {
        uint4 u;
        u.x = pack_bf16x2(x[8 * c + 0], x[8 * c + 1]);
        u.y = pack_bf16x2(x[8 * c + 2], x[8 * c + 3]);
        u.z = pack_bf16x2(x[8 * c + 4], x[8 * c + 5]);
        u.w = pack_bf16x2(x[8 * c + 6], x[8 * c + 7]);
        reinterpret_cast<uint4 *>(dst)[c] = u;
    }
}

struct Maps {
    CUtensorMap q, k, v, g;
};

// Shared bookkeeping at the start of dynamic shared memory.
struct Ctl {
    uint64_t tma_bar[2];
    uint64_t mma_bar;
    uint32_t tmem_base;
    int abort;
    float gC[DK];       // GLA: gamma at chunk end per key dim; ELU: z0 staging
    float b2[C];        // GDN: log2 cumulative alpha
    float alpha[C], beta[C];
};

__device__ __forceinline__ uint32_t align1k(uint32_t x) { return (x + 1023u) & ~1023u; }

// Bytes of a [rows] x DK tile as KA atom columns.
constexpr uint32_t tile_bytes(int rows) { return (uint32_t)rows * 128u * KA; }

// ---------------------------------------------------------------------------
// Common prologue / epilogue helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ void issue_loads(const Maps &m, Ctl *ctl, int stage, uint8_t *qdst,
                                            uint8_t *kdst, uint32_t q_acs, uint32_t k_acs,
                                            uint8_t *vdst, uint8_t *gdst, int64_t b, int64_t h,
                                            int t0, int dvt, bool has_g) {
    const uint32_t bytes = 2u * KA * C * 128u + C * DVT * 2u + (has_g ? C * DK * 4u : 0u);
    mbar_arrive_expect_tx(&ctl->tma_bar[stage], bytes);
#pragma unroll
    for (int a = 0; a < KA; ++a) {
        tma_load_4d(qdst + a * q_acs, &m.q, &ctl->tma_bar[stage], 64 * a, (int)h, t0, (int)b);
        tma_load_4d(kdst + a * k_acs, &m.k, &ctl->tma_bar[stage], 64 * a, (int)h, t0, (int)b);
    }
    tma_load_4d(vdst, &m.v, &ctl->tma_bar[stage], dvt * DVT, (int)h, t0, (int)b);
    if (has_g) tma_load_4d(gdst, &m.g, &ctl->tma_bar[stage], 0, (int)h, t0, (int)b);
}

// ---------------------------------------------------------------------------
// GLA and ELU+1 share one kernel body (RULE selects the feature map / gates).
// ---------------------------------------------------------------------------
template <int RULE>
struct LayoutGE {
    // staged: Q, K (KA x 64 rows), V (64 x 64 B), G (GLA: 64 x DK fp32)
    static constexpr uint32_t Q = 0;
    static constexpr uint32_t K = Q + 2 * tile_bytes(C);
    static constexpr uint32_t V = K + 2 * tile_bytes(C);
    static constexpr uint32_t G = V + 2 * 4096;
    static constexpr uint32_t GSZ = (RULE == kRuleGLA) ? C * DK * 4 : 0;
    // Kx: [K~ or phiK (64 rows); S^T (32 rows); ELU: z^T + 7 zero rows]
    static constexpr int KX_ROWS = (RULE == kRuleELU) ? 104 : 96;
    static constexpr uint32_t KX = G + 2 * GSZ;
    static constexpr uint32_t KX_ACS = KX_ROWS * 128;
    static constexpr uint32_t P = KX + tile_bytes(KX_ROWS);
    static constexpr uint32_t END = P + C * 128;
    static constexpr int N1 = KX_ROWS;   // N of the score/inter MMA
};

template <int RULE>
__global__ void __launch_bounds__(NT, 1)
chunk_ge_kernel(const __grid_constant__ Maps maps, const ChunkParams p) {
    using L = LayoutGE<RULE>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // control block first, tiles from the next 1 KB boundary
    Ctl *ctl = reinterpret_cast<Ctl *>(smem_raw);
    uint8_t *tiles = smem_raw + align1k((uint32_t)sizeof(Ctl) + (smem_u32(smem_raw) & 1023u)) -
                     (smem_u32(smem_raw) & 1023u);
    const uint32_t tiles_s = smem_u32(tiles);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nslab = (int)(p.dv / DVT);
    const int dvt = (int)(blockIdx.x % nslab);
    const int64_t bh = blockIdx.x / nslab;
    const int64_t b = bh / p.H, h = bh % p.H;
    const int nchunks = (int)((p.T + C - 1) / C);

    if (tid == 0) {
        mbar_init(&ctl->tma_bar[0], 1);
        mbar_init(&ctl->tma_bar[1], 1);
        mbar_init(&ctl->mma_bar, 1);
        ctl->abort = 0;
        fence_barrier_init();
        tma_prefetch_desc(&maps.q);
        tma_prefetch_desc(&maps.k);
        tma_prefetch_desc(&maps.v);
        if (RULE == kRuleGLA) tma_prefetch_desc(&maps.g);
    }
    if (warp == 0) {
        tmem_alloc(&ctl->tmem_base, TM_COLS);
        tc_fence_before_sync();
    }
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = ctl->tmem_base;
    const uint32_t tw = tmem + ((uint32_t)(32 * warp) << 16);   // this warp's lane quadrant

    // State slab: thread d owns row d (DVT fp32 values).
    float S[DVT];
    {
        const float *src = p.S0 ? p.S0 + ((bh * DK + tid) * p.dv + dvt * DVT) : nullptr;
#pragma unroll
        for (int j = 0; j < DVT; j += 4) {
            float4 x = src ? *reinterpret_cast<const float4 *>(src + j) : make_float4(0, 0, 0, 0);
            S[j] = x.x; S[j + 1] = x.y; S[j + 2] = x.z; S[j + 3] = x.w;
        }
    }
    float z = 0.f;  // ELU: normaliser z_d for d = tid
    if (RULE == kRuleELU && p.z0) z = p.z0[bh * DK + tid];

    uint8_t *Kx = tiles + L::KX;
    uint8_t *Ps = tiles + L::P;
    // bf16 copy of S^T (and z^T for ELU) into Kx rows 64.. ; zero rows 97..103
    auto write_state_copy = [&]() {
        const int a = tid >> 6, d = tid & 63;
#pragma unroll
        for (int j = 0; j < DVT; ++j) *elem(Kx + a * L::KX_ACS, 64 + j, d) = __float2bfloat16_rn(S[j]);
        if (RULE == kRuleELU) *elem(Kx + a * L::KX_ACS, 96, d) = __float2bfloat16_rn(z);
    };
    if (RULE == kRuleELU) {
        const int a = tid >> 6, d = tid & 63;
#pragma unroll
        for (int r = 97; r < 104; ++r) *elem(Kx + a * L::KX_ACS, r, d) = __float2bfloat16_rn(0.f);
    }
    write_state_copy();

    if (tid == 0 && nchunks > 0)
        issue_loads(maps, ctl, 0, tiles + L::Q, tiles + L::K, C * 128, C * 128, tiles + L::V,
                    tiles + L::G, b, h, 0, dvt, RULE == kRuleGLA);

    uint32_t mma_phase = 0;
    constexpr uint32_t ID_SCORE = idesc_bf16(64, L::N1, false, false);
    constexpr uint32_t ID_UPD = idesc_bf16(128, DVT, true, true);
    constexpr uint32_t ID_PV = idesc_bf16(64, DVT, false, true);
    constexpr uint32_t COL_P = 0, COL_O = 64, COL_D = 128;  // TMEM columns

    for (int c = 0; c < nchunks; ++c) {
        const int st = c & 1;
        const int t0 = c * C;
        const int nvalid = (int)min((int64_t)C, p.T - t0);
        uint8_t *Qs = tiles + L::Q + st * tile_bytes(C);
        uint8_t *Ks = tiles + L::K + st * tile_bytes(C);
        uint8_t *Vs = tiles + L::V + st * 4096;
        float *Gs = reinterpret_cast<float *>(tiles + L::G + st * L::GSZ);

        // prefetch the next chunk into the other stage (its previous user, chunk c-1, is done)
        if (tid == 0 && c + 1 < nchunks && !ctl->abort) {
            const int s2 = st ^ 1;
            issue_loads(maps, ctl, s2, tiles + L::Q + s2 * tile_bytes(C),
                        tiles + L::K + s2 * tile_bytes(C), C * 128, C * 128,
                        tiles + L::V + s2 * 4096, tiles + L::G + s2 * L::GSZ, b, h, t0 + C, dvt,
                        RULE == kRuleGLA);
        }
        if (!mbar_wait(&ctl->tma_bar[st], (uint32_t)(c >> 1) & 1u)) ctl->abort = 1;

        // ---- feature map / gates on CUDA cores: thread tid owns key dim d = tid
        {
            const int d = tid, a = d >> 6, dc = d & 63;
            uint8_t *qa = Qs + a * (C * 128), *ka = Ks + a * (C * 128), *kxa = Kx + a * L::KX_ACS;
            if constexpr (RULE == kRuleGLA) {
                float gam = 1.f;
                for (int t = 0; t < C; ++t) {
                    const float gt = (t < nvalid) ? Gs[t * DK + d] : 1.f;
                    gam *= gt;
                    Gs[t * DK + d] = gam;
                }
                const float gC = gam;
                if (!(gC >= 1e-30f)) raise_error(kErrRange);
                for (int t = 0; t < C; ++t) {
                    const float gm = Gs[t * DK + d];
                    const float inv = 1.f / gm;
                    __nv_bfloat16 *qe = elem(qa, t, dc), *ke = elem(ka, t, dc);
                    const float qv = __bfloat162float(*qe), kv = __bfloat162float(*ke);
                    *qe = __float2bfloat16_rn(qv * gm);                 // Qt (in place)
                    *elem(kxa, t, dc) = __float2bfloat16_rn(kv * inv);   // Kt
                    *ke = __float2bfloat16_rn(kv * (inv * gC));          // Kh (in place)
                }
                ctl->gC[d] = gC;
            } else {  // ELU+1
                float zs = 0.f;
                for (int t = 0; t < C; ++t) {
                    __nv_bfloat16 *qe = elem(qa, t, dc);
                    const float pq = elu_feature(__bfloat162float(*qe));
                    const float pk = (t < nvalid) ? elu_feature(__bfloat162float(*elem(ka, t, dc))) : 0.f;
                    *qe = __float2bfloat16_rn(pq);
                    const __nv_bfloat16 pkb = __float2bfloat16_rn(pk);
                    *elem(kxa, t, dc) = pkb;
                    zs += pk;
                }
                ctl->gC[d] = zs;   // chunk sum of phi(k) for dim d
            }
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncthreads();
        if (ctl->abort) break;

        // ---- MMA 1: [P | O_inter (| den_inter)] = Q' [K' ; S^T (; z^T)]^T ; MMA 2: dS = K''^T V
        if (tid == 0) {
            tc_fence_after_sync();
            const uint32_t qb = smem_u32(Qs), kxb = smem_u32(Kx);
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk)
                umma_bf16(tmem + COL_P, desc_k(qb, C * 128, kk), desc_k(kxb, L::KX_ACS, kk), ID_SCORE,
                          kk > 0);
            // update operand: GLA uses Kh (in place in Ks); ELU uses phiK (Kx rows 0..63)
            const uint32_t ub = (RULE == kRuleGLA) ? smem_u32(Ks) : kxb;
            const uint32_t ulbo = (RULE == kRuleGLA) ? (uint32_t)(C * 128) : L::KX_ACS;
            const uint32_t vb = smem_u32(Vs);
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk)
                umma_bf16(tmem + COL_D, desc_mn128(ub, ulbo, kk), desc_mn64(vb, kk), ID_UPD, kk > 0);
            umma_commit(&ctl->mma_bar);
        }
        if (!mbar_wait(&ctl->mma_bar, mma_phase)) ctl->abort = 1;
        mma_phase ^= 1u;
        tc_fence_after_sync();

        // ---- P (rows 16w+lane for lane < 16), masked -> bf16; den (ELU); state update
        float den = 0.f;
        {
            float x[64];
            tmem_ld32(tw + COL_P, *reinterpret_cast<float(*)[32]>(x));
            tmem_ld32(tw + COL_P + 32, *reinterpret_cast<float(*)[32]>(x + 32));
            float dI[16];
            if (RULE == kRuleELU) tmem_ld16(tw + 96, dI);   // col 96 = phiQ z0
            float dS[DVT];
            tmem_ld32(tw + COL_D, *reinterpret_cast<float(*)[32]>(dS));
            tmem_wait_ld();
            const int t = 16 * warp + lane;
            if (lane < 16) {
                float rs = 0.f;
#pragma unroll
                for (int i = 0; i < 64; ++i) {
                    x[i] = (i <= t) ? x[i] : 0.f;
                    rs += x[i];
                }
                store_row_bf16(Ps, t, x);
                if (RULE == kRuleELU) den = dI[0] + rs + p.eps;
            }
            // S <- diag(gamma_C) S + dS (GLA) / S + dS (ELU); thread tid owns row tid
            const float gC = ctl->gC[tid];
            if (RULE == kRuleGLA) {
#pragma unroll
                for (int j = 0; j < DVT; ++j) S[j] = fmaf(gC, S[j], dS[j]);
            } else {
#pragma unroll
                for (int j = 0; j < DVT; ++j) S[j] += dS[j];
                z += gC;
            }
            write_state_copy();
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncthreads();

        // ---- MMA 3: O += P V
        if (tid == 0) {
            tc_fence_after_sync();
            const uint32_t pb = smem_u32(Ps), vb = smem_u32(Vs);
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk)
                umma_bf16(tmem + COL_O, desc_k(pb, C * 128, kk), desc_mn64(vb, kk), ID_PV, 1u);
            umma_commit(&ctl->mma_bar);
        }
        if (!mbar_wait(&ctl->mma_bar, mma_phase)) ctl->abort = 1;
        mma_phase ^= 1u;
        tc_fence_after_sync();
        {
            float x[DVT];
            tmem_ld32(tw + COL_O, x);
            tmem_wait_ld();
            const int t = 16 * warp + lane;
            if (lane < 16 && t < nvalid) {
                if (RULE == kRuleELU) {
                    const float inv = 1.f / den;
#pragma unroll
                    for (int j = 0; j < DVT; ++j) x[j] *= inv;
                }
                store_out_row(p.o, p, b, h, t0 + t, dvt, x);
            }
        }
        tc_fence_before_sync();
        __syncthreads();
        if (ctl->abort) break;
    }

    if (ctl->abort) {
        // let any copy still in flight land before the shared memory is released
        if (tid == 0)
            for (int s = 0; s < 2; ++s) (void)mbar_try_wait(&ctl->tma_bar[s], 0);
    } else {
        if (p.S_out) {
            float *dst = p.S_out + ((bh * DK + tid) * p.dv + dvt * DVT);
#pragma unroll
            for (int j = 0; j < DVT; j += 4)
                *reinterpret_cast<float4 *>(dst + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
        }
        if (RULE == kRuleELU && p.z_out && dvt == 0) p.z_out[bh * DK + tid] = z;
    }
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, TM_COLS);
}

}  // namespace ck
}  // namespace la

#include "chunk_gdn.cuh"

namespace la {

// Host launcher.  Returns an la_status value (0 = ok).
// Device workspace the chunked path needs: the gated delta rule keeps the
// per-chunk T diag(beta) | T diag(beta gamma) operand images (16 KB per
// (batch, head, chunk)); the other rules need none.
inline size_t chunk_workspace_bytes(int rule, int64_t B, int64_t T, int64_t H) {
    if (rule != kRuleGDN || T <= 0) return 0;
    return (size_t)(B * H * ((T + ck::C - 1) / ck::C)) * ck::gdn::TT_BYTES;
}

inline int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        n = 148;
    return n;
}

inline int launch_chunk_tc(int rule, const ChunkParams &p, void *ws, size_t ws_bytes, cudaStream_t st,
                           std::string *err) {
    using namespace ck;
    if (p.dv % DVT != 0) {
        *err = "chunk kernel needs dv % 32 == 0";
        return 2;
    }
    Maps m;
    memset(&m, 0, sizeof(m));
    bool okm = make_map_4d(&m.q, p.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.B, p.T, p.H, DK, 64, C,
                           CU_TENSOR_MAP_SWIZZLE_128B) &&
               make_map_4d(&m.k, p.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.B, p.T, p.H, DK, 64, C,
                           CU_TENSOR_MAP_SWIZZLE_128B) &&
               make_map_4d(&m.v, p.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.B, p.T, p.H, p.dv, DVT, C,
                           CU_TENSOR_MAP_SWIZZLE_64B);
    if (okm && rule == kRuleGLA)
        okm = make_map_4d(&m.g, p.g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, p.B, p.T, p.H, DK, DK, C,
                          CU_TENSOR_MAP_SWIZZLE_NONE);
    if (!okm) {
        *err = "cuTensorMapEncodeTiled failed (driver entry point missing or bad layout)";
        return 4;
    }
    const unsigned grid = (unsigned)(p.B * p.H * (p.dv / DVT));
    const int ctl = (int)((sizeof(Ctl) + 1023) / 1024 * 1024) + 1024;
    cudaError_t e;
    if (rule == kRuleGDN) {
        const size_t need = chunk_workspace_bytes(rule, p.B, p.T, p.H);
        if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 15u)) {
            *err = "the gated delta rule needs a 16-byte aligned workspace of la_fwd_workspace_size() bytes";
            return 8;
        }
        GdnPrepParams pp{};
        pp.B = p.B; pp.T = p.T; pp.H = p.H;
        pp.nchunks = (int)((p.T + C - 1) / C);
        pp.alpha = p.g; pp.beta = p.beta;
        pp.ws = static_cast<uint8_t *>(ws);
        const int64_t items = p.B * p.H * (int64_t)pp.nchunks;
        const int psmem = (int)((sizeof(gdn::PCtl) + 1023) / 1024 * 1024) + 1024 + (int)gdn::P_END;
        const unsigned pgrid = (unsigned)std::min<int64_t>(items, (int64_t)sm_count() * 4);
        e = allow_smem((const void *)gdn_prep_kernel, psmem);
        if (e == cudaSuccess) gdn_prep_kernel<<<pgrid, gdn::PREP_THREADS, psmem, st>>>(m.k, pp);
        const int smem = (int)((sizeof(gdn::GCtl) + 1023) / 1024 * 1024) + 1024 + (int)gdn::TEND;
        if (e == cudaSuccess) e = allow_smem((const void *)chunk_gdn_kernel, smem);
        if (e == cudaSuccess)
            chunk_gdn_kernel<<<grid, gdn::NTHREADS, smem, st>>>(m, p, static_cast<const uint8_t *>(ws));
    } else if (rule == kRuleGLA) {
        const int smem = ctl + (int)LayoutGE<kRuleGLA>::END;
        e = allow_smem((const void *)chunk_ge_kernel<kRuleGLA>, smem);
        if (e == cudaSuccess) chunk_ge_kernel<kRuleGLA><<<grid, NT, smem, st>>>(m, p);
    } else {
        const int smem = ctl + (int)LayoutGE<kRuleELU>::END;
        e = allow_smem((const void *)chunk_ge_kernel<kRuleELU>, smem);
        if (e == cudaSuccess) chunk_ge_kernel<kRuleELU><<<grid, NT, smem, st>>>(m, p);
    }
    if (e != cudaSuccess) {
        *err = std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e);
        return 4;
    }
    return 0;
}

}  // namespace la
