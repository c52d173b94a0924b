// chunk_agg.cuh — sequence-parallel prefill of normalized ELU+1 and GLA, first
// pass.
//
// Over a range of tokens both recurrences are affine in the state that enters
// the range, with a diagonal (ELU+1: identity) linear part:
//   ELU+1 (page "Linear / RNN 路线", §2.1): S_t = S_{t-1} + phi(k_t) v_t^T,
//     z_t = z_{t-1} + phi(k_t), so S_end = S_in + dS with dS = sum_t phi(k_t)
//     v_t^T and dz = sum_t phi(k_t);
//   GLA (§2.2): S_t = diag(g_t) S_{t-1} + k_t v_t^T, so S_end = diag(D) S_in + dS
//     with D = prod_t g_t and dS = sum_t diag(prod_{s>t} g_s) k_t v_t^T (products
//     over the range's tokens, per key dim).
// A sequence cut into segments can then be processed by independent CTAs once
// each segment j knows its entering state, S0 folded through the ranges of the
// segments < j in order.  This kernel computes the range summaries: for every
// (batch, head) and every segment but the last, split into `nparts` chunk
// ranges handled by separate CTAs, dS (dk x dv) and dz (ELU+1) or D (GLA).
//
// 9 warps per CTA:
//   warps 0-7  ELU+1: phi(K) in place (zero past T) and the running sums of
//              phi(k) per key dim.  GLA: the range is walked from its last chunk
//              back, keeping R = the product of the gates of the chunks already
//              walked; each key row is scaled in place by R times the product of
//              the later gates inside its chunk (every factor <= 1, so nothing
//              overflows), and D = R at the end;
//   warp 8     TMA loads of k, v (and g) into a ring of stages and, lane 0, the
//              MMAs dS += K'^T V, accumulated in TMEM over the whole range.
// Afterwards warps 0-3 copy the accumulator (one key-dim row per thread) out.
#pragma once

#include "device.cuh"

namespace la {

struct AggParams {
    int64_t B, T, H, dv;
    float *agg;     // [B*H][nseg-1][nparts] blocks of DK*dv (dS, row-major) + DK (dz or D) floats
    int nseg, nparts, seg_chunks;
    uint32_t *seq_flags = nullptr;   // GLA: see ChunkParams
    uint32_t call_id = 0;
};

namespace ck {

template <int RULE, int DV>
struct AG {
    static constexpr bool kGLA = (RULE == kRuleGLA);
    static constexpr int NSTG = kGLA ? 3 : 4;
    static constexpr uint32_t K_BYTES = C * 128 * KA;   // K', [atom col][64 rows], 128-byte swizzle
    static constexpr uint32_t V_BYTES = C * DV * 2;     // DV/32 slabs of [64][32], 64-byte swizzle
    static constexpr uint32_t G_BYTES = kGLA ? C * DK * 4 : 0;   // GLA gates, fp32 [64][128]
    static constexpr uint32_t STG_BYTES = K_BYTES + V_BYTES + G_BYTES;
    static constexpr uint32_t END = NSTG * STG_BYTES;
    static constexpr uint32_t TMEM_COLS = DV;           // 32, 64 or 128
    static_assert(END + 3072 <= 232448, "chunk_agg_kernel tiles exceed shared memory");
};

struct AGCtl {
    uint64_t full[4], pfull[4], mdone[4], done;
    uint32_t tmem_base;
    int abort, stop[2];
    alignas(16) float2 tot[4][64];
};

template <int RULE, int DV>
__global__ void __launch_bounds__(288, 1)
chunk_agg_kernel(const __grid_constant__ Maps maps, const AggParams p) {
    using L = AG<RULE, DV>;
    constexpr int NSTG = L::NSTG;
    constexpr bool kGLA = L::kGLA;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    AGCtl *ctl = reinterpret_cast<AGCtl *>(smem_raw);
    uint8_t *tiles = smem_raw + align1k((uint32_t)sizeof(AGCtl) + (smem_u32(smem_raw) & 1023u)) -
                     (smem_u32(smem_raw) & 1023u);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int part = (int)(blockIdx.x % p.nparts);
    const int rest = (int)(blockIdx.x / p.nparts);
    const int seg = rest % (p.nseg - 1);
    const int64_t bh = rest / (p.nseg - 1);
    const int64_t b = bh / p.H, h = bh % p.H;
    const int cseg = seg * p.seg_chunks;   // segments before the last are full
    const int cbeg = cseg + (int)((int64_t)p.seg_chunks * part / p.nparts);
    const int cend = cseg + (int)((int64_t)p.seg_chunks * (part + 1) / p.nparts);
    const int n = cend - cbeg;
    float *out = p.agg + ((bh * (p.nseg - 1) + seg) * p.nparts + part) * (int64_t)(DK * DV + DK);

    auto stg = [&](int c) { return tiles + (uint32_t)(c % NSTG) * L::STG_BYTES; };

    if (tid == 0) {
        for (int s = 0; s < NSTG; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->pfull[s], 8);
            mbar_init(&ctl->mdone[s], 1);
        }
        mbar_init(&ctl->done, 1);
        ctl->abort = 0;
        fence_barrier_init();
        tma_prefetch_desc(&maps.k);
        tma_prefetch_desc(&maps.v);
        if (kGLA) tma_prefetch_desc(&maps.g);
    }
    if (warp == 0) {
        tmem_alloc(&ctl->tmem_base, L::TMEM_COLS);
        tc_fence_before_sync();
    }
    __syncthreads();
    tc_fence_after_sync();
    // the main pass, launched as a programmatic dependent, may be scheduled now: its
    // CTAs wait for this grid's completion before they read the summaries or flags
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const uint32_t tmem = ctl->tmem_base;

    if (warp < 8) {
        // K' in place; thread (pr, qt) owns key dims 2pr, 2pr+1 of tokens
        // 16qt..16qt+15 (a warp covers a full 128-byte row per access)
        const bool leader = (tid == 0);
        const int pr = tid & 63, qt = tid >> 6;
        const int a = pr >> 5;
        const uint32_t cpos = (uint32_t)((pr & 31) >> 2), cin = (uint32_t)(pr & 3) << 2;
        // ELU+1: running sum of phi(k); GLA: R, the gate product of the chunks walked
        float2 zacc = kGLA ? make_float2(1.f, 1.f) : make_float2(0.f, 0.f);
        for (int c = 0; c < n; ++c) {
            const int s = c % NSTG;
            const int ci = kGLA ? cend - 1 - c : cbeg + c;   // the chunk of iteration c
            const int nvalid = (int)min((int64_t)C, p.T - (int64_t)ci * C);
            // (the flag alternates between two words: the leader's write for the
            // next chunk cannot reach a thread still reading this one's)
            if (leader) ctl->stop[c & 1] = ctl->abort;
            bar_named(1, 256);
            if (ctl->stop[c & 1]) break;
            if (!mbar_wait(&ctl->full[s], (uint32_t)(c / NSTG) & 1u)) ctl->abort = 1;
            uint8_t *ka = stg(c) + a * (C * 128);
            auto off = [&](int i) {
                const uint32_t t = (uint32_t)(16 * qt + i);
                return t * 128u + (((cpos ^ t) & 7u) << 4) + cin;
            };
            uint32_t kv[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) kv[i] = *reinterpret_cast<const uint32_t *>(ka + off(i));
            if constexpr (kGLA) {
                // sf[i] = product of the gates of this thread's tokens after 16qt+i
                // (1 past T), then the product over its 16 tokens to share
                const uint8_t *G = stg(c) + L::K_BYTES + L::V_BYTES;   // fp32 [64][128]
                float2 sf[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int t = 16 * qt + i;
                    sf[i] = t < nvalid ? *reinterpret_cast<const float2 *>(G + t * 512 + pr * 8)
                                       : make_float2(1.f, 1.f);
                }
                float2 run = make_float2(1.f, 1.f);
#pragma unroll
                for (int i = 15; i >= 0; --i) {
                    const float2 gi = sf[i];
                    sf[i] = run;
                    run = __fmul2_rn(run, gi);
                }
                ctl->tot[qt][pr] = run;
                bar_named(1, 256);
                // the gates of the later token quarters of this chunk, and R
                float2 post = zacc;
                for (int q2 = 3; q2 > qt; --q2) post = __fmul2_rn(post, ctl->tot[q2][pr]);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float2 kf = __fmul2_rn(unpack_bf16x2(kv[i]), __fmul2_rn(sf[i], post));
                    if (16 * qt + i >= nvalid) kf = make_float2(0.f, 0.f);
                    *reinterpret_cast<uint32_t *>(ka + off(i)) = pack_bf16x2(kf.x, kf.y);
                }
                const float2 gc = __fmul2_rn(__fmul2_rn(ctl->tot[0][pr], ctl->tot[1][pr]),
                                             __fmul2_rn(ctl->tot[2][pr], ctl->tot[3][pr]));
                zacc = __fmul2_rn(zacc, gc);
                // a chunk the main pass cannot take in its chunked form: the
                // sequence is recomputed by the recurrent kernel (these summaries
                // stay exact: every factor above is <= 1)
                if (qt == 0 && p.seq_flags && !(fminf(gc.x, gc.y) >= kGlaMinChunkGate))
                    p.seq_flags[bh] = p.call_id;
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float2 fk = elu_feature2(unpack_bf16x2(kv[i]));
                    if (16 * qt + i >= nvalid) fk = make_float2(0.f, 0.f);
                    *reinterpret_cast<uint32_t *>(ka + off(i)) = pack_bf16x2(fk.x, fk.y);
                    zacc = __fadd2_rn(zacc, fk);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->pfull[s]);
        }
        if constexpr (kGLA) {   // D = R (the same in every token quarter)
            if (qt == 0 && !ctl->abort) *reinterpret_cast<float2 *>(out + DK * DV + 2 * pr) = zacc;
        } else {
            ctl->tot[qt][pr] = zacc;
            bar_named(1, 256);
            if (qt == 0 && !ctl->abort) {
                const float2 z = __fadd2_rn(__fadd2_rn(ctl->tot[0][pr], ctl->tot[1][pr]),
                                            __fadd2_rn(ctl->tot[2][pr], ctl->tot[3][pr]));
                *reinterpret_cast<float2 *>(out + DK * DV + 2 * pr) = z;
            }
        }
    } else if (lane == 0) {
        // TMA producer and MMA issuer
        constexpr uint32_t ID = idesc_bf16(128, DV, true, true);
        int issued = -1;
        auto load = [&](int c) {
            const int s = c % NSTG;
            uint8_t *st = stg(c);
            const int t0 = (kGLA ? cend - 1 - c : cbeg + c) * C;
            mbar_arrive_expect_tx(&ctl->full[s], L::STG_BYTES);
#pragma unroll
            for (int a = 0; a < KA; ++a)
                tma_load_4d(st + a * (C * 128), &maps.k, &ctl->full[s], 64 * a, (int)h, t0, (int)b);
#pragma unroll
            for (int j = 0; j < DV / DVT; ++j)
                tma_load_4d(st + L::K_BYTES + j * (C * DVT * 2), &maps.v, &ctl->full[s], j * DVT, (int)h, t0, (int)b);
            if (kGLA) tma_load_4d(st + L::K_BYTES + L::V_BYTES, &maps.g, &ctl->full[s], 0, (int)h, t0, (int)b);
            issued = c;
        };
        for (int c = 0; c < NSTG && c < n; ++c) load(c);
        for (int c = 0; c < n; ++c) {
            const int s = c % NSTG;
            if (!mbar_wait(&ctl->pfull[s], (uint32_t)(c / NSTG) & 1u)) {
                ctl->abort = 1;
                break;
            }
            tc_fence_after_sync();
            const uint32_t kb = smem_u32(stg(c)), vb = kb + L::K_BYTES;
            const uint64_t du = dmn128_0(kb, C * 128), dv = dmn64_0(vb);
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk)
                umma_bf16(tmem, kstep_mn128(du, kk), kstep_mn64(dv, kk), ID, (c > 0 || kk > 0) ? 1u : 0u);
            umma_commit(&ctl->mdone[s]);
            // the stage of chunk c-1 is free once its MMA is done: refill it
            if (c >= 1 && c - 1 + NSTG < n) {
                if (!mbar_wait(&ctl->mdone[(c - 1) % NSTG], (uint32_t)((c - 1) / NSTG) & 1u)) {
                    ctl->abort = 1;
                    break;
                }
                load(c - 1 + NSTG);
            }
        }
        umma_commit(&ctl->done);
        if (ctl->abort)   // let copies still in flight land before the CTA exits
            for (int c = (issued - NSTG + 1 > 0 ? issued - NSTG + 1 : 0); c <= issued; ++c)
                (void)mbar_drain(&ctl->full[c % NSTG], (uint32_t)(c / NSTG) & 1u);
    }
    if (warp < 4) {   // dS rows out: thread d = key dim
        // the long limit: TMEM is released below, so every MMA must have finished
        const bool ok = __all_sync(0xffffffffu, mbar_drain(&ctl->done, 0u));
        tc_fence_after_sync();
        const int d = 32 * warp + lane;
        const uint32_t tq = tmem + ((uint32_t)(32 * warp) << 16);
#pragma unroll
        for (int j = 0; j < DV / 32; ++j) {
            float x[32];
            tmem_ld32(tq + 32u * (uint32_t)j, x);
            tmem_wait_ld();
            if (ok && !ctl->abort) {
                float *dst = out + (int64_t)d * DV + 32 * j;
#pragma unroll
                for (int e = 0; e < 32; e += 4)
                    *reinterpret_cast<float4 *>(dst + e) = make_float4(x[e], x[e + 1], x[e + 2], x[e + 3]);
            }
        }
        tc_fence_before_sync();
    }
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, L::TMEM_COLS);
}

}  // namespace ck
}  // namespace la
