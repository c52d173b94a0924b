// chunk_ge.cuh — GLA and normalized ELU+1 chunked prefill, warp-specialised and
// software-pipelined across chunks.
//
// One CTA per (batch, head, value slab), 17 warps.  The slab is DVS = 32 value
// columns (GLA) or 64 (ELU+1 when dv allows): a tcgen05 MMA costs about the same
// issue time at N = 32 and N = 64, and the feature-map work per chunk does not
// depend on the slab, so 64 columns per CTA halve both per value column (the
// freed CTAs go to more sequence segments).  With DVS = 64 two accumulators fit
// in TMEM instead of three.
//   warps 0-7    prep: the feature map / gate scaling of q and k on CUDA cores.
//                Thread (pr, qt) owns key dims 2pr, 2pr+1 of tokens 16qt..16qt+15
//                (a warp covers a full 128-byte row per access, conflict-free).
//                GLA: gamma_t = prod_{s<=t} g_s per key dim (local products, then
//                the product of the earlier token quarters), Qt = Q o gamma,
//                Kt = K / gamma (both in place), gamma_C.  ELU+1: phi(Q), phi(K)
//                in place and the chunk's sum of phi(k).  The GLA gate tiles come
//                through a two-slot TMA ring of their own (prefetched into L2 two
//                chunks ahead); the ELU exponential runs on the FMA pipe.
//   warps 8-11   group A: the score epilogue (causal mask of P, bf16 P tile for
//                MMA3; ELU row sums of P) and the output epilogue; its thread 0
//                issues the TMA loads of q, k, v into a ring of stages.
//   warps 12-15  group B: owns the fp32 state slab (one key-dim row per thread),
//                applies each chunk's dS and writes the bf16 copy of the state
//                that the next chunk's MMA1 reads.
//   warp 16      issues every MMA (lane 0), in dependency order.
// A stage holds Q and a K tile whose rows 64.. carry the bf16 S^T (and ELU z^T)
// of the state entering the chunk, so [K' ; S^T (; z^T)] is one operand; it is
// refilled as soon as MMA1 and MMA2 of its chunk are done.  V has a ring of its
// own (its last reader, MMA3, comes later).
// Per chunk c the tensor core computes
//   MMA2(c)  dS = K'^T V                                   -> DS[c%2]
//   MMA1(c)  [P | O_inter (| den_inter)] = Q' [K' ; S^T (; z^T)]^T -> ACC[c%3]
//   MMA3(c)  O += P V                                      -> ACC[c%3] (O columns)
// and the state update is S <- diag(gamma_C) (S + dS) (ELU: S + dS, z += sum phi(k)).
// MMA2 runs two chunks ahead (it does not need the state), MMA1(c+1) starts as
// soon as the state copy of chunk c exists, and MMA3(c) once the P tile of c is
// written; TMEM accumulators are triple-buffered, DS and the P tile doubled.
// Method and notation: see the header of chunk_tc.cuh.
#pragma once

#include "device.cuh"

namespace la {
namespace ck {

template <int RULE, int DVS_>
struct GE {
    static constexpr bool kGLA = (RULE == kRuleGLA);
    static constexpr int DVS = DVS_;                  // value columns per CTA: 32 or 64
    static constexpr int NSTG = (kGLA || DVS == 64) ? 3 : 4;
    static constexpr int NTHREADS = 544;
    static constexpr uint32_t TMEM_COLS = 512;
    // TMEM: NACC accumulators ACC[j] at ACCS j: P (0-63), O (64..64+DVS-1),
    // ELU den (64+DVS); then DS[b] at C_DS + DVS b (M=128)
    static constexpr int NACC = DVS == 64 ? 2 : 3;
    static constexpr uint32_t ACCS = DVS == 64 ? 160 : 128;
    static constexpr uint32_t C_ACC = 0;
    static constexpr uint32_t C_DS = NACC * ACCS;
    static constexpr int KR = 64 + DVS + (kGLA ? 0 : 8);   // K tile rows: K', S^T, ELU z^T, zeros
    static constexpr uint32_t K_ACS = KR * 128;                // bytes per atom column of the K tile
    static constexpr uint32_t Q_BYTES = C * 128 * KA;           // [atom col][64 rows]
    static constexpr uint32_t K_BYTES = K_ACS * KA;
    static constexpr uint32_t V_BYTES = C * DVS * 2;            // [64][DVS], 64- or 128-byte swizzle
    static constexpr uint32_t STG_BYTES = Q_BYTES + K_BYTES;
    // V ring slots and GLA gate slots: GLA with 64 columns keeps three q/k stages
    // (the scarcer lead) by holding one gate tile, loaded as soon as the prep
    // warps have the previous one in registers
    static constexpr int NV = (kGLA && DVS == 64) ? 3 : 4;
    static constexpr int NG = (kGLA && DVS == 64) ? 1 : 2;
    static constexpr uint32_t G_BYTES = C * DK * 4;             // GLA gate tile, fp32 [64][128]
    // tiles
    static constexpr uint32_t STG = 0;
    static constexpr uint32_t VR = STG + NSTG * STG_BYTES;      // V ring
    static constexpr uint32_t GT = VR + NV * V_BYTES;           // GLA: NG gate slots
    static constexpr uint32_t PS = GT + (kGLA ? NG * G_BYTES : 0);
    static constexpr uint32_t END = PS + 2 * C * 128;
    // with the control block (5 KB) and the 1 KB alignment slack, within the
    // 227 KB a CTA may use
    static_assert(END + 6144 <= 232448, "chunk_ge_kernel tiles exceed shared memory");
    static constexpr int N1 = KR;
};

struct GECtl {
    uint64_t full[4];                // TMA of a stage's q and k landed
    uint64_t vfull[4];               // TMA of a V slot landed
    uint64_t pfull[4];               // the stage's chunk prepared (8 prep warps)
    uint64_t gfull[2];               // GLA gate slot landed
    uint64_t mP[3];                  // MMA1 of the chunk (and everything issued before it) done
    uint64_t m3[3];                  // MMA3 of the chunk done
    uint64_t oA[3];                  // output epilogue of the chunk done (128)
    uint64_t mD[2];                  // MMA2 of the chunk done
    uint64_t pA[2];                  // P tile written (128)
    uint64_t sB[2];                  // state copy written (128)
    uint64_t s0;                     // initial state copy written (128)
    uint64_t drain;
    uint32_t tmem_base;
    int abort, stopP;
    int seqfail;                     // GLA: a chunk of this CTA left the chunked form's range
    alignas(16) float gC[4][128];    // GLA: gamma at chunk end per key dim; ELU: chunk sum of phi(k)
    alignas(16) float2 tot[4][64];   // prep: per-quarter gate products (GLA) / sums of phi(k) (ELU)
};

__device__ __forceinline__ bool aborted(const GECtl *ctl) {
    return __any_sync(0xffffffffu, *reinterpret_cast<const volatile int *>(&ctl->abort) != 0);
}

template <int RULE, int DVS>
__global__ void __launch_bounds__(544, 1)
chunk_ge_kernel(const __grid_constant__ Maps maps, const ChunkParams p) {
    using L = GE<RULE, DVS>;
    constexpr int NACC = L::NACC;
    constexpr bool kGLA = L::kGLA;
    constexpr int NSTG = L::NSTG;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    GECtl *ctl = reinterpret_cast<GECtl *>(smem_raw);
    uint8_t *tiles = smem_raw + align1k((uint32_t)sizeof(GECtl) + (smem_u32(smem_raw) & 1023u)) -
                     (smem_u32(smem_raw) & 1023u);
    const uint32_t tb = smem_u32(tiles);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3;
    const int nslab = (int)(p.dv / DVS);
    const int dvt = (int)(blockIdx.x % nslab);
    const int seg = (int)((blockIdx.x / nslab) % p.nseg);
    const int64_t bh = blockIdx.x / nslab / p.nseg;
    const int64_t b = bh / p.H, h = bh % p.H;
    // this sequence's tokens (dense layout: all T of batch b; packed: its span of
    // the token axis) and this CTA's chunks [cbase, cbase + nchunks) of it
    const SeqSpan sq = seq_span(p.cu_seqlens, b, p.T, p.max_seqlen, threadIdx.x == 0 && h == 0 && dvt == 0);
    const int cbase = seg * p.seg_chunks;
    const int nchunks = (int)max((int64_t)0, min((int64_t)p.seg_chunks, (sq.len + C - 1) / C - cbase));

    auto stg = [&](int c) { return tiles + L::STG + (uint32_t)(c % NSTG) * L::STG_BYTES; };

    if (tid == 0) {
        for (int s = 0; s < L::NV; ++s) mbar_init(&ctl->vfull[s], 1);
        for (int s = 0; s < NSTG; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->pfull[s], 8);
        }
        for (int i = 0; i < 3; ++i) {
            mbar_init(&ctl->mP[i], 1);
            mbar_init(&ctl->m3[i], 1);
            mbar_init(&ctl->oA[i], 128);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&ctl->mD[i], 1);
            mbar_init(&ctl->gfull[i], 1);
            mbar_init(&ctl->pA[i], 128);
            mbar_init(&ctl->sB[i], 128);
        }
        mbar_init(&ctl->s0, 128);
        mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        ctl->seqfail = 0;
        fence_barrier_init();
        tma_prefetch_desc(&maps.q);
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
    const uint32_t tmem = ctl->tmem_base;
    const uint32_t tq = tmem + ((uint32_t)(32 * quad) << 16);

    if (warp < 8) {
        // ------------------------------------------------------------------ prep
        // Thread (pr, qt) owns key dims 2pr, 2pr+1 of tokens 16qt..16qt+15.  One
        // warp covers 32 consecutive pairs (a full 128-byte row of one atom
        // column) of one token per access, so its 4- and 8-byte shared-memory
        // accesses are free of bank conflicts.  All loads of a chunk are issued
        // before its first store.
        const int lt = tid;
        const bool leader = (lt == 0);
        const int pr = lt & 63, qt = lt >> 6;
        const int a = pr >> 5;                                   // atom column
        const uint32_t cpos = (uint32_t)((pr & 31) >> 2), cin = (uint32_t)(pr & 3) << 2;
        // GLA gate tile of chunk c into slot c % NG (issued by prep thread 0 once
        // every prep thread is done with the slot's previous chunk: with two slots
        // at the top of chunk c-1, with one as soon as chunk c-1's gates are in
        // registers)
        int g_issued = -1, g_used = -1;   // thread 0: last gate tiles loaded / seen landed
        auto gate_load = [&](int c) {
            const int j = c % L::NG;
            uint64_t *bar = &ctl->gfull[j];
            mbar_arrive_expect_tx(bar, L::G_BYTES);
            tma_load_4d(tiles + L::GT + (uint32_t)j * L::G_BYTES, &maps.g, bar, 0, (int)h,
                        sq.t0 + (cbase + c) * C, sq.b0);
            g_issued = c;
        };
        if (kGLA && leader)
            for (int c = 0; c < L::NG && c < nchunks; ++c) gate_load(c);
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % NSTG;
            const int nvalid = (int)min((int64_t)C, sq.len - (int64_t)(cbase + c) * C);
            if (leader) ctl->stopP = ctl->abort;
            bar_named(1, 256);
            if (ctl->stopP) break;
            if (kGLA && L::NG == 2 && leader && c >= 1 && c + 1 < nchunks) {
                fence_proxy_async_smem();
                gate_load(c + 1);
            }
            if (kGLA) {
                if (mbar_wait(&ctl->gfull[c % L::NG], (uint32_t)(c / L::NG) & 1u)) g_used = c;
                else ctl->abort = 1;
            }
            if (!mbar_wait(&ctl->full[s], (uint32_t)(c / NSTG) & 1u)) ctl->abort = 1;
            uint8_t *st = stg(c);
            uint8_t *qa = st + a * (C * 128), *ka = st + L::Q_BYTES + a * L::K_ACS;
            auto off = [&](int i) {
                const uint32_t t = (uint32_t)(16 * qt + i);
                return t * 128u + (((cpos ^ t) & 7u) << 4) + cin;
            };
            if constexpr (kGLA) {
                // gamma_t = prod_{s<=t} g_s inside the chunk: local products over
                // this thread's 16 tokens, then the product of the earlier quarters.
                const uint8_t *G = tiles + L::GT + (uint32_t)(c % L::NG) * L::G_BYTES;   // fp32 [64][128]
                float2 gv[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int t = 16 * qt + i;
                    gv[i] = *reinterpret_cast<const float2 *>(G + t * 512 + pr * 8);
                    if (t >= nvalid) gv[i] = make_float2(1.f, 1.f);
                }
#pragma unroll
                for (int i = 1; i < 16; ++i) gv[i] = __fmul2_rn(gv[i - 1], gv[i]);
                ctl->tot[qt][pr] = gv[15];
                bar_named(1, 256);
                if (L::NG == 1 && leader && c + 1 < nchunks && !ctl->abort) {
                    fence_proxy_async_smem();   // every prep thread holds chunk c's gates in registers
                    gate_load(c + 1);
                }
                float2 pre = make_float2(1.f, 1.f);
                for (int q2 = 0; q2 < qt; ++q2) pre = __fmul2_rn(pre, ctl->tot[q2][pr]);
                if (qt == 3) {
                    const float2 gc = __fmul2_rn(pre, gv[15]);
                    *reinterpret_cast<float2 *>(&ctl->gC[c & 3][2 * pr]) = gc;
                    // out of the chunked form's range: this CTA's results for the
                    // sequence are discarded and the recurrent kernel recomputes it
                    if (!(fminf(gc.x, gc.y) >= kGlaMinChunkGate)) {
                        ctl->seqfail = 1;
                        if (p.seq_flags) p.seq_flags[bh] = p.call_id;
                    }
                }
                // Qt = Q o gamma, Kt = K / gamma (both in place), 8 tokens at a time
#pragma unroll
                for (int h8 = 0; h8 < 16; h8 += 8) {
                    uint32_t qv[8], kv[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        qv[i] = *reinterpret_cast<const uint32_t *>(qa + off(h8 + i));
                        kv[i] = *reinterpret_cast<const uint32_t *>(ka + off(h8 + i));
                    }
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float2 gm = __fmul2_rn(pre, gv[h8 + i]);
                        const float2 ig = make_float2(rcp_approx(gm.x), rcp_approx(gm.y));
                        const float2 qs = __fmul2_rn(unpack_bf16x2(qv[i]), gm);
                        const float2 ks = __fmul2_rn(unpack_bf16x2(kv[i]), ig);
                        *reinterpret_cast<uint32_t *>(qa + off(h8 + i)) = pack_bf16x2(qs.x, qs.y);
                        *reinterpret_cast<uint32_t *>(ka + off(h8 + i)) = pack_bf16x2(ks.x, ks.y);
                    }
                }
                // last chunk of a sequence: in a packed layout the rows past its
                // end hold the next sequence's keys, which must not reach dS = K'^T V
                if (nvalid < C) {
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        if (16 * qt + i >= nvalid) *reinterpret_cast<uint32_t *>(ka + off(i)) = 0u;
                }
            } else {
                // phi(Q), phi(K) in place (phi(k) = 0 past T), chunk sum of phi(k)
                uint32_t qv[16], kv[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    qv[i] = *reinterpret_cast<const uint32_t *>(qa + off(i));
                    kv[i] = *reinterpret_cast<const uint32_t *>(ka + off(i));
                }
                float2 zs = make_float2(0.f, 0.f);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float2 qf = unpack_bf16x2(qv[i]), kf = unpack_bf16x2(kv[i]);
                    float2 fk = elu_feature2(kf);
                    if (16 * qt + i >= nvalid) fk = make_float2(0.f, 0.f);
                    const float2 fq = elu_feature2(qf);
                    *reinterpret_cast<uint32_t *>(qa + off(i)) = pack_bf16x2(fq.x, fq.y);
                    *reinterpret_cast<uint32_t *>(ka + off(i)) = pack_bf16x2(fk.x, fk.y);
                    zs = __fadd2_rn(zs, fk);
                }
                ctl->tot[qt][pr] = zs;
                bar_named(1, 256);
                if (qt == 0) {
                    float2 z = __fadd2_rn(ctl->tot[0][pr], ctl->tot[1][pr]);
                    z = __fadd2_rn(z, __fadd2_rn(ctl->tot[2][pr], ctl->tot[3][pr]));
                    *reinterpret_cast<float2 *>(&ctl->gC[c & 3][2 * pr]) = z;
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->pfull[s]);
        }
        // after an abort, let gate copies still in flight land before the CTA can exit
        if (kGLA && leader)
            for (int c = g_used + 1; c <= g_issued; ++c)
                (void)mbar_drain(&ctl->gfull[c % L::NG], (uint32_t)(c / L::NG) & 1u);
    } else if (warp < 12) {
        // ------------------------------------------------------------------ group A
        const bool a0 = (tid == 256);
        const int tr = 16 * quad + (lane & 15);     // chunk row of the M=64 accumulators
        const int hf = lane >> 4;
        int issued = -1, issued_v = -1;             // last chunks whose TMA thread a0 issued
        // TMA of q and k for chunk c
        auto load_chunk = [&](int c) {
            const int s = c % NSTG;
            uint8_t *st = stg(c);
            const int t0 = sq.t0 + (cbase + c) * C;   // tensor-map coordinate of the chunk's first token
            mbar_arrive_expect_tx(&ctl->full[s], 2u * L::Q_BYTES);
#pragma unroll
            for (int a = 0; a < KA; ++a) {
                tma_load_4d(st + a * (C * 128), &maps.q, &ctl->full[s], 64 * a, (int)h, t0, sq.b0);
                tma_load_4d(st + L::Q_BYTES + a * L::K_ACS, &maps.k, &ctl->full[s], 64 * a, (int)h, t0, sq.b0);
            }
            // the gate tile of chunk c+2 is loaded about one chunk period from
            // now: start bringing it into L2
            if (kGLA && dvt == 0 && c + 2 < nchunks) tma_prefetch_l2_4d(&maps.g, 0, (int)h, t0 + 2 * C, sq.b0);
            issued = c;
        };
        // TMA of this CTA's V slab for chunk c
        auto load_v = [&](int c) {
            const int j = c % L::NV;
            mbar_arrive_expect_tx(&ctl->vfull[j], L::V_BYTES);
            tma_load_4d(tiles + L::VR + (uint32_t)j * L::V_BYTES, &maps.v, &ctl->vfull[j], dvt * DVS, (int)h,
                        sq.t0 + (cbase + c) * C, sq.b0);
            issued_v = c;
        };
        if (a0) {
            for (int c = 0; c < NSTG && c < nchunks; ++c) load_chunk(c);
            for (int c = 0; c < L::NV && c < nchunks; ++c) load_v(c);
        }
        for (int c = 0; c < nchunks; ++c) {
            const int bb = c & 1, j3 = c % NACC;
            const uint32_t acc = L::C_ACC + L::ACCS * (uint32_t)j3;
            const int64_t t0 = (int64_t)(cbase + c) * C;   // position in the sequence
            const int nvalid = (int)min((int64_t)C, sq.len - t0);
            if (aborted(ctl)) break;
            if (!__all_sync(0xffffffffu, mbar_wait(&ctl->mP[j3], (uint32_t)(c / NACC) & 1u))) {
                ctl->abort = 1;
                break;
            }
            // MMA1(c) and MMA2(c) were the last readers of the stage's q and k
            if (a0 && !ctl->abort && c + NSTG < nchunks) load_chunk(c + NSTG);
            tc_fence_after_sync();
            float den = 0.f;
            {   // P row tr, columns 32*hf..: causal mask -> bf16 tile PS[bb]; ELU row sums
                float x[32];
                tmem_ld16x2_32<32>(tq + acc, x);
                float dI[16];
                if (!kGLA) tmem_ld16(tq + acc + 64 + DVS, dI);
                tmem_wait_ld();
                float rs = 0.f;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    x[i] = (32 * hf + i <= tr) ? x[i] : 0.f;
                    rs += x[i];
                }
                uint8_t *ps = tiles + L::PS + bb * (C * 128);
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    uint4 u;
                    u.x = pack_bf16x2(x[8 * cc + 0], x[8 * cc + 1]);
                    u.y = pack_bf16x2(x[8 * cc + 2], x[8 * cc + 3]);
                    u.z = pack_bf16x2(x[8 * cc + 4], x[8 * cc + 5]);
                    u.w = pack_bf16x2(x[8 * cc + 6], x[8 * cc + 7]);
                    const int chunk = 4 * hf + cc;
                    *reinterpret_cast<uint4 *>(ps + tr * 128 + (((chunk ^ tr) & 7) << 4)) = u;
                }
                if (!kGLA) {
                    rs += __shfl_xor_sync(0xffffffffu, rs, 16);
                    const float dz = __shfl_sync(0xffffffffu, dI[0], lane & 15);
                    den = dz + rs + p.eps;
                }
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            mbar_arrive(&ctl->pA[bb]);
            if (!__all_sync(0xffffffffu, mbar_wait(&ctl->m3[j3], (uint32_t)(c / NACC) & 1u))) {
                ctl->abort = 1;
                break;
            }
            tc_fence_after_sync();
            {   // row tr, columns (DVS/2) hf .. of the slab
                constexpr int OH = DVS / 2;
                float o[OH];
                if constexpr (DVS == 64) tmem_ld16x2_32<32>(tq + acc + 64, o);
                else tmem_ld16x2_16<16>(tq + acc + 64, o);
                tmem_wait_ld();
                if (tr < nvalid) {
                    if (!kGLA) {
                        const float inv = 1.f / den;
#pragma unroll
                        for (int jj = 0; jj < OH; ++jj) o[jj] *= inv;
                    }
                    __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(p.o) +
                                         ((sq.row0 + t0 + tr) * p.H + h) * p.dv + dvt * DVS + OH * hf;
#pragma unroll
                    for (int cc = 0; cc < OH / 8; ++cc) {
                        uint4 u;
                        u.x = pack_bf16x2(o[8 * cc + 0], o[8 * cc + 1]);
                        u.y = pack_bf16x2(o[8 * cc + 2], o[8 * cc + 3]);
                        u.z = pack_bf16x2(o[8 * cc + 4], o[8 * cc + 5]);
                        u.w = pack_bf16x2(o[8 * cc + 6], o[8 * cc + 7]);
                        reinterpret_cast<uint4 *>(dst)[cc] = u;
                    }
                }
            }
            tc_fence_before_sync();
            mbar_arrive(&ctl->oA[j3]);
            // MMA3(c) was the last reader of the chunk's V slot: refill it
            if (a0 && !ctl->abort && c + L::NV < nchunks) load_v(c + L::NV);
        }
        if (a0 && ctl->abort) {   // let copies still in flight land before the CTA exits
            for (int c = (issued - NSTG + 1 > 0 ? issued - NSTG + 1 : 0); c <= issued; ++c)
                (void)mbar_drain(&ctl->full[c % NSTG], (uint32_t)(c / NSTG) & 1u);
            for (int c = (issued_v - L::NV + 1 > 0 ? issued_v - L::NV + 1 : 0); c <= issued_v; ++c)
                (void)mbar_drain(&ctl->vfull[c % L::NV], (uint32_t)(c / L::NV) & 1u);
        }
    } else if (warp < 16) {
        // ------------------------------------------------------------------ group B
        const int d = 32 * quad + lane;             // state row (key dim)
        float S[DVS];
        float z = 0.f;
        {
            const float *src = p.S0 ? p.S0 + ((bh * DK + d) * p.dv + dvt * DVS) : nullptr;
#pragma unroll
            for (int jj = 0; jj < DVS; jj += 4) {
                float4 x = src ? *reinterpret_cast<const float4 *>(src + jj) : make_float4(0, 0, 0, 0);
                S[jj] = x.x; S[jj + 1] = x.y; S[jj + 2] = x.z; S[jj + 3] = x.w;
            }
            if (!kGLA && p.z0) z = p.z0[bh * DK + d];
            // sequence-parallel pass: fold the state through the token ranges of the
            // earlier segments, in order (ELU+1: S += dS, z += dz; GLA: S <- D o S + dS).
            // This kernel is then a programmatic dependent of the summary pass: the
            // summaries (and its range flags, read at the end) are complete and visible
            // once the wait returns.  The first segment needs neither.
            if (seg > 0) asm volatile("griddepcontrol.wait;" ::: "memory");
            const int64_t blk = (int64_t)DK * p.dv + DK;
            for (int i = 0; i < seg * p.nparts; ++i) {
                const float *a = p.agg + (bh * (p.nseg - 1) * p.nparts + i) * blk;
                const float *row = a + (int64_t)d * p.dv + dvt * DVS;
                const float dd = kGLA ? a[DK * p.dv + d] : 1.f;
#pragma unroll
                for (int jj = 0; jj < DVS; jj += 4) {
                    const float4 x = *reinterpret_cast<const float4 *>(row + jj);
                    S[jj] = fmaf(dd, S[jj], x.x);
                    S[jj + 1] = fmaf(dd, S[jj + 1], x.y);
                    S[jj + 2] = fmaf(dd, S[jj + 2], x.z);
                    S[jj + 3] = fmaf(dd, S[jj + 3], x.w);
                }
                if (!kGLA) z += a[DK * p.dv + d];
            }
        }
        // bf16 copy of S^T (and z^T) into rows 64.. of the K tile of stage s
        auto write_state = [&](int s) {
            uint8_t *ka = tiles + L::STG + (uint32_t)s * L::STG_BYTES + L::Q_BYTES + (d >> 6) * L::K_ACS;
            const int dc = d & 63;
#pragma unroll
            for (int jj = 0; jj < DVS; ++jj) *elem(ka, 64 + jj, dc) = __float2bfloat16_rn(S[jj]);
            if (!kGLA) *elem(ka, 64 + DVS, dc) = __float2bfloat16_rn(z);
        };
        if (!kGLA) {   // rows 97..103 of every stage's K tile stay zero
            for (int s = 0; s < NSTG; ++s) {
                uint8_t *ka = tiles + L::STG + (uint32_t)s * L::STG_BYTES + L::Q_BYTES + (d >> 6) * L::K_ACS;
#pragma unroll
                for (int r = 64 + DVS + 1; r < L::KR; ++r) *elem(ka, r, d & 63) = __float2bfloat16_rn(0.f);
            }
        }
        write_state(0);
        fence_proxy_async_smem();
        mbar_arrive(&ctl->s0);
        bool ok = nchunks == 0 || __all_sync(0xffffffffu, mbar_wait(&ctl->pfull[0], 0u));
        if (!ok) ctl->abort = 1;
        for (int c = 0; c < nchunks && ok; ++c) {
            const int bb = c & 1;
            if (aborted(ctl)) break;
            if (!__all_sync(0xffffffffu, mbar_wait(&ctl->mD[bb], (uint32_t)(c >> 1) & 1u))) {
                ctl->abort = 1;
                break;
            }
            tc_fence_after_sync();
            {
                const float g = ctl->gC[c & 3][d];
#pragma unroll
                for (int hh = 0; hh < DVS / 16; ++hh) {   // 16 columns of dS at a time
                    float ds[16];
                    tmem_ld16(tq + L::C_DS + (uint32_t)DVS * (uint32_t)bb + 16u * hh, ds);
                    tmem_wait_ld();
                    if (kGLA) {
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj) S[16 * hh + jj] = g * (S[16 * hh + jj] + ds[jj]);
                    } else {
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj) S[16 * hh + jj] += ds[jj];
                    }
                }
                if (!kGLA) z += g;
            }
            if (c + 1 < nchunks) {
                write_state((c + 1) % NSTG);
                // the prep of c+1 is complete (its gamma_C / sum of phi(k) is readable)
                if (!__all_sync(0xffffffffu, mbar_wait(&ctl->pfull[(c + 1) % NSTG],
                                                               (uint32_t)((c + 1) / NSTG) & 1u))) {
                    ctl->abort = 1;
                    break;
                }
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            mbar_arrive(&ctl->sB[bb]);
        }
        // a sequence flagged here or, for the earlier segments, by the summary
        // pass keeps S_out untouched (S0 may alias it): the recurrent kernel
        // recomputes it from S0
        const bool last = seg == p.nseg - 1;
        const bool flagged = kGLA && last && (*reinterpret_cast<volatile int *>(&ctl->seqfail) != 0 ||
                                              (p.seq_flags && p.seq_flags[bh] == p.call_id));
        if (!ctl->abort && last && !flagged) {
            if (p.S_out) {
                float *dst = p.S_out + ((bh * DK + d) * p.dv + dvt * DVS);
#pragma unroll
                for (int jj = 0; jj < DVS; jj += 4)
                    *reinterpret_cast<float4 *>(dst + jj) = make_float4(S[jj], S[jj + 1], S[jj + 2], S[jj + 3]);
            }
            if (!kGLA && p.z_out && dvt == 0) p.z_out[bh * DK + d] = z;
        }
    } else if (lane == 0) {
        // ------------------------------------------------------------------ MMA issue
        constexpr uint32_t ID1 = idesc_bf16(64, L::N1, false, false);
        constexpr uint32_t ID2 = idesc_bf16(128, DVS, true, true);
        constexpr uint32_t ID3 = idesc_bf16(64, DVS, false, true);
        // V as the MN-major B operand: [64 tokens][DVS] with the 64-byte (DVS = 32)
        // or 128-byte (DVS = 64) swizzle
        auto vdesc = [&](uint32_t vb) { return DVS == 64 ? dmn128_0(vb, 8192u) : dmn64_0(vb); };
        auto vstep = [&](uint64_t d0, int kk) { return DVS == 64 ? kstep_mn128(d0, kk) : kstep_mn64(d0, kk); };
        // MMA1(c): [P | O_inter (| den)] = Q'(c) [K'(c) ; S^T (; z^T)]^T, K = dk
        auto issue_mma1 = [&](int c) {
            const uint32_t qb = smem_u32(stg(c)), kb = qb + L::Q_BYTES;
            const uint64_t dq = dk0(qb), dkx = dk0(kb);
            const uint32_t acc = tmem + L::C_ACC + L::ACCS * (uint32_t)(c % NACC);
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk)
                umma_bf16(acc, kstep_k(dq, C * 128, kk), kstep_k(dkx, L::K_ACS, kk), ID1, kk > 0);
            umma_commit(&ctl->mP[c % NACC]);
        };
        // MMA2(c): dS = K'(c)^T V(c), K = tokens
        auto issue_mma2 = [&](int c) {
            const uint32_t kb = smem_u32(stg(c)) + L::Q_BYTES, vb = tb + L::VR + (uint32_t)(c % L::NV) * L::V_BYTES;
            const uint64_t du = dmn128_0(kb, L::K_ACS), dv = vdesc(vb);
            const uint32_t ds = tmem + L::C_DS + (uint32_t)DVS * (uint32_t)(c & 1);
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk)
                umma_bf16(ds, kstep_mn128(du, kk), vstep(dv, kk), ID2, kk > 0);
            umma_commit(&ctl->mD[c & 1]);
        };
        // MMA3(c): O += P(c) V(c)
        auto issue_mma3 = [&](int c) {
            const uint32_t vb = tb + L::VR + (uint32_t)(c % L::NV) * L::V_BYTES;
            const uint64_t dp = dk0(tb + L::PS + (uint32_t)(c & 1) * (C * 128)), dv = vdesc(vb);
            const uint32_t acc = tmem + L::C_ACC + L::ACCS * (uint32_t)(c % NACC) + 64u;
#pragma unroll
            for (int kk = 0; kk < C / 16; ++kk)
                umma_bf16(acc, kstep_k(dp, C * 128, kk), vstep(dv, kk), ID3, 1u);
            umma_commit(&ctl->m3[c % NACC]);
        };
        auto ready = [&](bool w) {
            if (!w) ctl->abort = 1;
            fence_proxy_async_smem();
            tc_fence_after_sync();
            return w;
        };
        // MMA2(c) needs the chunk prepared and its V slot landed
        auto mma2_ready = [&](int c) {
            return ready(mbar_wait(&ctl->pfull[c % NSTG], (uint32_t)(c / NSTG) & 1u) &&
                         mbar_wait(&ctl->vfull[c % L::NV], (uint32_t)(c / L::NV) & 1u));
        };
        bool ok = true;
        if (nchunks > 0) {
            ok = mma2_ready(0);
            if (ok) issue_mma2(0);
            ok = ok && ready(mbar_wait(&ctl->s0, 0u));
            if (ok) issue_mma1(0);
            if (ok && nchunks > 1) {
                ok = mma2_ready(1);
                if (ok) issue_mma2(1);
            }
        }
        for (int c = 0; c < nchunks && ok; ++c) {
            if (*reinterpret_cast<volatile int *>(&ctl->abort)) break;
            if (c + 1 < nchunks) {
                // the state copy of chunk c is written (and DS[c&1] read); ACC[(c+1)%NACC]
                // was released by the output epilogue of chunk c+1-NACC
                ok = mbar_wait(&ctl->sB[c & 1], (uint32_t)(c >> 1) & 1u);
                if (ok && c + 1 >= NACC)
                    ok = mbar_wait(&ctl->oA[(c + 1) % NACC], (uint32_t)((c + 1 - NACC) / NACC) & 1u);
                if (!ready(ok)) break;
                issue_mma1(c + 1);
            }
            if (!ready(mbar_wait(&ctl->pA[c & 1], (uint32_t)(c >> 1) & 1u))) break;
            issue_mma3(c);
            if (c + 2 < nchunks) {
                if (!mma2_ready(c + 2)) break;
                issue_mma2(c + 2);
            }
        }
        // every MMA issued so far has finished before TMEM is released
        umma_commit(&ctl->drain);
        (void)mbar_drain(&ctl->drain, 0u);
    }
    // GLA: the exact recomputation kernel that follows may be scheduled now (it
    // waits for this grid's completion before reading anything)
    if (kGLA) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, L::TMEM_COLS);
}

}  // namespace ck
}  // namespace la
