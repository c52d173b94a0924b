// chunk_ge.cuh — GLA and normalized ELU+1 chunked prefill, warp-specialised.
//
// One CTA per (batch, head, 32-column value slab), 12 warps:
//   warps 0-7   "prep" group, one chunk ahead: the feature map / gate scaling of
//               q and k on CUDA cores (8 key dims x 4 tokens per thread, 16-byte
//               accesses).  GLA: gamma_t = prod_{s<=t} g_s per key dim (local
//               products over 4 tokens, then an exclusive product over the 16
//               token groups),
//               Qt = Q o gamma (in place), Kt = K / gamma (operand tile Kx),
//               Kh = Kt o gamma_C (in place), gamma_C per dim.  ELU+1:
//               phi(Q) in place, phi(K) into Kx, the chunk's sum of phi(k) per dim;
//   warps 8-11  "state" group: issues the TMA loads of q, k, v (and the GLA
//               gate) into a ring of stages and the MMAs of its chunk, and owns
//               the fp32 state (one key-dim row per thread):
//                 MMA1  [P | O_inter (| den_inter)] = Q' [K' ; S^T (; z^T)]^T,
//                 MMA2  dS = K''^T V,
//                 P masked -> bf16, S <- diag(gamma_C) S + dS (ELU: S + dS, z += sum phi(k)),
//                 MMA3  O += P V,  O -> global (ELU: / (phi(q).z0 + rowsum(P) + eps)).
// Method and notation: see the header of chunk_tc.cuh.
#pragma once

#include "device.cuh"

namespace la {
namespace ck {

template <int RULE>
struct GE {
    static constexpr bool kGLA = (RULE == kRuleGLA);
    static constexpr int NSTG = kGLA ? 2 : 3;
    static constexpr int NTHREADS = 384;
    static constexpr uint32_t TMEM_COLS = 256;
    static constexpr uint32_t C_ACC = 0;     // MMA1: P (0-63), O (64-95), ELU den (96)
    static constexpr uint32_t C_DS = 128;    // MMA2: dS, M=128
    static constexpr int KX_ROWS = kGLA ? 96 : 104;   // K' (0-63), S^T (64-95), ELU z^T (96), zeros
    static constexpr uint32_t KX_ACS = KX_ROWS * 128;
    static constexpr uint32_t KX_BYTES = KX_ACS * KA;
    static constexpr uint32_t Q_BYTES = C * 128 * KA;           // [atom col][64 rows]
    static constexpr uint32_t G_BYTES = kGLA ? C * DK * 4 : 0;  // fp32 [64][128]
    static constexpr uint32_t STG_BYTES = 2 * Q_BYTES + 4096 + G_BYTES;
    // tiles
    static constexpr uint32_t STG = 0;
    static constexpr uint32_t KX = STG + NSTG * STG_BYTES;
    static constexpr uint32_t PS = KX + 2 * KX_BYTES;
    static constexpr uint32_t END = PS + C * 128;
    static constexpr int N1 = KX_ROWS;
};

struct GECtl {
    uint64_t full[3];
    uint64_t pfull[2], pempty[2], m1_done, m3_done;
    uint32_t tmem_base;
    int abort, stopP, stopS;
    alignas(16) float gC[2][128];    // GLA: gamma at chunk end per key dim; ELU: chunk sum of phi(k)
    alignas(16) float tot[16][128];  // prep: per token-group products (GLA) / sums of phi(k) (ELU)
};

template <int RULE>
__global__ void __launch_bounds__(384, 1)
chunk_ge_kernel(const __grid_constant__ Maps maps, const ChunkParams p) {
    using L = GE<RULE>;
    constexpr bool kGLA = L::kGLA;
    constexpr int NSTG = L::NSTG;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    GECtl *ctl = reinterpret_cast<GECtl *>(smem_raw);
    uint8_t *tiles = smem_raw + align1k((uint32_t)sizeof(GECtl) + (smem_u32(smem_raw) & 1023u)) -
                     (smem_u32(smem_raw) & 1023u);
    const uint32_t tb = smem_u32(tiles);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3;
    const int nslab = (int)(p.dv / DVT);
    const int dvt = (int)(blockIdx.x % nslab);
    const int64_t bh = blockIdx.x / nslab;
    const int64_t b = bh / p.H, h = bh % p.H;
    const int nchunks = (int)((p.T + C - 1) / C);

    auto stg = [&](int c) { return tiles + L::STG + (uint32_t)(c % NSTG) * L::STG_BYTES; };

    if (tid == 0) {
        for (int s = 0; s < NSTG; ++s) mbar_init(&ctl->full[s], 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&ctl->pfull[i], 256);
            mbar_init(&ctl->pempty[i], 1);
        }
        mbar_init(&ctl->m1_done, 1);
        mbar_init(&ctl->m3_done, 1);
        ctl->abort = 0;
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

    // TMA of chunk c into its stage (issued by the state group's leader)
    auto load_chunk = [&](int c) {
        const int s = c % NSTG;
        uint8_t *st = stg(c);
        const int t0 = c * C;
        mbar_arrive_expect_tx(&ctl->full[s], 2u * L::Q_BYTES + C * DVT * 2u + L::G_BYTES);
#pragma unroll
        for (int a = 0; a < KA; ++a) {
            tma_load_4d(st + a * (C * 128), &maps.q, &ctl->full[s], 64 * a, (int)h, t0, (int)b);
            tma_load_4d(st + L::Q_BYTES + a * (C * 128), &maps.k, &ctl->full[s], 64 * a, (int)h, t0, (int)b);
        }
        tma_load_4d(st + 2 * L::Q_BYTES, &maps.v, &ctl->full[s], dvt * DVT, (int)h, t0, (int)b);
        if (kGLA) tma_load_4d(st + 2 * L::Q_BYTES + 4096, &maps.g, &ctl->full[s], 0, (int)h, t0, (int)b);
    };

    if (warp < 8) {
        // ------------------------------------------------------------------ prep group
        const int lt = tid;
        const bool leader = (lt == 0);
        const int j = lt & 15, tg = lt >> 4;           // dims 8j..8j+7, tokens 4tg..4tg+3
        const int a = j >> 3, cj = j & 7;              // atom column, 16-byte chunk in the row
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % NSTG, kb = c & 1;
            const int nvalid = (int)min((int64_t)C, p.T - (int64_t)c * C);
            if (leader) ctl->stopP = ctl->abort;
            bar_named(1, 256);
            if (ctl->stopP) break;
            if (!mbar_wait(&ctl->full[s], (uint32_t)(c / NSTG) & 1u)) ctl->abort = 1;
            if (c >= 2 && !mbar_wait(&ctl->pempty[kb], (uint32_t)((c - 2) >> 1) & 1u)) ctl->abort = 1;
            uint8_t *st = stg(c);
            uint8_t *qa = st + a * (C * 128), *ka = st + L::Q_BYTES + a * (C * 128);
            uint8_t *kxa = tiles + L::KX + kb * L::KX_BYTES + a * L::KX_ACS;
            if constexpr (kGLA) {
                const float *G = reinterpret_cast<const float *>(st + 2 * L::Q_BYTES + 4096);
                float gam[4][8];   // [token][dim], products from the start of this thread's 4 tokens
                float run[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) run[e] = 1.f;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int t = 4 * tg + i;
                    float gv[8];
                    const float4 g0 = *reinterpret_cast<const float4 *>(G + t * DK + 8 * j);
                    const float4 g1 = *reinterpret_cast<const float4 *>(G + t * DK + 8 * j + 4);
                    gv[0] = g0.x; gv[1] = g0.y; gv[2] = g0.z; gv[3] = g0.w;
                    gv[4] = g1.x; gv[5] = g1.y; gv[6] = g1.z; gv[7] = g1.w;
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        run[e] *= (t < nvalid) ? gv[e] : 1.f;
                        gam[i][e] = run[e];
                    }
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) ctl->tot[tg][8 * j + e] = run[e];
                bar_named(1, 256);
                if (lt < DK) {   // exclusive product over the 16 token groups, one key dim per thread
                    float acc = 1.f;
#pragma unroll
                    for (int g2 = 0; g2 < 16; ++g2) {
                        const float tv = ctl->tot[g2][lt];
                        ctl->tot[g2][lt] = acc;
                        acc *= tv;
                    }
                    ctl->gC[kb][lt] = acc;
                    if (!(acc >= 1e-30f)) raise_error(kErrRange);
                }
                bar_named(1, 256);
                float pre[8], gC[8];
                {
                    const float4 p0 = *reinterpret_cast<const float4 *>(&ctl->tot[tg][8 * j]);
                    const float4 p1 = *reinterpret_cast<const float4 *>(&ctl->tot[tg][8 * j + 4]);
                    const float4 c0 = *reinterpret_cast<const float4 *>(&ctl->gC[kb][8 * j]);
                    const float4 c1 = *reinterpret_cast<const float4 *>(&ctl->gC[kb][8 * j + 4]);
                    pre[0] = p0.x; pre[1] = p0.y; pre[2] = p0.z; pre[3] = p0.w;
                    pre[4] = p1.x; pre[5] = p1.y; pre[6] = p1.z; pre[7] = p1.w;
                    gC[0] = c0.x; gC[1] = c0.y; gC[2] = c0.z; gC[3] = c0.w;
                    gC[4] = c1.x; gC[5] = c1.y; gC[6] = c1.z; gC[7] = c1.w;
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int t = 4 * tg + i;
                    const uint32_t off = (uint32_t)t * 128u + (uint32_t)(((cj ^ t) & 7) << 4);
                    const uint4 qv = *reinterpret_cast<const uint4 *>(qa + off);
                    const uint4 kv = *reinterpret_cast<const uint4 *>(ka + off);
                    const uint32_t *qw = &qv.x, *kw = &kv.x;
                    uint4 q2, kt, kh;
                    uint32_t *q2w = &q2.x, *ktw = &kt.x, *khw = &kh.x;
#pragma unroll
                    for (int e2 = 0; e2 < 4; ++e2) {
                        const float2 qf = unpack_bf16x2(qw[e2]), kf = unpack_bf16x2(kw[e2]);
                        const float ga = pre[2 * e2] * gam[i][2 * e2], gb = pre[2 * e2 + 1] * gam[i][2 * e2 + 1];
                        const float ia = rcp_nr(ga), ib = rcp_nr(gb);
                        q2w[e2] = pack_bf16x2(qf.x * ga, qf.y * gb);
                        ktw[e2] = pack_bf16x2(kf.x * ia, kf.y * ib);
                        khw[e2] = pack_bf16x2(kf.x * (ia * gC[2 * e2]), kf.y * (ib * gC[2 * e2 + 1]));
                    }
                    *reinterpret_cast<uint4 *>(qa + off) = q2;
                    *reinterpret_cast<uint4 *>(kxa + off) = kt;
                    *reinterpret_cast<uint4 *>(ka + off) = kh;
                }
            } else {
                float zs[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) zs[e] = 0.f;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int t = 4 * tg + i;
                    const uint32_t off = (uint32_t)t * 128u + (uint32_t)(((cj ^ t) & 7) << 4);
                    const uint4 qv = *reinterpret_cast<const uint4 *>(qa + off);
                    const uint4 kv = *reinterpret_cast<const uint4 *>(ka + off);
                    const uint32_t *qw = &qv.x, *kw = &kv.x;
                    uint4 pq, pk;
                    uint32_t *pqw = &pq.x, *pkw = &pk.x;
                    const bool valid = t < nvalid;
#pragma unroll
                    for (int e2 = 0; e2 < 4; ++e2) {
                        const float2 qf = unpack_bf16x2(qw[e2]), kf = unpack_bf16x2(kw[e2]);
                        const float k0 = valid ? elu_feature(kf.x) : 0.f, k1 = valid ? elu_feature(kf.y) : 0.f;
                        pqw[e2] = pack_bf16x2(elu_feature(qf.x), elu_feature(qf.y));
                        pkw[e2] = pack_bf16x2(k0, k1);
                        zs[2 * e2] += k0;
                        zs[2 * e2 + 1] += k1;
                    }
                    *reinterpret_cast<uint4 *>(qa + off) = pq;
                    *reinterpret_cast<uint4 *>(kxa + off) = pk;
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) ctl->tot[tg][8 * j + e] = zs[e];
                bar_named(1, 256);
                if (lt < DK) {   // chunk sum of phi(k) per key dim over the 16 token groups
                    float zsum = 0.f;
#pragma unroll
                    for (int g2 = 0; g2 < 16; ++g2) zsum += ctl->tot[g2][lt];
                    ctl->gC[kb][lt] = zsum;
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(&ctl->pfull[kb]);
        }
    } else {
        // ------------------------------------------------------------------ state group
        const int st = tid - 256;
        const bool leader = (st == 0);
        const int d = 32 * quad + lane;             // state row (key dim)
        const int tr = 16 * quad + (lane & 15);     // chunk row of M=64 accumulators
        const int hf = lane >> 4;
        constexpr uint32_t ID1 = idesc_bf16(64, L::N1, false, false);
        constexpr uint32_t ID2 = idesc_bf16(128, DVT, true, true);
        constexpr uint32_t ID3 = idesc_bf16(64, DVT, false, true);
        float S[DVT];
        float z = 0.f;
        {
            const float *src = p.S0 ? p.S0 + ((bh * DK + d) * p.dv + dvt * DVT) : nullptr;
#pragma unroll
            for (int jj = 0; jj < DVT; jj += 4) {
                float4 x = src ? *reinterpret_cast<const float4 *>(src + jj) : make_float4(0, 0, 0, 0);
                S[jj] = x.x; S[jj + 1] = x.y; S[jj + 2] = x.z; S[jj + 3] = x.w;
            }
            if (!kGLA && p.z0) z = p.z0[bh * DK + d];
        }
        // bf16 copy of S^T (and z^T) into rows 64.. of Kx buffer kb; ELU: zero rows 97..103
        auto write_state = [&](int kb) {
            uint8_t *kxa = tiles + L::KX + kb * L::KX_BYTES + (d >> 6) * L::KX_ACS;
            const int dc = d & 63;
#pragma unroll
            for (int jj = 0; jj < DVT; ++jj) *elem(kxa, 64 + jj, dc) = __float2bfloat16_rn(S[jj]);
            if (!kGLA) *elem(kxa, 96, dc) = __float2bfloat16_rn(z);
        };
        if (!kGLA) {
            for (int kb = 0; kb < 2; ++kb) {
                uint8_t *kxa = tiles + L::KX + kb * L::KX_BYTES + (d >> 6) * L::KX_ACS;
#pragma unroll
                for (int r = 97; r < 104; ++r) *elem(kxa, r, d & 63) = __float2bfloat16_rn(0.f);
            }
        }
        write_state(0);
        fence_proxy_async_smem();
        if (leader)
            for (int c = 0; c < NSTG && c < nchunks; ++c) load_chunk(c);
        for (int c = 0; c < nchunks; ++c) {
            const int kb = c & 1;
            const int t0 = c * C;
            const int nvalid = (int)min((int64_t)C, p.T - t0);
            if (leader) ctl->stopS = ctl->abort;
            bar_named(2, 128);
            if (ctl->stopS) break;
            if (!mbar_wait(&ctl->pfull[kb], (uint32_t)(c >> 1) & 1u)) ctl->abort = 1;
            uint8_t *sg = stg(c);
            const uint32_t qb = smem_u32(sg), kxb = tb + L::KX + kb * L::KX_BYTES;
            const uint32_t vb = qb + 2 * L::Q_BYTES;
            if (leader) {
                tc_fence_after_sync();
                const uint64_t dq = dk0(qb), dkx = dk0(kxb);
                const uint64_t du = kGLA ? dmn128_0(qb + L::Q_BYTES, C * 128) : dmn128_0(kxb, L::KX_ACS);
                const uint64_t dv = dmn64_0(vb);
#pragma unroll
                for (int kk = 0; kk < DK / 16; ++kk) {
                    umma_bf16(tmem + L::C_ACC, kstep_k(dq, C * 128, kk), kstep_k(dkx, L::KX_ACS, kk), ID1,
                              kk > 0);
                    if (kk < C / 16)
                        umma_bf16(tmem + L::C_DS, kstep_mn128(du, kk), kstep_mn64(dv, kk), ID2, kk > 0);
                }
                umma_commit(&ctl->m1_done);
            }
            if (!mbar_wait(&ctl->m1_done, (uint32_t)c & 1u)) ctl->abort = 1;
            tc_fence_after_sync();
            float den = 0.f;
            {   // P row tr, columns 32*hf..: causal mask -> bf16 tile; ELU row sums
                float x[32];
                tmem_ld16x2_32<32>(tq + L::C_ACC, x);
                float dI[16];
                if (!kGLA) tmem_ld16(tq + L::C_ACC + 96, dI);
                float ds[DVT];
                tmem_ld32(tq + L::C_DS, ds);
                tmem_wait_ld();
                float rs = 0.f;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    x[i] = (32 * hf + i <= tr) ? x[i] : 0.f;
                    rs += x[i];
                }
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    uint4 u;
                    u.x = pack_bf16x2(x[8 * cc + 0], x[8 * cc + 1]);
                    u.y = pack_bf16x2(x[8 * cc + 2], x[8 * cc + 3]);
                    u.z = pack_bf16x2(x[8 * cc + 4], x[8 * cc + 5]);
                    u.w = pack_bf16x2(x[8 * cc + 6], x[8 * cc + 7]);
                    const int chunk = 4 * hf + cc;
                    *reinterpret_cast<uint4 *>(tiles + L::PS + tr * 128 + (((chunk ^ tr) & 7) << 4)) = u;
                }
                if (!kGLA) {
                    rs += __shfl_xor_sync(0xffffffffu, rs, 16);
                    const float dz = __shfl_sync(0xffffffffu, dI[0], lane & 15);
                    den = dz + rs + p.eps;
                }
                // state update (row d), then its bf16 copy for the next chunk
                const float g = ctl->gC[kb][d];
                if (kGLA) {
#pragma unroll
                    for (int jj = 0; jj < DVT; ++jj) S[jj] = fmaf(g, S[jj], ds[jj]);
                } else {
#pragma unroll
                    for (int jj = 0; jj < DVT; ++jj) S[jj] += ds[jj];
                    z += g;
                }
                if (c + 1 < nchunks) write_state(kb ^ 1);
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            bar_named(2, 128);
            if (leader) {
                tc_fence_after_sync();
                const uint64_t dp = dk0(tb + L::PS), dv = dmn64_0(vb);
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    umma_bf16(tmem + L::C_ACC + 64, kstep_k(dp, C * 128, kk), kstep_mn64(dv, kk), ID3, 1u);
                umma_commit(&ctl->m3_done);
                umma_commit(&ctl->pempty[kb]);
            }
            if (!mbar_wait(&ctl->m3_done, (uint32_t)c & 1u)) ctl->abort = 1;
            if (leader && c + NSTG < nchunks && !ctl->abort) load_chunk(c + NSTG);   // its stage is free now
            tc_fence_after_sync();
            {
                float o[16];
                tmem_ld16x2_16<16>(tq + L::C_ACC + 64, o);
                tmem_wait_ld();
                if (tr < nvalid) {
                    if (!kGLA) {
                        const float inv = 1.f / den;
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj) o[jj] *= inv;
                    }
                    __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(p.o) +
                                         ((b * p.T + t0 + tr) * p.H + h) * p.dv + dvt * DVT + 16 * hf;
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
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
        }
        if (!ctl->abort) {
            if (p.S_out) {
                float *dst = p.S_out + ((bh * DK + d) * p.dv + dvt * DVT);
#pragma unroll
                for (int jj = 0; jj < DVT; jj += 4)
                    *reinterpret_cast<float4 *>(dst + jj) = make_float4(S[jj], S[jj + 1], S[jj + 2], S[jj + 3]);
            }
            if (!kGLA && p.z_out && dvt == 0) p.z_out[bh * DK + d] = z;
        }
    }
    if (tid == 256 && ctl->abort) {   // let copies still in flight land before exit
        for (int s = 0; s < NSTG; ++s) (void)mbar_try_wait(&ctl->full[s], 0);
        for (int s = 0; s < NSTG; ++s) (void)mbar_try_wait(&ctl->full[s], 1);
    }
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, L::TMEM_COLS);
}

}  // namespace ck
}  // namespace la
