// recurrent.cuh — per-token recurrent kernel on CUDA cores (fp32 arithmetic).
//
// One CTA owns one (batch, head) state S (dk x dv fp32) in registers for the
// whole call and walks the tokens in order, applying the update rule and
// reading the output after the update of the same token:
//   ELU+1  S += phi(k) v^T, z += phi(k), o = S^T phi(q) / (phi(q).z + eps)
//          (page "Linear / RNN 路线", §2.1; eps as in page "状态空间与线性注意力",
//          section 线性注意力)
//   GLA    S = diag(g) S + k v^T, o = S^T q  (page "Linear / RNN 路线", §2.2)
//   GDN    r = S^T k, p = S^T q, u = v - alpha r,
//          S = alpha S + beta k u^T  (= alpha (I - beta k k^T) S + beta k v^T,
//          page "线性注意力与 SSM", GDN box, dk x dv orientation),
//          o = S^T q = alpha p + beta (q.k) u.
//   KDA    Sbar = Diag(alpha) S (alpha per key channel), r = Sbar^T k,
//          p = Sbar^T q, u = v - r, S = Sbar + beta k u^T, o = p + beta (q.k) u
//          (page "状态空间与线性注意力", section KDA：逐通道遗忘与误差写入).
//
// Used for the decode step (T = 1, state in place: one streaming pass over S
// with 128-bit loads and stores, warp-shuffle dot products and a cross-warp
// reduction in shared memory) and for prefill with fp32 inputs (T tokens with
// the state held in registers; exact fp32 FMA, no tensor cores).
//
// Thread layout: 256 threads; thread (rg, cg) holds rows [rg*RPT, rg*RPT+RPT)
// and columns [4*cg, 4*cg+4) of S as float4s, CG = dv/4, RG = 256/CG,
// RPT = dk/RG.  A warp covers whole 128-byte-aligned row segments, so every
// S load/store is fully coalesced.
#pragma once

#include "device.cuh"

namespace la {

enum : int { kRuleELU = 0, kRuleGLA = 1, kRuleGDN = 2, kRuleKDA = 3 };

struct RecurrentParams {
    int64_t B, T, H;
    const void *q, *k, *v;      // [B,T,H,dk] / [B,T,H,dv]
    const float *g;             // GLA [B,T,H,dk]; GDN alpha [B,T,H]
    const float *beta;          // GDN [B,T,H]
    const float *S_in;          // [B,H,dk,dv] or null (zeros)
    float *S_out;               // [B,H,dk,dv] or null; may equal S_in
    const float *z_in;          // ELU [B,H,dk] or null
    float *z_out;               // ELU [B,H,dk] or null; may equal z_in
    void *o;                    // [B,T,H,dv]
    float eps;
    // packed sequences: sequence b is tokens [cu_seqlens[b], cu_seqlens[b+1]) of
    // one token axis of T tokens (tensors [1,T,H,*]); nullptr = dense layout
    const int64_t *cu_seqlens = nullptr;
    int64_t max_seqlen = 0;
    // set: only the sequences (b, h) with seq_flags[b*H + h] == call_id run (the
    // exact recomputation of GLA sequences the chunked kernels could not take)
    const uint32_t *seq_flags = nullptr;
    uint32_t call_id = 0;
};

__device__ __forceinline__ float elu_feature_precise(float x) {
    return x > 0.f ? x + 1.f : expf(x);
}

template <int RULE, int DK, int DV, typename TIO>
__global__ void __launch_bounds__(256, 2) recurrent_kernel(const RecurrentParams p) {
    constexpr int NT = 256;
    constexpr int CG = DV / 4;
    constexpr int RG = NT / CG;
    constexpr int RPT = DK / RG;
    static_assert(RPT >= 1 && RG * RPT == DK, "unsupported dk/dv");

    __shared__ float s_q[DK], s_k[DK], s_g[DK], s_v[DV];
    __shared__ float s_z[DK];
    __shared__ float4 s_red[2][RG][CG];
    __shared__ float s_vec[2][DV];
    __shared__ float s_scal[4];
    __shared__ float s_warp[NT / 32][2];

    const int tid = threadIdx.x;
    const int cg = tid % CG, rg = tid / CG;
    const int64_t bh = blockIdx.x;
    if (p.seq_flags) {
        // launched as a programmatic dependent of the chunked kernel: wait for it
        // to finish (and its writes to be visible) before reading its flags
        asm volatile("griddepcontrol.wait;" ::: "memory");
        if (p.seq_flags[bh] != p.call_id) return;   // uniform over the CTA
    }
    const int64_t b = bh / p.H, h = bh % p.H;
    const int64_t H = p.H, T = p.T;

    // State slab -> registers (streaming loads; issued before anything else).
    float4 s[RPT];
    const int64_t sbase = bh * (int64_t)DK * DV;
    if (p.S_in) {
        const float4 *src = reinterpret_cast<const float4 *>(p.S_in + sbase);
#pragma unroll
        for (int r = 0; r < RPT; ++r) s[r] = __ldcs(src + (int64_t)(rg * RPT + r) * CG + cg);
    } else {
#pragma unroll
        for (int r = 0; r < RPT; ++r) s[r] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (RULE == kRuleELU && tid < DK) s_z[tid] = p.z_in ? p.z_in[bh * DK + tid] : 0.f;

    const TIO *q = static_cast<const TIO *>(p.q);
    const TIO *k = static_cast<const TIO *>(p.k);
    const TIO *v = static_cast<const TIO *>(p.v);
    TIO *o = static_cast<TIO *>(p.o);

    const SeqSpan sq = seq_span(p.cu_seqlens, b, T, p.max_seqlen, tid == 0 && h == 0);
    for (int64_t t = 0; t < sq.len; ++t) {
        const int64_t row = (sq.row0 + t) * H + h;  // token row index into [B,T,H,*] / [1,T,H,*]
        if (tid < DK) {
            float qx = to_f32(q[row * DK + tid]);
            float kx = to_f32(k[row * DK + tid]);
            if (RULE == kRuleELU) {
                qx = elu_feature_precise(qx);
                kx = elu_feature_precise(kx);
            }
            s_q[tid] = qx;
            s_k[tid] = kx;
            if (RULE == kRuleGLA || RULE == kRuleKDA) s_g[tid] = p.g[row * DK + tid];
        }
        if (tid < DV) s_v[tid] = to_f32(v[row * DV + tid]);
        if (RULE == kRuleGDN && tid == 0) {
            s_scal[0] = p.g[row];
            s_scal[1] = p.beta[row];
        }
        if (RULE == kRuleKDA && tid == 0) {
            s_scal[0] = 1.f;   // the decay is per key row (s_g), applied below
            s_scal[1] = p.beta[row];
        }
        __syncthreads();

        if constexpr (RULE == kRuleGDN || RULE == kRuleKDA) {
            // r = S^T k and p = S^T q over this thread's rows, then across rows.
            // KDA reads the decayed state Sbar = Diag(alpha) S: r = S^T (alpha o k),
            // p = S^T (alpha o q) (one pass, no decayed copy).
            float4 pr = make_float4(0.f, 0.f, 0.f, 0.f), pp = pr;
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const float ad = RULE == kRuleKDA ? s_g[rg * RPT + r] : 1.f;
                const float kd = ad * s_k[rg * RPT + r], qd = ad * s_q[rg * RPT + r];
                pr.x = fmaf(kd, s[r].x, pr.x); pr.y = fmaf(kd, s[r].y, pr.y);
                pr.z = fmaf(kd, s[r].z, pr.z); pr.w = fmaf(kd, s[r].w, pr.w);
                pp.x = fmaf(qd, s[r].x, pp.x); pp.y = fmaf(qd, s[r].y, pp.y);
                pp.z = fmaf(qd, s[r].z, pp.z); pp.w = fmaf(qd, s[r].w, pp.w);
            }
            s_red[0][rg][cg] = pr;
            s_red[1][rg][cg] = pp;
            // q.k (warp-shuffle dot product within each warp, then across warps)
            float qk = 0.f;
            if (tid < DK) qk = s_q[tid] * s_k[tid];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) qk += __shfl_xor_sync(0xffffffffu, qk, off);
            if ((tid & 31) == 0) s_warp[tid >> 5][0] = qk;
            __syncthreads();
            if (tid < DV) {
                const int c = tid >> 2, e = tid & 3;
                float ar = 0.f, ap = 0.f;
#pragma unroll 8
                for (int g2 = 0; g2 < RG; ++g2) {
                    ar += reinterpret_cast<const float *>(&s_red[0][g2][c])[e];
                    ap += reinterpret_cast<const float *>(&s_red[1][g2][c])[e];
                }
                s_vec[0][tid] = ar;
                s_vec[1][tid] = ap;
            }
            if (tid == 0) {
                float a = 0.f;
#pragma unroll
                for (int w = 0; w < NT / 32; ++w) a += s_warp[w][0];
                s_scal[2] = a;
            }
            __syncthreads();
            const float al = s_scal[0], be = s_scal[1];
            float u[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) u[e] = s_v[4 * cg + e] - al * s_vec[0][4 * cg + e];
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const float bk = be * s_k[rg * RPT + r];
                const float ar = RULE == kRuleKDA ? s_g[rg * RPT + r] : al;   // decay of row d
                s[r].x = fmaf(ar, s[r].x, bk * u[0]);
                s[r].y = fmaf(ar, s[r].y, bk * u[1]);
                s[r].z = fmaf(ar, s[r].z, bk * u[2]);
                s[r].w = fmaf(ar, s[r].w, bk * u[3]);
            }
            if (tid < DV) {
                const float uj = s_v[tid] - al * s_vec[0][tid];
                const float oj = fmaf(al, s_vec[1][tid], be * s_scal[2] * uj);
                o[row * DV + tid] = from_f32<TIO>(oj);
            }
        } else {
            // ELU / GLA: update rows, then o = S^T q' over rows.
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            const float4 vv = make_float4(s_v[4 * cg], s_v[4 * cg + 1], s_v[4 * cg + 2],
                                          s_v[4 * cg + 3]);
#pragma unroll
            for (int r = 0; r < RPT; ++r) {
                const int d = rg * RPT + r;
                const float kd = s_k[d], qd = s_q[d];
                if constexpr (RULE == kRuleGLA) {
                    const float gd = s_g[d];
                    s[r].x = fmaf(gd, s[r].x, kd * vv.x); s[r].y = fmaf(gd, s[r].y, kd * vv.y);
                    s[r].z = fmaf(gd, s[r].z, kd * vv.z); s[r].w = fmaf(gd, s[r].w, kd * vv.w);
                } else {
                    s[r].x = fmaf(kd, vv.x, s[r].x); s[r].y = fmaf(kd, vv.y, s[r].y);
                    s[r].z = fmaf(kd, vv.z, s[r].z); s[r].w = fmaf(kd, vv.w, s[r].w);
                }
                acc.x = fmaf(qd, s[r].x, acc.x); acc.y = fmaf(qd, s[r].y, acc.y);
                acc.z = fmaf(qd, s[r].z, acc.z); acc.w = fmaf(qd, s[r].w, acc.w);
            }
            s_red[0][rg][cg] = acc;
            float den = 0.f;
            if (RULE == kRuleELU) {
                if (tid < DK) {
                    const float zn = s_z[tid] + s_k[tid];
                    s_z[tid] = zn;
                    den = s_q[tid] * zn;
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
                if ((tid & 31) == 0) s_warp[tid >> 5][0] = den;
            }
            __syncthreads();
            if (tid < DV) {
                const int c = tid >> 2, e = tid & 3;
                float a = 0.f;
#pragma unroll 8
                for (int g2 = 0; g2 < RG; ++g2)
                    a += reinterpret_cast<const float *>(&s_red[0][g2][c])[e];
                if (RULE == kRuleELU) {
                    float dsum = 0.f;
#pragma unroll
                    for (int w = 0; w < NT / 32; ++w) dsum += s_warp[w][0];
                    a = a / (dsum + p.eps);
                }
                o[row * DV + tid] = from_f32<TIO>(a);
            }
        }
        __syncthreads();  // shared inputs of this token are reused by the next one
    }

    if (p.S_out) {
        float4 *dst = reinterpret_cast<float4 *>(p.S_out + sbase);
#pragma unroll
        for (int r = 0; r < RPT; ++r) __stcs(dst + (int64_t)(rg * RPT + r) * CG + cg, s[r]);
    }
    if (RULE == kRuleELU && p.z_out && tid < DK) p.z_out[bh * DK + tid] = s_z[tid];
}

}  // namespace la
