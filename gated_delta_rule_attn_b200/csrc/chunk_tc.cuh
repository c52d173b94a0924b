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
//     Qt = Q o gamma,  Kt = K / gamma
//     P = (Qt Kt^T) o M,  O = Qt S0 + P V,  S <- diag(gamma_C) (S0 + Kt^T V)
//   Gated delta rule (page "线性注意力与 SSM", GDN box): gamma_t = prod alpha,
//     Gamma_ti = gamma_t / gamma_i (computed as exp2 of log2 differences <= 0),
//     A = diag(beta) (K K^T o Gamma o strict-lower), T = (I + A)^-1,
//     U = T diag(beta gamma) K,                          (state independent)
//     W = T diag(beta) V - U S0,  O = diag(gamma) Q S0 + P W,  P = (Q K^T) o Gamma o M,
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
#include <atomic>
#include <string>
#include <utility>

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
    // sequence-parallel ELU+1 / GLA (nseg > 1): segment j of every (batch, head)
    // starts from S0 folded through the range summaries in `agg` of segments < j
    int nseg = 1, nparts = 1, seg_chunks = 0;
    const float *agg = nullptr;
    // packed sequences (tensors [1,T,H,*], sequence b = tokens [cu[b], cu[b+1]));
    // nullptr = dense [B,T,H,*].  max_seqlen bounds every sequence's length (the
    // launch sets it to T for the dense layout).
    const int64_t *cu_seqlens = nullptr;
    int64_t max_seqlen = 0;
    // GLA: per-sequence flags in the workspace.  A sequence with a chunk whose
    // gate product leaves the chunked form's range gets seq_flags[b*H + h] =
    // call_id (an ID unique to the call, so the flags need no clearing); the
    // chunked kernels then leave its final state unwritten and the recurrent
    // kernel recomputes the sequence exactly.
    uint32_t *seq_flags = nullptr;
    uint32_t call_id = 0;
};

// Smallest per-key-dim gate product over one 64-token chunk that GLA's chunked
// form handles: it scales keys by 1 / (the gate product from the chunk's start),
// which for products >= 2^-120 stays a normal fp32 and bf16 number (as does
// q times the product).
constexpr float kGlaMinChunkGate = 0x1p-120f;

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
    CUtensorMap kc;   // KDA: the prep kernel's Kc = K o Gamma_C / Gamma
};

__device__ __forceinline__ uint32_t align1k(uint32_t x) { return (x + 1023u) & ~1023u; }

// Bytes of a [rows] x DK tile as KA atom columns.
constexpr uint32_t tile_bytes(int rows) { return (uint32_t)rows * 128u * KA; }

__device__ __forceinline__ void bar_named(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

}  // namespace ck
}  // namespace la

#include "chunk_gdn.cuh"
#include "chunk_kda.cuh"
#include "chunk_ge.cuh"
#include "chunk_agg.cuh"

namespace la {


// Sequence parallelism for ELU+1 and GLA: when the (batch, head, value slab) CTAs
// fill only a fraction of the SMs, every sequence is cut into `nseg` segments of
// `seg_chunks` chunks that run side by side; a first pass summarises each
// segment but the last, in `nparts` chunk ranges per segment, as the affine map
// its tokens apply to the state (chunk_agg.cuh).
struct SegPlan {
    int nseg = 1, nparts = 1, seg_chunks = 0;
};

// Value columns per CTA of the GLA / ELU chunked kernel: 64 when dv allows (one
// CTA covers twice the columns for the same MMA instruction count and the same
// feature-map or gate work, and the freed CTAs go to more segments), else 32.
inline int ge_slab(int rule, int64_t dv) { (void)rule; return dv % 64 == 0 ? 64 : ck::DVT; }

inline SegPlan seg_plan(int rule, int64_t B, int64_t T, int64_t H, int64_t dv) {
    SegPlan sp;
    const int64_t nch = (T + ck::C - 1) / ck::C;
    sp.seg_chunks = (int)nch;
    if ((rule != kRuleELU && rule != kRuleGLA) || nch < 16 || dv % ck::DVT != 0) return sp;
    const int64_t sms = sm_count(), ctas = B * H * (dv / ge_slab(rule, dv));
    const int64_t nseg = std::min<int64_t>(sms / ctas, nch / 8);
    if (nseg < 2) return sp;
    sp.seg_chunks = (int)((nch + nseg - 1) / nseg);
    sp.nseg = (int)((nch + sp.seg_chunks - 1) / sp.seg_chunks);   // no empty segment
    if (sp.nseg < 2) return SegPlan{1, 1, (int)nch};
    const int64_t units = B * H * (sp.nseg - 1);
    sp.nparts = (int)std::max<int64_t>(1, std::min<int64_t>(sms / units, sp.seg_chunks / 4));
    return sp;
}

// CTAs of `kernel` that can be resident on one SM at once, from its registers,
// its shared memory and the TMEM columns each CTA allocates.  (The runtime's
// occupancy query returns 1 for these tcgen05 kernels, although more fit.)
inline int resident_per_sm(const void *kernel, int threads, int dyn_smem, int tmem_cols) {
    int dev = 0, regs_sm = 65536, smem_sm = 233472, smem_res = 1024, thr_sm = 2048;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev);
    cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    cudaDeviceGetAttribute(&smem_res, cudaDevAttrReservedSharedMemoryPerBlock, dev);
    cudaDeviceGetAttribute(&thr_sm, cudaDevAttrMaxThreadsPerMultiProcessor, dev);
    cudaFuncAttributes fa{};
    if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess) return 1;
    const int warps = (threads + 31) / 32;
    const int regs_warp = (fa.numRegs * 32 + 255) / 256 * 256;   // allocated per warp in units of 256
    int n = regs_warp > 0 ? regs_sm / (regs_warp * warps) : 1;
    n = std::min(n, smem_sm / (dyn_smem + (int)fa.sharedSizeBytes + smem_res));
    n = std::min(n, thr_sm / threads);
    n = std::min(n, 512 / tmem_cols);
    return std::max(n, 1);
}

// KDA workspace: the per-chunk items (T diag(beta), P and -U images, Gamma_C),
// then the Qp and Kc tensors [B,Ls,H,128] bf16, each at a 256-byte aligned offset
// (Ls = T dense; 64 ceil(max_seqlen / 64) for packed sequences, one row block
// per sequence).
struct KdaWorkspace {
    size_t items, qp, kc, total;
};
inline KdaWorkspace kda_workspace(int64_t B, int64_t T, int64_t H) {
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    KdaWorkspace w{};
    w.items = 0;
    const size_t tensor = up((size_t)(B * T * H) * ck::DK * 2);
    w.qp = up((size_t)(B * H * ((T + ck::C - 1) / ck::C)) * ck::kda::ITEM_BYTES);
    w.kc = w.qp + tensor;
    w.total = w.kc + tensor;
    return w;
}

// Segment summaries of sequence-parallel ELU+1 / GLA (none when packed).
inline size_t chunk_agg_bytes(int rule, int64_t B, int64_t T, int64_t H, int64_t dv, bool packed) {
    if (packed || (rule != kRuleELU && rule != kRuleGLA)) return 0;
    const SegPlan sp = seg_plan(rule, B, T, H, dv);
    if (sp.nseg < 2) return 0;
    return (size_t)(B * H * (sp.nseg - 1) * sp.nparts) * (size_t)(ck::DK * dv + ck::DK) * sizeof(float);
}
// GLA's per-sequence flags (uint32 per (batch, head)), after the summaries.
inline size_t gla_flag_bytes(int64_t B, int64_t H) { return ((size_t)(B * H) * 4 + 255) & ~(size_t)255; }

// Device workspace the chunked path needs: the gated delta rule keeps the
// per-chunk operand images of T diag(beta), P and -U (32 KB per (batch, head, chunk)); KDA
// its prep kernel's items and scaled q/k tensors; sequence-parallel ELU+1 and GLA the range
// summaries of their first pass; GLA its per-sequence range flags.  `packed`: the
// sequences are packed on one token axis with lengths up to max_seqlen (no
// sequence-parallel pass then).
inline size_t chunk_workspace_bytes(int rule, int64_t B, int64_t T, int64_t H, int64_t dv,
                                    bool packed = false, int64_t max_seqlen = 0) {
    if (T <= 0) return 0;
    const int64_t L = packed ? max_seqlen : T;
    if (rule == kRuleGDN) return (size_t)(B * H * ((L + ck::C - 1) / ck::C)) * ck::gdn::ITEM_BYTES;
    if (rule == kRuleKDA) return kda_workspace(B, packed ? (L + ck::C - 1) / ck::C * ck::C : T, H).total;
    return chunk_agg_bytes(rule, B, T, H, dv, packed) + (rule == kRuleGLA ? gla_flag_bytes(B, H) : 0);
}

// Launch `kern` as a programmatic dependent of the kernel before it in `st`
// (when `dependent`): it may be scheduled once every CTA of that kernel has
// signalled, and it waits (griddepcontrol.wait) before reading that kernel's
// results.
template <typename... Params, typename... Args>
cudaError_t launch_maybe_dependent(void (*kern)(Params...), unsigned grid, unsigned block, int smem,
                                   cudaStream_t st, bool dependent, Args &&...args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = dependent ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// GLA / ELU: one CTA per (batch, head, value slab, segment); a programmatic
// dependent of the summary pass when there is one.
template <int RULE, int DVS>
cudaError_t launch_ge(const ck::Maps &m, const ChunkParams &p, cudaStream_t st) {
    using L = ck::GE<RULE, DVS>;
    const int smem = (int)((sizeof(ck::GECtl) + 1023) / 1024 * 1024) + 1024 + (int)L::END;
    cudaError_t e = allow_smem((const void *)ck::chunk_ge_kernel<RULE, DVS>, smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)(p.B * p.H * (p.dv / DVS) * p.nseg);
    e = launch_maybe_dependent(ck::chunk_ge_kernel<RULE, DVS>, grid, (unsigned)L::NTHREADS, smem, st, p.nseg > 1, m, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// First pass of sequence-parallel ELU+1 / GLA.
template <int RULE, int DV>
cudaError_t launch_agg(const ck::Maps &m, const AggParams &a, cudaStream_t st) {
    using L = ck::AG<RULE, DV>;
    const int smem = (int)((sizeof(ck::AGCtl) + 1023) / 1024 * 1024) + 1024 + (int)L::END;
    cudaError_t e = allow_smem((const void *)ck::chunk_agg_kernel<RULE, DV>, smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)(a.B * a.H * (a.nseg - 1) * a.nparts);
    ck::chunk_agg_kernel<RULE, DV><<<grid, 288, smem, st>>>(m, a);
    return cudaGetLastError();
}
template <int RULE>
cudaError_t launch_agg_dv(const ck::Maps &m, const AggParams &a, cudaStream_t st) {
    return a.dv == 32 ? launch_agg<RULE, 32>(m, a, st)
         : a.dv == 64 ? launch_agg<RULE, 64>(m, a, st) : launch_agg<RULE, 128>(m, a, st);
}

// The recurrent kernel over the GLA sequences flagged in p.seq_flags for this call.
inline cudaError_t launch_gla_recompute(const ChunkParams &p, cudaStream_t st) {
    RecurrentParams r{};
    r.B = p.B; r.T = p.T; r.H = p.H;
    r.q = p.q; r.k = p.k; r.v = p.v; r.g = p.g; r.beta = nullptr;
    r.S_in = p.S0; r.S_out = p.S_out; r.z_in = nullptr; r.z_out = nullptr;
    r.o = p.o; r.eps = p.eps;
    r.cu_seqlens = p.cu_seqlens; r.max_seqlen = p.max_seqlen;
    r.seq_flags = p.seq_flags; r.call_id = p.call_id;
    // a programmatic dependent launch: scheduled as the chunked kernel's CTAs
    // finish instead of after a full kernel boundary (the kernel waits for that
    // grid's completion before it reads the flags)
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(p.B * p.H));
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    switch (p.dv) {
        case 32: return cudaLaunchKernelEx(&cfg, recurrent_kernel<kRuleGLA, 128, 32, __nv_bfloat16>, r);
        case 64: return cudaLaunchKernelEx(&cfg, recurrent_kernel<kRuleGLA, 128, 64, __nv_bfloat16>, r);
        default: return cudaLaunchKernelEx(&cfg, recurrent_kernel<kRuleGLA, 128, 128, __nv_bfloat16>, r);
    }
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
    const bool packed = p.cu_seqlens != nullptr;
    const int64_t MB = packed ? 1 : p.B;   // outer extent of the 4-D tensor maps
    bool okm = make_map_4d(&m.q, p.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, MB, p.T, p.H, DK, 64, C,
                           CU_TENSOR_MAP_SWIZZLE_128B) &&
               make_map_4d(&m.k, p.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, MB, p.T, p.H, DK, 64, C,
                           CU_TENSOR_MAP_SWIZZLE_128B) &&
               make_map_4d(&m.v, p.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, MB, p.T, p.H, p.dv, DVT, C,
                           CU_TENSOR_MAP_SWIZZLE_64B);
    if (okm && rule == kRuleGLA)
        okm = make_map_4d(&m.g, p.g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, MB, p.T, p.H, DK, DK, C,
                          CU_TENSOR_MAP_SWIZZLE_NONE);
    ChunkParams pq = p;
    if (!packed) pq.max_seqlen = p.T;
    const int64_t Lmax = pq.max_seqlen;
    if (!okm) {
        *err = "cuTensorMapEncodeTiled failed (driver entry point missing or bad layout)";
        return 4;
    }
    const unsigned grid = (unsigned)(p.B * p.H * (p.dv / DVT));
    cudaError_t e;
    if (rule == kRuleKDA) {
        const int nch = (int)((Lmax + C - 1) / C);
        const int64_t Ls = packed ? (int64_t)nch * C : p.T;
        const KdaWorkspace kw = kda_workspace(p.B, Ls, p.H);
        if (!ws || ws_bytes < kw.total || (reinterpret_cast<uintptr_t>(ws) & 15u)) {
            *err = "KDA needs a 16-byte aligned workspace of la_fwd_workspace_size() bytes";
            return 8;
        }
        uint8_t *w8 = static_cast<uint8_t *>(ws);
        KdaPrepParams kp{};
        kp.B = p.B; kp.T = p.T; kp.H = p.H;
        kp.nchunks = nch;
        kp.Ls = Ls;
        kp.cu_seqlens = p.cu_seqlens;
        kp.max_seqlen = Lmax;
        kp.q = static_cast<const __nv_bfloat16 *>(p.q);
        kp.k = static_cast<const __nv_bfloat16 *>(p.k);
        kp.alpha = p.g; kp.beta = p.beta;
        kp.items = w8 + kw.items;
        kp.qp = reinterpret_cast<__nv_bfloat16 *>(w8 + kw.qp);
        kp.kc = reinterpret_cast<__nv_bfloat16 *>(w8 + kw.kc);
        Maps mk = m;
        if (!make_map_4d(&mk.q, kp.qp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.B, Ls, p.H, DK, 64, C,
                         CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_map_4d(&mk.kc, kp.kc, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.B, Ls, p.H, DK, 64, C,
                         CU_TENSOR_MAP_SWIZZLE_128B)) {
            *err = "cuTensorMapEncodeTiled failed (driver entry point missing or bad layout)";
            return 4;
        }
        const int64_t items = p.B * p.H * (int64_t)kp.nchunks;
        const int psmem = (int)((sizeof(KCtl) + 1023) / 1024 * 1024) + 1024 + (int)kda::P_END;
        e = allow_smem((const void *)kda_prep_kernel, psmem);
        const int per_sm = resident_per_sm((const void *)kda_prep_kernel, kda::PREP_THREADS, psmem, 256);
        const unsigned pgrid = (unsigned)std::min<int64_t>(items, (int64_t)sm_count() * per_sm);
        if (e == cudaSuccess) kda_prep_kernel<<<pgrid, kda::PREP_THREADS, psmem, st>>>(kp);
        const int smem = (int)((sizeof(gdn::MCtl) + 1023) / 1024 * 1024) + 1024 + (int)gdn::ML<true>::TEND;
        if (e == cudaSuccess) e = allow_smem((const void *)gdn_main_kernel<true>, smem);
        if (e == cudaSuccess)
            e = launch_maybe_dependent(gdn_main_kernel<true>, grid, (unsigned)gdn::NTHREADS, smem, st, true, mk, pq,
                                       (const uint8_t *)(w8 + kw.items));
    } else if (rule == kRuleGDN) {
        const size_t need = chunk_workspace_bytes(rule, p.B, p.T, p.H, p.dv, packed, Lmax);
        if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 15u)) {
            *err = "the gated delta rule needs a 16-byte aligned workspace of la_fwd_workspace_size() bytes";
            return 8;
        }
        GdnPrepParams pp{};
        pp.B = p.B; pp.T = p.T; pp.H = p.H;
        pp.nchunks = (int)((Lmax + C - 1) / C);
        pp.alpha = p.g; pp.beta = p.beta;
        pp.cu_seqlens = p.cu_seqlens; pp.max_seqlen = Lmax;
        pp.ws = static_cast<uint8_t *>(ws);
        const int64_t items = p.B * p.H * (int64_t)pp.nchunks;
        // tiles (1 KB aligned from a base that may sit anywhere), then the control block
        const int psmem = 1023 + (int)gdn::P_END + (int)((sizeof(gdn::PCtl) + 15) / 16 * 16);
        e = allow_smem((const void *)gdn_prep_kernel, psmem);
        // one wave of resident CTAs walks all items (a second, partial wave
        // would double the time)
        const int per_sm =
            resident_per_sm((const void *)gdn_prep_kernel, gdn::PREP_THREADS, psmem, (int)gdn::PREP_TMEM_COLS);
        const unsigned pgrid = (unsigned)std::min<int64_t>(items, (int64_t)sm_count() * per_sm);
        if (e == cudaSuccess && items > 0) gdn_prep_kernel<<<pgrid, gdn::PREP_THREADS, psmem, st>>>(m.q, m.k, pp);
        const int smem = (int)((sizeof(gdn::MCtl) + 1023) / 1024 * 1024) + 1024 + (int)gdn::ML<false>::TEND;
        if (e == cudaSuccess) e = allow_smem((const void *)gdn_main_kernel<false>, smem);
        if (e == cudaSuccess)
            e = launch_maybe_dependent(gdn_main_kernel<false>, grid, (unsigned)gdn::NTHREADS, smem, st, items > 0, m,
                                       pq, static_cast<const uint8_t *>(ws));
    } else {
        // packed sequences walk each sequence in one pass (no segments)
        const SegPlan sp = packed ? SegPlan{1, 1, (int)((Lmax + C - 1) / C)} : seg_plan(rule, p.B, p.T, p.H, p.dv);
        ChunkParams q = pq;
        const size_t need = chunk_workspace_bytes(rule, p.B, p.T, p.H, p.dv, packed, Lmax);
        if (need && (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 15u))) {
            *err = rule == kRuleGLA ? "GLA needs a 16-byte aligned workspace of la_fwd_workspace_size() bytes"
                                    : "sequence-parallel ELU+1 needs a 16-byte aligned workspace of "
                                      "la_fwd_workspace_size() bytes";
            return 8;
        }
        if (rule == kRuleGLA) {
            // flags after the summaries; a call ID that no earlier call used
            static std::atomic<uint32_t> next_call{0};
            uint32_t id = next_call.fetch_add(1) + 1u;
            if (id == 0u) id = next_call.fetch_add(1) + 1u;
            q.seq_flags = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(ws) +
                                                       chunk_agg_bytes(rule, p.B, p.T, p.H, p.dv, packed));
            q.call_id = id;
        }
        if (sp.nseg > 1) {
            AggParams a{};
            a.B = p.B; a.T = p.T; a.H = p.H; a.dv = p.dv;
            a.agg = static_cast<float *>(ws);
            a.nseg = sp.nseg; a.nparts = sp.nparts; a.seg_chunks = sp.seg_chunks;
            a.seq_flags = q.seq_flags; a.call_id = q.call_id;
            e = rule == kRuleGLA ? launch_agg_dv<kRuleGLA>(m, a, st) : launch_agg_dv<kRuleELU>(m, a, st);
            if (e != cudaSuccess) {
                *err = std::string("chunk kernel launch: ") + cudaGetErrorString(e);
                return 4;
            }
            q.agg = a.agg;
        }
        q.nseg = sp.nseg; q.nparts = sp.nparts; q.seg_chunks = sp.seg_chunks;
        if (ge_slab(rule, p.dv) == 64) {
            // 64-column V tiles with the 128-byte swizzle
            Maps m64 = m;
            if (!make_map_4d(&m64.v, p.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, MB, p.T, p.H, p.dv, 64, C,
                             CU_TENSOR_MAP_SWIZZLE_128B)) {
                *err = "cuTensorMapEncodeTiled failed (driver entry point missing or bad layout)";
                return 4;
            }
            e = rule == kRuleGLA ? launch_ge<kRuleGLA, 64>(m64, q, st) : launch_ge<kRuleELU, 64>(m64, q, st);
        } else {
            e = rule == kRuleGLA ? launch_ge<kRuleGLA, DVT>(m, q, st) : launch_ge<kRuleELU, DVT>(m, q, st);
        }
        // GLA sequences with a chunk out of the chunked form's range: recomputed
        // exactly by the per-token recurrent kernel from S0 (every other CTA exits
        // at once)
        if (e == cudaSuccess && rule == kRuleGLA) e = launch_gla_recompute(q, st);
    }
    if (e != cudaSuccess) {
        *err = std::string("chunk kernel launch: ") + cudaGetErrorString(e);
        return 4;
    }
    return 0;
}

}  // namespace la
