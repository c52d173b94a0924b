// la.cu — the C ABI declared in include/la.h: argument validation on the host,
// kernel selection, the host-buffer entry point and the device error word.
//
// Kernel selection for la_fwd:
//   bf16, dk = 128           -> chunked tensor-core kernels (chunk_tc.cuh)
//   fp32, or bf16 with dk < 128 -> per-token recurrent kernel (recurrent.cuh)
// la_step always uses the recurrent kernel with T = 1 and the state in place.
// With out_norm set, a second pass normalises each (token, head) row of o
// (out_norm.cuh).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstddef>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "la.h"
#include "la_testing.h"
#include "device.cuh"
#include "recurrent.cuh"
#include "chunk_tc.cuh"
#include "out_norm.cuh"

namespace {

thread_local std::string g_last_error;

la_status fail(la_status s, const std::string &msg) {
    g_last_error = msg;
    return s;
}

la_status ok() {
    g_last_error.clear();
    return LA_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool supported_dim(int64_t d) { return d == 32 || d == 64 || d == 128; }

size_t elem_size(la_dtype t) { return t == LA_BF16 ? 2 : 4; }

struct Shape {
    int64_t B, T, H, dk, dv;
};

la_status validate_common(la_rule rule, la_dtype dtype, const Shape &s) {
    if (rule != LA_RULE_ELU && rule != LA_RULE_GLA && rule != LA_RULE_GDN && rule != LA_RULE_KDA)
        return fail(LA_ERR_INVALID_ARG, "rule must be LA_RULE_ELU, LA_RULE_GLA, LA_RULE_GDN or LA_RULE_KDA");
    if (dtype != LA_F32 && dtype != LA_BF16)
        return fail(LA_ERR_INVALID_ARG, "dtype must be LA_F32 or LA_BF16");
    if (s.B < 1 || s.H < 1 || s.T < 0)
        return fail(LA_ERR_INVALID_ARG, "need B >= 1, H >= 1, T >= 0");
    if (!supported_dim(s.dk) || !supported_dim(s.dv))
        return fail(LA_ERR_UNSUPPORTED, "dk and dv must each be 32, 64 or 128");
    // element counts stay far below 2^62 and the grid below 2^31
    const double n = (double)s.B * (double)(s.T > 0 ? s.T : 1) * (double)s.H * 128.0;
    if (n > 4.0e18 || (double)s.B * (double)s.H * 4.0 > 2.0e9)
        return fail(LA_ERR_INVALID_ARG, "problem too large");
    return LA_OK;
}

// `need` is false for an empty sequence (T == 0), whose gate tensors hold no
// elements and may be passed as NULL.
la_status validate_gates(la_rule rule, const float *g, const float *beta, const void *z0,
                         const void *z1, bool need) {
    if (rule == LA_RULE_ELU) {
        if (g || beta) return fail(LA_ERR_INVALID_ARG, "ELU takes no gate: g and beta must be NULL");
    } else {
        if (z0 || z1) return fail(LA_ERR_INVALID_ARG, "z0/z_out (and step z) are ELU-only");
        if (need && !g)
            return fail(LA_ERR_INVALID_ARG, rule == LA_RULE_GLA   ? "GLA needs the gate g"
                                            : rule == LA_RULE_KDA ? "KDA needs alpha (g)"
                                                                  : "GDN needs alpha (g)");
        if (rule == LA_RULE_GLA && beta) return fail(LA_ERR_INVALID_ARG, "GLA takes no beta");
        if (need && (rule == LA_RULE_GDN || rule == LA_RULE_KDA) && !beta)
            return fail(LA_ERR_INVALID_ARG, rule == LA_RULE_KDA ? "KDA needs beta" : "GDN needs beta");
    }
    return LA_OK;
}

la_status check_launch(const char *what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return fail(LA_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
    return ok();
}

// ---------------------------------------------------------------------------
// Recurrent kernel dispatch (fp32 prefill, small-dk bf16 prefill, decode).
// ---------------------------------------------------------------------------
template <int RULE, int DK, int DV>
la_status launch_rec_typed(const la::RecurrentParams &p, la_dtype dt, cudaStream_t st) {
    const dim3 grid((unsigned)(p.B * p.H)), block(256);
    if (dt == LA_BF16)
        la::recurrent_kernel<RULE, DK, DV, __nv_bfloat16><<<grid, block, 0, st>>>(p);
    else
        la::recurrent_kernel<RULE, DK, DV, float><<<grid, block, 0, st>>>(p);
    return check_launch("recurrent kernel launch");
}

template <int RULE, int DK>
la_status launch_rec_dv(const la::RecurrentParams &p, int64_t dv, la_dtype dt, cudaStream_t st) {
    switch (dv) {
        case 32: return launch_rec_typed<RULE, DK, 32>(p, dt, st);
        case 64: return launch_rec_typed<RULE, DK, 64>(p, dt, st);
        default: return launch_rec_typed<RULE, DK, 128>(p, dt, st);
    }
}

template <int RULE>
la_status launch_rec_dk(const la::RecurrentParams &p, int64_t dk, int64_t dv, la_dtype dt,
                        cudaStream_t st) {
    switch (dk) {
        case 32: return launch_rec_dv<RULE, 32>(p, dv, dt, st);
        case 64: return launch_rec_dv<RULE, 64>(p, dv, dt, st);
        default: return launch_rec_dv<RULE, 128>(p, dv, dt, st);
    }
}

la_status launch_recurrent(la_rule rule, const la::RecurrentParams &p, int64_t dk, int64_t dv,
                           la_dtype dt, cudaStream_t st) {
    switch (rule) {
        case LA_RULE_ELU: return launch_rec_dk<la::kRuleELU>(p, dk, dv, dt, st);
        case LA_RULE_GLA: return launch_rec_dk<la::kRuleGLA>(p, dk, dv, dt, st);
        case LA_RULE_KDA: return launch_rec_dk<la::kRuleKDA>(p, dk, dv, dt, st);
        default: return launch_rec_dk<la::kRuleGDN>(p, dk, dv, dt, st);
    }
}

// ---------------------------------------------------------------------------
// TMA descriptor encoding through the driver entry point (no -lcuda needed).
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

}  // namespace

namespace la {
// 4-D map over a [B,T,H,D] tensor (innermost first: D, H, T, B), box
// {box_d, 1, box_t, 1}.  Rows past T read as zero.
bool make_map_4d(CUtensorMap *map, const void *base, CUtensorMapDataType dtype, int esize,
                 int64_t B, int64_t T, int64_t H, int64_t D, int box_d, int box_t,
                 CUtensorMapSwizzle swz) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)(D * esize), (cuuint64_t)(H * D * esize),
                             (cuuint64_t)(T * H * D * esize)};
    cuuint32_t box[4] = {(cuuint32_t)box_d, 1u, (cuuint32_t)box_t, 1u};
    cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    CUresult r = fn(map, dtype, 4, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Opt a kernel into more than 48 KB of dynamic shared memory (once per process
// and device is enough; repeating it is harmless).
// Opt the kernel in to `bytes` of dynamic shared memory and ask for the largest
// shared-memory carveout, so that several CTAs of a small-footprint kernel can
// be resident on one SM (and the occupancy query counts them).
cudaError_t allow_smem(const void *kernel, int bytes) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared);
    return e;
}
}  // namespace la

namespace {

bool uses_chunk_kernels(const la_fwd_args &a) {
    return a.dtype == LA_BF16 && a.dk == 128 && a.T > 0;
}

// Output normalisation arguments (ABI version 3), shared by la_fwd and la_step.
la_status validate_norm(int32_t out_norm, float norm_eps, const float *norm_w, bool device_ptrs) {
    if (out_norm != 0 && out_norm != 1) return fail(LA_ERR_INVALID_ARG, "out_norm must be 0 or 1");
    if (!out_norm) return LA_OK;
    if (!(norm_eps > 0.f) || !std::isfinite(norm_eps))
        return fail(LA_ERR_INVALID_ARG, "out_norm needs a finite norm_eps > 0");
    if (device_ptrs && norm_w && !aligned16(norm_w))
        return fail(LA_ERR_ALIGNMENT, "device pointers must be 16-byte aligned");
    return LA_OK;
}

// In-place head-wise RMS normalisation of `rows` rows of dv values of o.
la_status launch_norm(la_dtype dtype, void *o, int64_t rows, int64_t dv, const float *w, float eps,
                      cudaStream_t st) {
    const cudaError_t e =
        dtype == LA_BF16
            ? la::launch_out_rmsnorm(static_cast<__nv_bfloat16 *>(o), rows, dv, w, eps, st)
            : la::launch_out_rmsnorm(static_cast<float *>(o), rows, dv, w, eps, st);
    if (e != cudaSuccess) return fail(LA_ERR_CUDA, std::string("output norm launch: ") + cudaGetErrorString(e));
    return ok();
}

// `recurrent`: run on the per-token recurrent kernel even where the chunked
// kernels apply (la_fwd_noalloc for KDA problems whose chunked scratch exceeds
// the library's array).
la_status launch_fwd_core(const la_fwd_args &a, cudaStream_t st, bool recurrent) {
    const Shape s{a.B, a.T, a.H, a.dk, a.dv};
    if (a.T == 0 || (a.cu_seqlens && a.max_seqlen == 0)) {   // no token in any sequence
        const size_t sb = (size_t)(s.B * s.H * s.dk * s.dv) * sizeof(float);
        const size_t zb = (size_t)(s.B * s.H * s.dk) * sizeof(float);
        if (a.S_out && a.S_out != a.S0) {
            cudaError_t e = a.S0 ? cudaMemcpyAsync(a.S_out, a.S0, sb, cudaMemcpyDeviceToDevice, st)
                                 : cudaMemsetAsync(a.S_out, 0, sb, st);
            if (e != cudaSuccess) return fail(LA_ERR_CUDA, cudaGetErrorString(e));
        }
        if (a.z_out && a.z_out != a.z0) {
            cudaError_t e = a.z0 ? cudaMemcpyAsync(a.z_out, a.z0, zb, cudaMemcpyDeviceToDevice, st)
                                 : cudaMemsetAsync(a.z_out, 0, zb, st);
            if (e != cudaSuccess) return fail(LA_ERR_CUDA, cudaGetErrorString(e));
        }
        return ok();
    }
    if (!recurrent && uses_chunk_kernels(a)) {
        la::ChunkParams p{};
        p.B = a.B; p.T = a.T; p.H = a.H; p.dv = a.dv;
        p.q = a.q; p.k = a.k; p.v = a.v; p.g = a.g; p.beta = a.beta;
        p.S0 = a.S0; p.z0 = a.z0; p.S_out = a.S_out; p.z_out = a.z_out;
        p.o = a.o; p.eps = a.eps;
        p.cu_seqlens = a.cu_seqlens; p.max_seqlen = a.max_seqlen;
        std::string err;
        const la_status r =
            (la_status)la::launch_chunk_tc((int)a.rule, p, a.workspace, a.workspace_bytes, st, &err);
        if (r != LA_OK) return fail(r, err);
        return check_launch("chunk kernel launch");
    }
    la::RecurrentParams p{};
    p.B = a.B; p.T = a.T; p.H = a.H;
    p.q = a.q; p.k = a.k; p.v = a.v; p.g = a.g; p.beta = a.beta;
    p.S_in = a.S0; p.S_out = a.S_out; p.z_in = a.z0; p.z_out = a.z_out;
    p.o = a.o; p.eps = a.eps;
    p.cu_seqlens = a.cu_seqlens; p.max_seqlen = a.max_seqlen;
    return launch_recurrent(a.rule, p, a.dk, a.dv, a.dtype, st);
}

la_status launch_fwd(const la_fwd_args &a, cudaStream_t st, bool recurrent = false) {
    la_status r = launch_fwd_core(a, st, recurrent);
    if (r != LA_OK || !a.out_norm || a.T == 0) return r;
    // o is [B,T,H,dv] dense or [1,T,H,dv] packed
    const int64_t rows = (a.cu_seqlens ? a.T : a.B * a.T) * a.H;
    return launch_norm(a.dtype, a.o, rows, a.dv, a.norm_w, a.norm_eps, st);
}

// The caller's arguments as this library's la_fwd_args: a struct from an older
// header (ABI version 1, without the packed-sequence fields) is accepted and the
// missing fields read as NULL / 0.
la_status load_fwd_args(const la_fwd_args *in, la_fwd_args *out) {
    if (!in) return fail(LA_ERR_INVALID_ARG, "args is NULL");
    constexpr size_t v1 = offsetof(la_fwd_args, cu_seqlens);
    if (in->struct_size < v1)
        return fail(LA_ERR_INVALID_ARG, "struct_size smaller than the version-1 la_fwd_args");
    memset(out, 0, sizeof(*out));
    memcpy(out, in, in->struct_size < sizeof(la_fwd_args) ? in->struct_size : sizeof(la_fwd_args));
    out->struct_size = sizeof(la_fwd_args);
    return LA_OK;
}

// `host_bufs`: the data pointers are host pointers (la_fwd_host).
la_status validate_fwd(const la_fwd_args *a, bool device_ptrs, bool host_bufs = false) {
    const Shape s{a->B, a->T, a->H, a->dk, a->dv};
    la_status r = validate_common(a->rule, a->dtype, s);
    if (r != LA_OK) return r;
    r = validate_gates(a->rule, a->g, a->beta, a->z0, a->z_out, a->T > 0);
    if (r != LA_OK) return r;
    if (a->T > 0 && (!a->q || !a->k || !a->v || !a->o))
        return fail(LA_ERR_INVALID_ARG, "q, k, v and o must be non-NULL when T > 0");
    if (!(a->eps >= 0.f)) return fail(LA_ERR_INVALID_ARG, "eps must be >= 0");
    r = validate_norm(a->out_norm, a->norm_eps, a->norm_w, device_ptrs);
    if (r != LA_OK) return r;
    if (a->cu_seqlens) {
        if (host_bufs)
            return fail(LA_ERR_UNSUPPORTED, "packed sequences (cu_seqlens) need device buffers: use la_fwd");
        if (reinterpret_cast<uintptr_t>(a->cu_seqlens) & 7u)
            return fail(LA_ERR_ALIGNMENT, "cu_seqlens must be 8-byte aligned");
        if (a->max_seqlen < 0 || a->max_seqlen > a->T)
            return fail(LA_ERR_INVALID_ARG, "packed sequences need 0 <= max_seqlen <= T");
    }
    if (device_ptrs) {
        const void *ps[] = {a->q, a->k, a->v, a->g, a->beta, a->S0, a->z0, a->o, a->S_out, a->z_out};
        for (const void *p : ps)
            if (p && !aligned16(p)) return fail(LA_ERR_ALIGNMENT, "device pointers must be 16-byte aligned");
    }
    return LA_OK;
}

}  // namespace

extern "C" {

la_status la_fwd(const la_fwd_args *in, void *stream) {
    la_fwd_args A;
    la_status r = load_fwd_args(in, &A);
    if (r != LA_OK) return r;
    r = validate_fwd(&A, true);
    if (r != LA_OK) return r;
    if (uses_chunk_kernels(A)) {
        const size_t need = la::chunk_workspace_bytes((int)A.rule, A.B, A.T, A.H, A.dv, A.cu_seqlens != nullptr,
                                                      A.max_seqlen);
        if (need && (!A.workspace || A.workspace_bytes < need || !aligned16(A.workspace)))
            return fail(LA_ERR_WORKSPACE,
                        "workspace missing, misaligned or smaller than la_fwd_workspace_size()");
    }
    return launch_fwd(A, static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------------------
// la_fwd_noalloc: the workspace is this library's own fixed device array.
// ---------------------------------------------------------------------------
static __device__ __align__(256) uint8_t g_noalloc_scratch[LA_NOALLOC_SCRATCH_BYTES];

namespace {
// The array's device address in the calling thread's current CUDA context,
// cached per context.  A context is named by its driver-assigned ID
// (cuCtxGetId), which is never reused within a process: after
// cudaDeviceReset, or under a context the caller created, the address is
// looked up again instead of reusing one from a context that no longer holds
// the array.  Without the driver entry points the address is looked up on every
// call (cudaGetSymbolAddress allocates nothing).
std::mutex g_noalloc_mu;
constexpr int kNoallocCache = 64;
struct NoallocEntry {
    unsigned long long ctx_id;
    void *ptr;
};
NoallocEntry g_noalloc_cache[kNoallocCache];
int g_noalloc_used = 0, g_noalloc_next = 0;

using PfnCtxGetCurrent = CUresult (*)(CUcontext *);
using PfnCtxGetId = CUresult (*)(CUcontext, unsigned long long *);

void *driver_fn(const char *name) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return nullptr;
    return p;
}

// ID of the calling thread's current context (false if it cannot be read).
bool current_context_id(unsigned long long *id) {
    static PfnCtxGetCurrent get_current = nullptr;
    static PfnCtxGetId get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        get_current = reinterpret_cast<PfnCtxGetCurrent>(driver_fn("cuCtxGetCurrent"));
        get_id = reinterpret_cast<PfnCtxGetId>(driver_fn("cuCtxGetId"));
    });
    CUcontext ctx = nullptr;
    return get_current && get_id && get_current(&ctx) == CUDA_SUCCESS && ctx &&
           get_id(ctx, id) == CUDA_SUCCESS;
}

la_status noalloc_scratch(void **out) {
    // no context current yet (the runtime binds the primary one lazily): the
    // lookup below binds it, and the next call finds it named
    unsigned long long id = 0;
    const bool named = current_context_id(&id);
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (named)
        for (int i = 0; i < g_noalloc_used; ++i)
            if (g_noalloc_cache[i].ctx_id == id) {
                *out = g_noalloc_cache[i].ptr;
                return LA_OK;
            }
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p)
        return fail(LA_ERR_CUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
    if (named) {
        const int slot = g_noalloc_used < kNoallocCache ? g_noalloc_used++ : (g_noalloc_next++ % kNoallocCache);
        g_noalloc_cache[slot] = NoallocEntry{id, p};
    }
    *out = p;
    return LA_OK;
}
}  // namespace

la_status la_fwd_noalloc(const la_fwd_args *args, void *stream) {
    la_fwd_args a;
    la_status r = load_fwd_args(args, &a);
    if (r != LA_OK) return r;
    r = validate_fwd(&a, true);
    if (r != LA_OK) return r;
    a.workspace = nullptr;
    a.workspace_bytes = 0;
    size_t need = uses_chunk_kernels(a) ? la::chunk_workspace_bytes((int)a.rule, a.B, a.T, a.H, a.dv,
                                                                    a.cu_seqlens != nullptr, a.max_seqlen)
                                        : 0;
    // KDA has a kernel that needs no scratch (the per-token recurrent one): a
    // problem whose chunked scratch does not fit the array runs there instead
    const bool recurrent = need > LA_NOALLOC_SCRATCH_BYTES && a.rule == LA_RULE_KDA;
    if (recurrent) need = 0;
    if (need > LA_NOALLOC_SCRATCH_BYTES)
        return fail(LA_ERR_WORKSPACE, "problem needs " + std::to_string(need) +
                                          " bytes of scratch; la_fwd_noalloc has " +
                                          std::to_string((size_t)LA_NOALLOC_SCRATCH_BYTES) +
                                          " (use la_fwd with a caller workspace)");
    if (need) {
        r = noalloc_scratch(&a.workspace);
        if (r != LA_OK) return r;
        a.workspace_bytes = LA_NOALLOC_SCRATCH_BYTES;
    }
    return launch_fwd(a, static_cast<cudaStream_t>(stream), recurrent);
}

la_status la_fwd_workspace_size(const la_fwd_args *args, size_t *bytes) {
    if (!bytes) return fail(LA_ERR_INVALID_ARG, "bytes is NULL");
    la_fwd_args a;
    la_status r = load_fwd_args(args, &a);
    if (r != LA_OK) return r;
    r = validate_fwd(&a, false);
    if (r != LA_OK) return r;
    *bytes = uses_chunk_kernels(a) ? la::chunk_workspace_bytes((int)a.rule, a.B, a.T, a.H, a.dv,
                                                               a.cu_seqlens != nullptr, a.max_seqlen)
                                   : 0;
    return ok();
}

la_status la_step(const la_step_args *in, void *stream) {
    if (!in) return fail(LA_ERR_INVALID_ARG, "args is NULL");
    // a struct from an ABI version-2 header ends at `o`: no output normalisation
    constexpr size_t v2 = offsetof(la_step_args, out_norm);
    if (in->struct_size < v2)
        return fail(LA_ERR_INVALID_ARG, "struct_size smaller than the version-2 la_step_args");
    la_step_args A;
    memset(&A, 0, sizeof(A));
    memcpy(&A, in, in->struct_size < sizeof(la_step_args) ? in->struct_size : sizeof(la_step_args));
    A.struct_size = sizeof(la_step_args);
    const la_step_args *a = &A;
    const Shape s{a->N, 1, a->H, a->dk, a->dv};
    la_status r = validate_common(a->rule, a->dtype, s);
    if (r != LA_OK) return r;
    r = validate_gates(a->rule, a->g, a->beta, a->z, nullptr, true);
    if (r != LA_OK) return r;
    if (!a->q || !a->k || !a->v || !a->o || !a->S)
        return fail(LA_ERR_INVALID_ARG, "q, k, v, o and S must be non-NULL");
    if (a->rule == LA_RULE_ELU && !a->z) return fail(LA_ERR_INVALID_ARG, "ELU decode needs z");
    if (!(a->eps >= 0.f)) return fail(LA_ERR_INVALID_ARG, "eps must be >= 0");
    r = validate_norm(a->out_norm, a->norm_eps, a->norm_w, true);
    if (r != LA_OK) return r;
    const void *ps[] = {a->q, a->k, a->v, a->g, a->beta, a->S, a->z, a->o};
    for (const void *p : ps)
        if (p && !aligned16(p)) return fail(LA_ERR_ALIGNMENT, "device pointers must be 16-byte aligned");
    la::RecurrentParams p{};
    p.B = a->N; p.T = 1; p.H = a->H;
    p.q = a->q; p.k = a->k; p.v = a->v; p.g = a->g; p.beta = a->beta;
    p.S_in = a->S; p.S_out = a->S; p.z_in = a->z; p.z_out = a->z;
    p.o = a->o; p.eps = a->eps;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    r = launch_recurrent(a->rule, p, a->dk, a->dv, a->dtype, st);
    if (r != LA_OK || !a->out_norm) return r;
    return launch_norm(a->dtype, a->o, a->N * a->H, a->dv, a->norm_w, a->norm_eps, st);
}

// Host-buffer path: staging layout = each tensor at a 256-byte aligned offset.
constexpr int kStaged = 12;
struct StagingLayout {
    size_t off[kStaged];  // q k v g beta S0 z0 o S_out z_out workspace norm_w
    size_t bytes[kStaged];
    size_t total;
};

static void staging_layout(const la_fwd_args *a, StagingLayout *L) {
    const size_t es = elem_size(a->dtype);
    const size_t tok = (size_t)(a->B * a->T * a->H);
    size_t gb = 0;
    if (a->g) gb = tok * (a->rule == LA_RULE_GLA || a->rule == LA_RULE_KDA ? (size_t)a->dk : 1) * 4;
    const size_t sb = (size_t)(a->B * a->H * a->dk * a->dv) * 4;
    const size_t zb = (size_t)(a->B * a->H * a->dk) * 4;
    const size_t wb = uses_chunk_kernels(*a)
                          ? la::chunk_workspace_bytes((int)a->rule, a->B, a->T, a->H, a->dv)
                          : 0;
    const size_t nb = (a->out_norm && a->norm_w) ? (size_t)a->dv * 4 : 0;
    const size_t b[kStaged] = {tok * a->dk * es, tok * a->dk * es, tok * a->dv * es, gb,
                               a->beta ? tok * 4 : 0, a->S0 ? sb : 0, a->z0 ? zb : 0,
                               tok * a->dv * es, a->S_out ? sb : 0, a->z_out ? zb : 0, wb, nb};
    size_t o = 0;
    for (int i = 0; i < kStaged; ++i) {
        L->off[i] = o;
        L->bytes[i] = b[i];
        o += (b[i] + 255) & ~(size_t)255;
    }
    L->total = o;
}

la_status la_fwd_host_staging_size(const la_fwd_args *args, size_t *bytes) {
    if (!bytes) return fail(LA_ERR_INVALID_ARG, "bytes is NULL");
    la_fwd_args a;
    la_status r = load_fwd_args(args, &a);
    if (r != LA_OK) return r;
    r = validate_fwd(&a, false, true);
    if (r != LA_OK) return r;
    StagingLayout L;
    staging_layout(&a, &L);
    *bytes = L.total;
    return ok();
}

la_status la_fwd_host(const la_fwd_args *h_in, void *staging, size_t staging_bytes, void *stream) {
    la_fwd_args H_args;
    la_status r = load_fwd_args(h_in, &H_args);
    if (r != LA_OK) return r;
    const la_fwd_args *h = &H_args;
    r = validate_fwd(h, false, true);
    if (r != LA_OK) return r;
    if (!staging || (reinterpret_cast<uintptr_t>(staging) & 255u))
        return fail(LA_ERR_ALIGNMENT, "staging must be a 256-byte aligned device buffer");
    StagingLayout L;
    staging_layout(h, &L);
    if (staging_bytes < L.total) return fail(LA_ERR_WORKSPACE, "staging buffer too small");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char *base = static_cast<char *>(staging);
    const void *src[kStaged] = {h->q, h->k, h->v, h->g, h->beta, h->S0, h->z0,
                                nullptr, nullptr, nullptr, nullptr, h->norm_w};
    void *dptr[kStaged];
    for (int i = 0; i < kStaged; ++i) dptr[i] = L.bytes[i] ? base + L.off[i] : nullptr;
    for (int i = 0; i < kStaged; ++i) {
        if (!L.bytes[i] || !src[i]) continue;
        cudaError_t e = cudaMemcpyAsync(dptr[i], src[i], L.bytes[i], cudaMemcpyHostToDevice, st);
        if (e != cudaSuccess) return fail(LA_ERR_CUDA, std::string("H2D copy: ") + cudaGetErrorString(e));
    }
    la_fwd_args d = *h;
    d.q = dptr[0]; d.k = dptr[1]; d.v = dptr[2];
    d.g = static_cast<const float *>(dptr[3]);
    d.beta = static_cast<const float *>(dptr[4]);
    d.S0 = static_cast<const float *>(dptr[5]);
    d.z0 = static_cast<const float *>(dptr[6]);
    d.o = dptr[7];
    d.S_out = static_cast<float *>(dptr[8]);
    d.z_out = static_cast<float *>(dptr[9]);
    d.workspace = dptr[10];
    d.workspace_bytes = L.bytes[10];
    d.norm_w = static_cast<const float *>(dptr[11]);
    r = la_fwd(&d, stream);
    if (r != LA_OK) return r;
    void *dst[3] = {h->o, h->S_out, h->z_out};
    for (int i = 0; i < 3; ++i) {
        if (!L.bytes[7 + i] || !h->T && i == 0) continue;
        cudaError_t e = cudaMemcpyAsync(dst[i], dptr[7 + i], L.bytes[7 + i], cudaMemcpyDeviceToHost, st);
        if (e != cudaSuccess) return fail(LA_ERR_CUDA, std::string("D2H copy: ") + cudaGetErrorString(e));
    }
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return fail(LA_ERR_CUDA, std::string("sync: ") + cudaGetErrorString(e));
    return ok();
}

la_status la_check_device(void *stream, uint32_t *flags) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(LA_ERR_CUDA, cudaGetErrorString(e));
    uint32_t w = 0, zero = 0;
    e = cudaMemcpyFromSymbol(&w, la::g_error_word, sizeof(w));
    if (e == cudaSuccess && w) e = cudaMemcpyToSymbol(la::g_error_word, &zero, sizeof(zero));
    if (e != cudaSuccess) return fail(LA_ERR_CUDA, cudaGetErrorString(e));
    if (flags) *flags = w;
    if (w & la::kErrTimeout) return fail(LA_ERR_TIMEOUT, "a bounded device wait ran out");
    if (w & la::kErrRange)
        return fail(LA_ERR_RANGE,
                    "a KDA retention product left the chunked kernels' range (an 8-token product "
                    "below 2^-60)");
    if (w & la::kErrSeqlen)
        return fail(LA_ERR_INVALID_ARG,
                    "cu_seqlens: offsets out of order or outside [0, T], or a sequence longer than "
                    "max_seqlen (clamped; those sequences' results are incomplete)");
    return ok();
}

const char *la_status_string(la_status s) {
    switch (s) {
        case LA_OK: return "LA_OK";
        case LA_ERR_INVALID_ARG: return "LA_ERR_INVALID_ARG";
        case LA_ERR_UNSUPPORTED: return "LA_ERR_UNSUPPORTED";
        case LA_ERR_ALIGNMENT: return "LA_ERR_ALIGNMENT";
        case LA_ERR_CUDA: return "LA_ERR_CUDA";
        case LA_ERR_TIMEOUT: return "LA_ERR_TIMEOUT";
        case LA_ERR_RANGE: return "LA_ERR_RANGE";
        case LA_ERR_INTERNAL: return "LA_ERR_INTERNAL";
        case LA_ERR_WORKSPACE: return "LA_ERR_WORKSPACE";
    }
    return "LA_ERR_UNKNOWN";
}

const char *la_last_error_message(void) { return g_last_error.c_str(); }

int la_abi_version(void) { return LA_ABI_VERSION; }

la_status la_testing_set_wait_limit(int64_t cycles, int64_t *previous) {
    long long prev = 0, next = cycles > 0 ? (long long)cycles : la::kWaitLimitCycles;
    cudaError_t e = cudaMemcpyFromSymbol(&prev, la::g_wait_limit, sizeof(prev));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(la::g_wait_limit, &next, sizeof(next));
    if (e != cudaSuccess) return fail(LA_ERR_CUDA, std::string("wait limit: ") + cudaGetErrorString(e));
    if (previous) *previous = (int64_t)prev;
    return ok();
}

}  // extern "C"
