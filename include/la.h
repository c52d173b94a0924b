/*
 * la.h — C ABI of the B200 (sm_100a) causal linear-attention library.
 *
 * The library computes the causal linear-attention forward that folds a
 * sequence into a fixed dk x dv matrix state per (batch, head), for these
 * update rules (KDA, the fourth, is described with la_rule below):
 *
 *   LA_RULE_ELU  normalized ELU+1 linear attention
 *       S_t = S_{t-1} + phi(k_t) v_t^T,  z_t = z_{t-1} + phi(k_t),
 *       o_t = phi(q_t)^T S_t / (phi(q_t)^T z_t + eps),  phi(x) = ELU(x) + 1
 *       (page "Linear / RNN 路线：砍 softmax，固定 state 替代 KV", §2.1; eps in
 *       the denominator as in page "状态空间与线性注意力", section 线性注意力)
 *   LA_RULE_GLA  gated linear attention, per-key-dimension gate g_t in (0,1)^dk
 *       S_t = diag(g_t) S_{t-1} + k_t v_t^T,  o_t = S_t^T q_t
 *       (page "Linear / RNN 路线", §2.2)
 *   LA_RULE_GDN  gated delta rule, scalar alpha_t, beta_t in (0,1)
 *       S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,
 *       o_t = S_t^T q_t
 *       (page "线性注意力与 SSM：把整张关系表变成一条状态流", GDN box, written
 *       there for the transposed dv x dk state; output read after the write as
 *       in page "状态空间与线性注意力", section KDA recurrent reference)
 *
 * Entry points
 *   la_fwd   chunked prefill over T tokens, optional initial state in, final
 *            state out (the selective-scan contract of page "状态空间与线性注意力":
 *            optional initial state, all outputs and the final state returned).
 *   la_step  one decode token per sequence, state updated in place.
 *   la_fwd_host  la_fwd on HOST buffers: copies in, runs, copies out.
 *   la_fwd_noalloc  la_fwd with a library-owned scratch array (no allocation).
 *   la_check_device  reads and clears the device-side error word.
 *
 * Conventions (all entry points)
 *   - Layouts are dense row-major: q,k [B,T,H,dk]; v,o [B,T,H,dv]; GLA gate
 *     [B,T,H,dk] fp32; GDN alpha,beta [B,T,H] fp32; KDA alpha [B,T,H,dk] and
 *     beta [B,T,H] fp32; state [B,H,dk,dv] fp32 with rows = key dims; ELU
 *     normaliser z [B,H,dk] fp32.  Decode drops the T axis.  Packed sequences
 *     (la_fwd_args.cu_seqlens) put the token tensors on one axis [1,T,H,*].
 *   - Device pointers must be 16-byte aligned.  The library reads and writes
 *     only the buffers it is given, never allocates or frees device memory,
 *     never synchronises the stream (except la_check_device / la_fwd_host,
 *     which say so) and never changes the current device.  The caller owns
 *     every buffer and keeps it alive until the stream work completes.
 *   - Each call enqueues work on `stream` (a cudaStream_t passed as void*;
 *     NULL = the legacy default stream) and returns immediately.  Arguments are
 *     validated on the host before any launch; an invalid call launches nothing.
 *   - Conditions detected on the device (a bounded wait that ran out, a KDA
 *     sub-chunk whose retention product leaves the chunked kernels' range,
 *     packed-sequence offsets that are out of order or out of range) set a
 *     device-wide error word; la_check_device() reads and clears it.
 *   - Supported sizes: dk, dv in {32, 64, 128}; B, H >= 1; T >= 0.  T == 0
 *     writes S_out = S0 (or zeros) and z_out = z0 (or zeros).
 *   - There is no CPU fallback: every result comes from a CUDA kernel.
 */
#ifndef LA_H_
#define LA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LA_ABI_VERSION 3

typedef enum {
    LA_OK = 0,
    LA_ERR_INVALID_ARG = 1,   /* null pointer, negative size, bad enum, size mismatch */
    LA_ERR_UNSUPPORTED = 2,   /* dk/dv/dtype combination without a kernel */
    LA_ERR_ALIGNMENT = 3,     /* a device pointer is not 16-byte aligned */
    LA_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
    LA_ERR_TIMEOUT = 5,       /* a bounded device-side wait ran out (la_check_device) */
    LA_ERR_RANGE = 6,         /* a gate product left a chunked kernel's range (la_check_device) */
    LA_ERR_INTERNAL = 7,
    LA_ERR_WORKSPACE = 8      /* workspace missing or smaller than la_fwd_workspace_size() */
} la_status;

/*
 * Update rules (S is dk x dv; every output is read after its token's update):
 *   ELU  normalised ELU+1 linear attention ("Linear / RNN 路线", §2.1)
 *   GLA  S_t = Diag(g_t) S_{t-1} + k_t v_t^T ("Linear / RNN 路线", §2.2),
 *        for every g in (0, 1].  bf16 GLA with dk = 128 runs chunked on the
 *        tensor cores; a sequence with a 64-token chunk whose gate product falls
 *        below 2^-120 in some key dim (the chunked form's range) is recomputed
 *        within the same call by the per-token recurrent kernel (exact, slower).
 *   GDN  S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T
 *        ("线性注意力与 SSM", GDN box, in the dk x dv orientation)
 *   KDA  S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
 *        alpha_t per key channel ("状态空间与线性注意力", KDA：逐通道遗忘与误差写入).
 *        bf16 KDA with dk = 128 (dense or packed) runs chunked on the tensor
 *        cores, for retention whose product over any 8 consecutive tokens stays
 *        >= 2^-60 per channel (the page's bounded log-decay, log alpha > -5,
 *        satisfies this); outside that domain la_check_device reports
 *        LA_ERR_RANGE.  fp32 and dk < 128 KDA run on the per-token recurrent
 *        kernel (CUDA cores), which has no such domain.
 */
typedef enum { LA_RULE_ELU = 0, LA_RULE_GLA = 1, LA_RULE_GDN = 2, LA_RULE_KDA = 3 } la_rule;

/* Element type of q, k, v and o.  Gates and the state are always fp32. */
typedef enum { LA_F32 = 0, LA_BF16 = 1 } la_dtype;

/*
 * Prefill arguments.  All pointers are device pointers.
 *   q, k   [B,T,H,dk] of `dtype`
 *   v      [B,T,H,dv] of `dtype`
 *   g      GLA: gate [B,T,H,dk], every entry in (0,1];  GDN: alpha [B,T,H] in (0,1];
 *          KDA: alpha [B,T,H,dk] in (0,1] (per key channel);  ELU: must be NULL
 *   beta   GDN, KDA: [B,T,H] in [0,1];  others: NULL
 *   S0     [B,H,dk,dv] initial state, or NULL for zeros
 *   z0     ELU: [B,H,dk] initial normaliser, or NULL for zeros; others: NULL
 *   eps    ELU: added to the denominator after the dot product; ignored otherwise
 *   o      [B,T,H,dv] of `dtype` (written)
 *   S_out  [B,H,dk,dv] final state (written), or NULL; may alias S0
 *   z_out  ELU: [B,H,dk] final normaliser, or NULL; may alias z0
 *   workspace / workspace_bytes: device scratch of at least
 *          la_fwd_workspace_size() bytes, 16-byte aligned (may be NULL when that
 *          size is 0).  The gated delta rule on the tensor-core path (bf16,
 *          dk = 128) needs 32 KB per (batch, head, 64-token chunk): the chunk's
 *          T diag(beta) (T = (I + A)^-1), masked decayed score and
 *          -T diag(beta gamma) K operands, written by a first kernel and read by
 *          the second within the same call.  ELU+1 and GLA over few heads and long
 *          sequences run segment-parallel and keep there the summary of each
 *          piece of every segment but the last (dk*dv + dk floats per piece: the
 *          piece's state contribution and its normaliser sum or gate product).
 *          Chunked GLA also keeps one 4-byte flag per (batch, head) there (a
 *          sequence to recompute, see la_rule), so its workspace is never 0.
 *          Chunked KDA keeps 32.5 KB per (batch, head, chunk) (the operand
 *          images of T diag(beta), P and -T diag(beta) (K o Gamma), and the
 *          chunk's retention product) plus two bf16 [B,Ls,H,128] tensors: q
 *          scaled by the cumulative retention, and k scaled by the retention
 *          from the token to its chunk's end (Ls = T;
 *          with packed sequences Ls = 64 ceil(max_seqlen / 64), one row block
 *          per sequence).
 *          Calls that share
 *          one workspace must be ordered (same stream), otherwise they race.
 *          A missing or short workspace returns LA_ERR_WORKSPACE before any launch.
 * q/k/v/o must not overlap S_out/z_out.
 *
 * Packed variable-length sequences (fields appended in ABI version 2; a caller
 * built against version 1 passes the smaller struct_size and gets the dense
 * layout above):
 *   cu_seqlens  device int64 [B+1], or NULL for the dense layout.  Sequence b
 *          is tokens [cu_seqlens[b], cu_seqlens[b+1]) of ONE packed token axis:
 *          q, k, g [1,T,H,*], v, o [1,T,H,dv], beta [1,T,H], with T the packed
 *          length.  B counts sequences; S0/S_out/z0/z_out stay [B,H,...] and
 *          every sequence starts from its own S0[b] (state reset at each
 *          sequence start; the "verification matrix" of page "状态空间与线性注意力"
 *          asks for exactly this reset).  Offsets must be nondecreasing, within
 *          [0, T], 8-byte aligned.  Sequences may be empty.
 *   max_seqlen  upper bound of cu_seqlens[b+1] - cu_seqlens[b] (0 <= max_seqlen
 *          <= T); sizes the gated delta rule's workspace and the grid.
 *   The offsets are read on the device only: offsets out of order or outside
 *   [0, T], or a sequence longer than max_seqlen, are clamped to stay in bounds
 *   and reported by la_check_device as LA_ERR_INVALID_ARG.  Packed sequences
 *   are not accepted by la_fwd_host (LA_ERR_UNSUPPORTED).
 *
 * Output normalisation (fields appended in ABI version 3, in la_fwd_args and
 * la_step_args; a caller built against an older header passes the older
 * struct_size and gets none):
 *   out_norm  0: o as above.  1: every (token, head) row of o is replaced by
 *          its head-wise RMS normalisation, o_j <- w_j o_j / sqrt(mean_j o_j^2 +
 *          norm_eps) over the dv values of the row: the output normalisation of
 *          Lightning attention, o_t = Norm(q_t^T S_t) (page "Linear / RNN 路线",
 *          §2.4, with GLA at g = 1), and the head-wise RMSNorm that K3 applies
 *          to the recurrent output (page "状态空间与线性注意力", KDA section).
 *          Applies to every rule.  The state and z are not affected.
 *   norm_eps  > 0 (finite), added to the mean square before the square root.
 *   norm_w    fp32 [dv] per-channel weight shared by the heads, or NULL (= 1);
 *          16-byte aligned device pointer (host pointer for la_fwd_host).
 *   The normalisation is a second pass over o on the same stream (a row spans
 *   every value slab of the chunked kernels); it reads o as stored, so for bf16
 *   problems it normalises the bf16-rounded output and rounds once more.
 */
typedef struct la_fwd_args {
    uint32_t struct_size;     /* = sizeof(la_fwd_args) */
    la_rule rule;
    la_dtype dtype;
    int64_t B, T, H, dk, dv;
    const void *q, *k, *v;
    const float *g;
    const float *beta;
    const float *S0;
    const float *z0;
    float eps;
    void *o;
    float *S_out;
    float *z_out;
    void *workspace;
    size_t workspace_bytes;
    const int64_t *cu_seqlens;   /* ABI version 2 */
    int64_t max_seqlen;          /* ABI version 2 */
    int32_t out_norm;            /* ABI version 3: output normalisation (below) */
    float norm_eps;              /* ABI version 3 */
    const float *norm_w;         /* ABI version 3 */
} la_fwd_args;

/*
 * Decode arguments (one token per sequence, N = batch).  Device pointers.
 *   q, k [N,H,dk]; v, o [N,H,dv] of `dtype`
 *   g    GLA [N,H,dk] / GDN alpha [N,H] / KDA alpha [N,H,dk] / ELU NULL;
 *        beta GDN, KDA [N,H] / NULL
 *   S    [N,H,dk,dv] fp32, read and overwritten with the updated state
 *   z    ELU [N,H,dk] fp32, read and overwritten; NULL otherwise
 *   out_norm, norm_eps, norm_w  as in la_fwd_args (ABI version 3)
 * The output is read from the state after this token's update.  A struct of
 * ABI version 2 (struct_size up to `o`) is accepted, without normalisation.
 */
typedef struct la_step_args {
    uint32_t struct_size;     /* = sizeof(la_step_args) */
    la_rule rule;
    la_dtype dtype;
    int64_t N, H, dk, dv;
    const void *q, *k, *v;
    const float *g;
    const float *beta;
    float *S;
    float *z;
    float eps;
    void *o;
    int32_t out_norm;            /* ABI version 3: output normalisation (below) */
    float norm_eps;              /* ABI version 3 */
    const float *norm_w;         /* ABI version 3 */
} la_step_args;

/* Chunked prefill (see the struct above).  Asynchronous on `stream`. */
la_status la_fwd(const la_fwd_args *args, void *stream);

/* Bytes of device workspace la_fwd needs for these arguments (often 0). */
la_status la_fwd_workspace_size(const la_fwd_args *args, size_t *bytes);

/* One decode step with in-place state update.  Asynchronous on `stream`. */
la_status la_step(const la_step_args *args, void *stream);

/*
 * la_fwd on HOST buffers.  `host_args` has the same fields as for la_fwd but
 * every data pointer (q,k,v,g,beta,S0,z0 read; o,S_out,z_out written) is a
 * host pointer (pinned memory gives asynchronous copies).  `staging` is a
 * caller-owned device buffer of at least la_fwd_host_staging_size() bytes,
 * 256-byte aligned, into which the inputs are copied; the kernels run on it and
 * the outputs are copied back; the staging also holds la_fwd's workspace.  The
 * call enqueues copies and kernels on
 * `stream` and then synchronises that stream, so the host outputs are valid on
 * return.  Allocates nothing.
 */
la_status la_fwd_host_staging_size(const la_fwd_args *host_args, size_t *bytes);
la_status la_fwd_host(const la_fwd_args *host_args, void *staging, size_t staging_bytes,
                      void *stream);

/*
 * la_fwd_noalloc — la_fwd for callers that cannot allocate device memory.
 *
 * No counterpart in the pages: this is an interface for integrators.  Some
 * callers of this library cannot call cudaMalloc (or any allocating routine):
 * code that runs under a host framework which owns all device memory, plugins
 * and embedded runtimes with a fixed memory budget, or a latency-critical path
 * that must not take the allocator's locks or trigger a synchronising
 * allocation.  They cannot provide la_fwd's `workspace` (the gated delta rule's
 * tensor-core path needs one).  This entry point takes the same arguments as
 * la_fwd but ignores args->workspace / workspace_bytes and uses a scratch array
 * that is part of the library itself: a file-scope `__device__` array of
 * LA_NOALLOC_SCRATCH_BYTES (16 MiB), 256-byte aligned.  Every GPU on which the
 * library is loaded holds that array until the process exits.
 *
 *   - The problem's scratch need (la_fwd_workspace_size) must be at most
 *     LA_NOALLOC_SCRATCH_BYTES, otherwise LA_ERR_WORKSPACE is returned before
 *     anything is launched.  For the gated delta rule that is 512
 *     (batch x head x 64-token chunk) units, e.g. B*H = 16 up to T = 2048.
 *     ELU+1 and GLA use the array when they split long sequences of few heads
 *     into segments (the segment summaries, dk*dv + dk floats per piece); the
 *     number of pieces is bounded by the SM count, so that need always fits.
 *     KDA is the exception: a KDA problem whose chunked scratch does not fit
 *     runs on the per-token recurrent kernel, which needs none (slower, same
 *     results within the bf16 tolerance).
 *   - The array's device address is looked up (cudaGetSymbolAddress) in the
 *     calling thread's current CUDA context on the first call made under that
 *     context and reused by later calls under it; a new context (another
 *     device, a context the caller created, or the primary context again after
 *     cudaDeviceReset) gets its own lookup.  Make the first call under a
 *     context before any stream capture.
 *   - All calls share the one array and it keeps the last call's contents; the
 *     kernels write every scratch byte they read within the same call, so no
 *     clearing is needed.  Calls that overlap on the GPU (different streams
 *     without ordering, or several host threads) race on the array, for every
 *     rule that uses it (the gated delta rule, KDA, segment-parallel ELU+1 and
 *     GLA): serialise them.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 * Otherwise identical to la_fwd (validation, status codes, asynchrony).
 */
#define LA_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
la_status la_fwd_noalloc(const la_fwd_args *args, void *stream);

/*
 * Synchronises `stream`, then reads and clears the device error word set by
 * earlier kernels.  Returns LA_OK, LA_ERR_TIMEOUT, LA_ERR_RANGE (KDA only),
 * LA_ERR_INVALID_ARG (packed-sequence offsets that had to be clamped) or
 * LA_ERR_CUDA.  `flags` (may be NULL) receives the raw word (bit 0 timeout,
 * bit 1 range, bit 2 clamped offsets).
 */
la_status la_check_device(void *stream, uint32_t *flags);

/* Static name of a status code. */
const char *la_status_string(la_status s);

/* Detail of the last error returned on the calling host thread ("" if none). */
const char *la_last_error_message(void);

/* LA_ABI_VERSION of the loaded library. */
int la_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LA_H_ */
