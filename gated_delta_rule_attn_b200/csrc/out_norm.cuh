// out_norm.cuh — head-wise RMS normalisation of the attention output.
//
// Lightning attention reads the state unnormalised and controls the range of
// the read with a normalisation of the output, o_t = Norm(q_t^T S_t) (page
// "Linear / RNN 路线", §2.4, RMSNorm); K3 / KDA normalises its recurrent output
// head by head the same way before the output gate (page "状态空间与线性注意力",
// KDA section).  For every (token, head) row x of dv values:
//     y_j = w_j * x_j / sqrt(mean_j x_j^2 + eps),
// with an optional per-channel weight w[dv] (shared by the heads; NULL = 1).
//
// The row spans every value slab of the chunked kernels (each CTA holds 32 or 64
// of the dv columns), so the normalisation is a second pass over o, in place,
// on the same stream: a warp per row, each lane holding dv/32 consecutive
// values (a warp reads the row's 64-512 contiguous bytes at once), the sum of
// squares reduced by shuffles in fp32.  It reads o as stored (bf16 rounded for
// bf16 problems) and rounds its result once.  HBM-bound: 2 x rows x dv x
// sizeof(o) bytes.
#pragma once

#include <algorithm>

#include "device.cuh"

namespace la {

// PER consecutive values of a row as one vector access (8, 4 or 2 bytes for
// bf16; 16, 8 or 4 for fp32: the row offsets keep them aligned).
template <typename T, int PER>
__device__ __forceinline__ void load_vals(const T *p, float *x);
template <typename T, int PER>
__device__ __forceinline__ void store_vals(T *p, const float *x);

template <>
__device__ __forceinline__ void load_vals<__nv_bfloat16, 4>(const __nv_bfloat16 *p, float *x) {
    const uint2 u = *reinterpret_cast<const uint2 *>(p);
    const float2 a = unpack_bf16x2(u.x), b = unpack_bf16x2(u.y);
    x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
}
template <>
__device__ __forceinline__ void load_vals<__nv_bfloat16, 2>(const __nv_bfloat16 *p, float *x) {
    const float2 a = unpack_bf16x2(*reinterpret_cast<const uint32_t *>(p));
    x[0] = a.x; x[1] = a.y;
}
template <>
__device__ __forceinline__ void load_vals<__nv_bfloat16, 1>(const __nv_bfloat16 *p, float *x) {
    x[0] = __bfloat162float(*p);
}
template <>
__device__ __forceinline__ void load_vals<float, 4>(const float *p, float *x) {
    const float4 a = *reinterpret_cast<const float4 *>(p);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
}
template <>
__device__ __forceinline__ void load_vals<float, 2>(const float *p, float *x) {
    const float2 a = *reinterpret_cast<const float2 *>(p);
    x[0] = a.x; x[1] = a.y;
}
template <>
__device__ __forceinline__ void load_vals<float, 1>(const float *p, float *x) { x[0] = *p; }

template <>
__device__ __forceinline__ void store_vals<__nv_bfloat16, 4>(__nv_bfloat16 *p, const float *x) {
    *reinterpret_cast<uint2 *>(p) = make_uint2(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]));
}
template <>
__device__ __forceinline__ void store_vals<__nv_bfloat16, 2>(__nv_bfloat16 *p, const float *x) {
    *reinterpret_cast<uint32_t *>(p) = pack_bf16x2(x[0], x[1]);
}
template <>
__device__ __forceinline__ void store_vals<__nv_bfloat16, 1>(__nv_bfloat16 *p, const float *x) {
    *p = __float2bfloat16_rn(x[0]);
}
template <>
__device__ __forceinline__ void store_vals<float, 4>(float *p, const float *x) {
    *reinterpret_cast<float4 *>(p) = make_float4(x[0], x[1], x[2], x[3]);
}
template <>
__device__ __forceinline__ void store_vals<float, 2>(float *p, const float *x) {
    *reinterpret_cast<float2 *>(p) = make_float2(x[0], x[1]);
}
template <>
__device__ __forceinline__ void store_vals<float, 1>(float *p, const float *x) { *p = x[0]; }

// Each warp takes RW consecutive rows per step and issues all their loads
// before the first reduction, so that enough bytes are in flight to stream at
// HBM speed.
constexpr int kNormRowsPerWarp = 4;

template <typename T, int DV>
__global__ void __launch_bounds__(256) out_rmsnorm_kernel(T *o, int64_t rows, const float *w, float eps) {
    constexpr int PER = DV / 32;   // values per lane: 1, 2 or 4
    constexpr int RW = kNormRowsPerWarp;
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    float wl[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) wl[e] = w ? w[lane * PER + e] : 1.f;
    for (int64_t r0 = (((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5) * RW; r0 < rows;
         r0 += nwarps * RW) {
        float x[RW][PER];
#pragma unroll
        for (int i = 0; i < RW; ++i) {
            if (r0 + i < rows) load_vals<T, PER>(o + (r0 + i) * DV + lane * PER, x[i]);
            else
#pragma unroll
                for (int e = 0; e < PER; ++e) x[i][e] = 0.f;
        }
        float ss[RW];
#pragma unroll
        for (int i = 0; i < RW; ++i) {
            ss[i] = 0.f;
#pragma unroll
            for (int e = 0; e < PER; ++e) ss[i] = fmaf(x[i][e], x[i][e], ss[i]);
        }
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1)
#pragma unroll
            for (int i = 0; i < RW; ++i) ss[i] += __shfl_xor_sync(0xffffffffu, ss[i], m);
#pragma unroll
        for (int i = 0; i < RW; ++i) {
            if (r0 + i >= rows) break;
            const float inv = rsqrtf(ss[i] * (1.f / DV) + eps);
            float y[PER];
#pragma unroll
            for (int e = 0; e < PER; ++e) y[e] = x[i][e] * inv * wl[e];
            store_vals<T, PER>(o + (r0 + i) * DV + lane * PER, y);
        }
    }
}

// o: `rows` rows of dv values of type T (contiguous), normalised in place.
template <typename T>
cudaError_t launch_out_rmsnorm(T *o, int64_t rows, int64_t dv, const float *w, float eps, cudaStream_t st) {
    if (rows <= 0) return cudaSuccess;
    // 8 warps per block, kNormRowsPerWarp rows per warp and step; at most one
    // wave of resident blocks (8 per SM), which strides over the rest
    const int64_t per_block = 8 * kNormRowsPerWarp;
    const int64_t blocks = std::min<int64_t>((rows + per_block - 1) / per_block, (int64_t)sm_count() * 8);
    const unsigned grid = (unsigned)blocks;
    if (dv == 32) out_rmsnorm_kernel<T, 32><<<grid, 256, 0, st>>>(o, rows, w, eps);
    else if (dv == 64) out_rmsnorm_kernel<T, 64><<<grid, 256, 0, st>>>(o, rows, w, eps);
    else out_rmsnorm_kernel<T, 128><<<grid, 256, 0, st>>>(o, rows, w, eps);
    return cudaGetLastError();
}

}  // namespace la
