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
// on the same stream: one warp per row, each lane holding dv/32 consecutive
// values (a warp reads the row's 64-512 contiguous bytes at once), the sum of
// squares reduced by shuffles in fp32.  It reads o as stored (bf16 rounded for
// bf16 problems) and rounds its result once.  HBM-bound: 2 x rows x dv x
// sizeof(o) bytes.
#pragma once

#include <algorithm>

#include "device.cuh"

namespace la {

template <typename T, int DV>
__global__ void __launch_bounds__(256) out_rmsnorm_kernel(T *o, int64_t rows, const float *w, float eps) {
    constexpr int PER = DV / 32;   // values per lane: 1, 2 or 4
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    float wl[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) wl[e] = w ? w[lane * PER + e] : 1.f;
    for (int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < rows; r += nwarps) {
        T *row = o + r * DV + lane * PER;
        float x[PER];
#pragma unroll
        for (int e = 0; e < PER; ++e) x[e] = to_f32(row[e]);
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < PER; ++e) ss = fmaf(x[e], x[e], ss);
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
        const float inv = rsqrtf(ss * (1.f / DV) + eps);
#pragma unroll
        for (int e = 0; e < PER; ++e) row[e] = from_f32<T>(x[e] * inv * wl[e]);
    }
}

// o: `rows` rows of dv values of type T (contiguous), normalised in place.
template <typename T>
cudaError_t launch_out_rmsnorm(T *o, int64_t rows, int64_t dv, const float *w, float eps, cudaStream_t st) {
    if (rows <= 0) return cudaSuccess;
    // 8 rows per block; a grid of a few waves of resident blocks strides over the rest
    const int64_t blocks = std::min<int64_t>((rows + 7) / 8, (int64_t)sm_count() * 16);
    const unsigned grid = (unsigned)blocks;
    if (dv == 32) out_rmsnorm_kernel<T, 32><<<grid, 256, 0, st>>>(o, rows, w, eps);
    else if (dv == 64) out_rmsnorm_kernel<T, 64><<<grid, 256, 0, st>>>(o, rows, w, eps);
    else out_rmsnorm_kernel<T, 128><<<grid, 256, 0, st>>>(o, rows, w, eps);
    return cudaGetLastError();
}

}  // namespace la
