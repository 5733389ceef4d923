// Backward of the fused path of section 3.4 (Eq. 13 feeding Eq. 14 of the Chimera paper):
// q = L2norm_h(mShortConv(x_q)), k = L2norm_h(mShortConv(x_k)), v = mShortConv(x_v),
// then the scan.  The chain rule runs in fp32 through the pieces of the library:
//   1. the conv outputs y_q, y_k, y_v are recomputed (fp32),
//   2. q, k = y / |y| per (token, head),
//   3. kda_backward on (q, k, v) gives dq, dk, dv, dg, dbeta, dS0,
//   4. dy = (dq - q (q . dq)) / |y_q| per (token, head) (0 where |y_q| = 0), same for k,
//   5. the conv backward of each tensor gives dx and the weight gradients.
// This file holds the elementwise pieces (widening to fp32 and the per-head norm and
// its derivative); the sequence of launches is in kda_api.cu.

#include <algorithm>

#include "internal.h"

namespace kda {
namespace {

template <typename T>
__global__ void __launch_bounds__(256) to_f32_kernel(const T* __restrict__ x, float* __restrict__ y, int64_t n)
{
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        y[i] = to_f32(x[i]);
}

// one warp per row of D values: y = x / |x| (0 for a zero row)
__global__ void __launch_bounds__(256) l2norm_rows_kernel(const float* __restrict__ x, float* __restrict__ y,
                                                          int64_t rows, int D)
{
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const float* xr = x + row * D;
    float ss = 0.f;
    for (int c = lane; c < D; c += 32) ss = fmaf(xr[c], xr[c], ss);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = ss > 0.f ? rsqrtf(ss) : 0.f;
    for (int c = lane; c < D; c += 32) y[row * D + c] = xr[c] * inv;
}

// in place: d <- (d - u (u . d)) / |x| with u = x / |x|; 0 for a zero row of x
__global__ void __launch_bounds__(256) l2norm_bwd_rows_kernel(const float* __restrict__ x, float* __restrict__ d,
                                                              int64_t rows, int D)
{
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const float* xr = x + row * D;
    float* dr = d + row * D;
    float ss = 0.f, xd = 0.f;
    for (int c = lane; c < D; c += 32) {
        ss = fmaf(xr[c], xr[c], ss);
        xd = fmaf(xr[c], dr[c], xd);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        ss += __shfl_xor_sync(0xffffffffu, ss, o);
        xd += __shfl_xor_sync(0xffffffffu, xd, o);
    }
    if (!(ss > 0.f)) {
        for (int c = lane; c < D; c += 32) dr[c] = 0.f;
        return;
    }
    const float inv = rsqrtf(ss);
    const float ud = xd * inv;   // u . d
    for (int c = lane; c < D; c += 32) dr[c] = (dr[c] - xr[c] * inv * ud) * inv;
}

unsigned grid_for(int64_t n) { return (unsigned)std::min<int64_t>((n + 255) / 256, 148 * 16); }

}  // namespace

cudaError_t launch_to_f32(const void* x, ElemType t, float* y, int64_t n, cudaStream_t s)
{
    if (n == 0) return cudaSuccess;
    count_launch();
    if (t == ET_BF16) to_f32_kernel<__nv_bfloat16><<<grid_for(n), 256, 0, s>>>((const __nv_bfloat16*)x, y, n);
    else if (t == ET_F16) to_f32_kernel<__half><<<grid_for(n), 256, 0, s>>>((const __half*)x, y, n);
    else return cudaMemcpyAsync(y, x, (size_t)n * sizeof(float), cudaMemcpyDeviceToDevice, s);
    return cudaGetLastError();
}

cudaError_t launch_l2norm_rows(const float* x, float* y, int64_t rows, int D, cudaStream_t s)
{
    if (rows == 0) return cudaSuccess;
    count_launch();
    l2norm_rows_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(x, y, rows, D);
    return cudaGetLastError();
}

cudaError_t launch_l2norm_bwd_rows(const float* x, float* d, int64_t rows, int D, cudaStream_t s)
{
    if (rows == 0) return cudaSuccess;
    count_launch();
    l2norm_bwd_rows_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(x, d, rows, D);
    return cudaGetLastError();
}

}  // namespace kda
