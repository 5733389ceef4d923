// Backward of the modality-aware short convolution (section 3.4 of the Chimera paper):
// for dL/dy, the gradients dL/dx and dL/dw of the per-segment depthwise conv.
//
// A segment is a box [F, Hgt, Wid] of tokens (text: [1, 1, len]; image: [1, H, W];
// video: [F, H, W], time-first raster order, Eq. 12) and
//   y[p] = sum_tap w[c, tap] x[p + off(tap)]     (shifted positions outside the box read 0)
// with off = (0, 0, j - (Kt-1)) for text tap j, (0, a-1, e-1) for image tap (a, e) and
// (tau-2, a-1, e-1) for video tap (tau, a, e).  It is linear in x and in w, so
//   dx[p] = sum_tap w[c, tap] dy[p - off(tap)]   (over taps with p - off in the box)
//   dw[c, tap] = sum_{rows, p} dy[p] x[p + off(tap)]
// dx: one thread per (row, position, 8 channels) gathers its taps (no atomics).
// dw: a block of 32 channels x 8 position lanes reduces a run of positions in registers
// (one accumulator per tap), then across lanes in shared memory, and adds its sums to dw
// with one atomic per (channel, tap).  fp32 arithmetic; x, dy in fp32 or bf16.

#include "internal.h"

namespace kda {
namespace {

constexpr int MAXTAPS = 27;

struct Taps {
    int n;
    int8_t df[MAXTAPS], dr[MAXTAPS], ds[MAXTAPS];
};

Taps taps_for(int modality, int Kt)
{
    Taps t{};
    if (modality == MSC_TEXT) {
        t.n = Kt;
        for (int j = 0; j < Kt; ++j) t.ds[j] = (int8_t)(j - (Kt - 1));
    } else if (modality == MSC_IMAGE) {
        t.n = 9;
        for (int a = 0; a < 3; ++a)
            for (int e = 0; e < 3; ++e) { t.dr[3 * a + e] = (int8_t)(a - 1); t.ds[3 * a + e] = (int8_t)(e - 1); }
    } else {
        t.n = 27;
        for (int tau = 0; tau < 3; ++tau)
            for (int a = 0; a < 3; ++a)
                for (int e = 0; e < 3; ++e) {
                    const int i = 9 * tau + 3 * a + e;
                    t.df[i] = (int8_t)(tau - 2); t.dr[i] = (int8_t)(a - 1); t.ds[i] = (int8_t)(e - 1);
                }
    }
    return t;
}

__device__ __forceinline__ void load8(const float* p, float (&v)[8])
{
    const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8])
{
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

// grid (ceil(npos * C/8 / 256), B); w: this segment's weight set [C][ntaps]
template <typename TIn>
__global__ void __launch_bounds__(256)
conv_dx_kernel(const TIn* __restrict__ dy, const float* __restrict__ w, float* __restrict__ dx, int T, int C,
               int64_t start, int F, int Hg, int Wd, Taps taps)
{
    const int CG = C / 8;
    const int64_t npos = (int64_t)F * Hg * Wd;
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= npos * CG) return;
    const int cg = (int)(idx % CG);
    const int64_t p = idx / CG;
    const int f = (int)(p / ((int64_t)Hg * Wd)), r = (int)((p / Wd) % Hg), s = (int)(p % Wd);
    const int64_t rowbase = (int64_t)blockIdx.y * T + start;
    const int c0 = cg * 8;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int tp = 0; tp < taps.n; ++tp) {
        const int ff = f - taps.df[tp], rr = r - taps.dr[tp], ss = s - taps.ds[tp];
        if (ff < 0 || ff >= F || rr < 0 || rr >= Hg || ss < 0 || ss >= Wd) continue;
        float g[8];
        load8(dy + (rowbase + ((int64_t)ff * Hg + rr) * Wd + ss) * C + c0, g);
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] = fmaf(w[(int64_t)(c0 + j) * taps.n + tp], g[j], acc[j]);
    }
    float4* o = reinterpret_cast<float4*>(dx + (rowbase + p) * C + c0);
    o[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    o[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
}

constexpr int DW_POS = 256;   // positions per block

// grid (ceil(npos / DW_POS), ceil(C / 32), B); block 256 = 32 channels x 8 position lanes
template <typename TIn>
__global__ void __launch_bounds__(256)
conv_dw_kernel(const TIn* __restrict__ x, const TIn* __restrict__ dy, float* __restrict__ dw, int T, int C,
               int64_t start, int F, int Hg, int Wd, Taps taps)
{
    __shared__ float red[8][MAXTAPS][33];
    const int cl = threadIdx.x & 31, pl = threadIdx.x >> 5;
    const int c = blockIdx.y * 32 + cl;
    const bool live = c < C;
    const int64_t npos = (int64_t)F * Hg * Wd;
    const int64_t p0 = (int64_t)blockIdx.x * DW_POS, p1 = live ? min(npos, p0 + DW_POS) : p0;
    const int64_t rowbase = (int64_t)blockIdx.z * T + start;
    float acc[MAXTAPS];
#pragma unroll
    for (int i = 0; i < MAXTAPS; ++i) acc[i] = 0.f;
    for (int64_t p = p0 + pl; p < p1; p += 8) {
        const int f = (int)(p / ((int64_t)Hg * Wd)), r = (int)((p / Wd) % Hg), s = (int)(p % Wd);
        const float g = to_f32(dy[(rowbase + p) * C + c]);
#pragma unroll
        for (int tp = 0; tp < MAXTAPS; ++tp) {
            if (tp >= taps.n) break;
            const int ff = f + taps.df[tp], rr = r + taps.dr[tp], ss = s + taps.ds[tp];
            if (ff < 0 || ff >= F || rr < 0 || rr >= Hg || ss < 0 || ss >= Wd) continue;
            acc[tp] = fmaf(g, to_f32(x[(rowbase + ((int64_t)ff * Hg + rr) * Wd + ss) * C + c]), acc[tp]);
        }
    }
#pragma unroll
    for (int tp = 0; tp < MAXTAPS; ++tp) red[pl][tp][cl] = acc[tp];
    __syncthreads();
    for (int e = threadIdx.x; e < taps.n * 32; e += 256) {
        const int tp = e / 32, ch = e % 32;
        if (blockIdx.y * 32 + ch >= C) continue;
        float s = 0.f;
#pragma unroll
        for (int l = 0; l < 8; ++l) s += red[l][tp][ch];
        atomicAdd(dw + (int64_t)(blockIdx.y * 32 + ch) * taps.n + tp, s);
    }
}

template <typename TIn>
cudaError_t launch_t(const void* x, const void* dy, float* dx, const float* w, float* dw, int B, int T, int C,
                     const ConvSeg& sg, int Kt, cudaStream_t s)
{
    const Taps taps = taps_for(sg.modality, Kt);
    const int F = sg.modality == MSC_VIDEO ? sg.F : 1;
    const int Hg = sg.modality == MSC_TEXT ? 1 : sg.Hgt;
    const int Wd = sg.Wid;
    const int64_t npos = (int64_t)F * Hg * Wd;
    ProfileScope prof("conv_bwd", s);
    {
        const int64_t n = npos * (C / 8);
        count_launch();
        conv_dx_kernel<TIn><<<dim3((unsigned)((n + 255) / 256), B), 256, 0, s>>>(
            (const TIn*)dy, w, dx, T, C, sg.start, F, Hg, Wd, taps);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (!dw) return cudaSuccess;
    count_launch();
    conv_dw_kernel<TIn><<<dim3((unsigned)((npos + DW_POS - 1) / DW_POS), (unsigned)((C + 31) / 32), B), 256, 0, s>>>(
        (const TIn*)x, (const TIn*)dy, dw, T, C, sg.start, F, Hg, Wd, taps);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_conv_backward_segment(const void* x, const void* dy, float* dx, const float* w, float* dw, int B,
                                         int T, int C, ElemType in_t, const ConvSeg& sg, int Kt, cudaStream_t s)
{
    if (in_t == ET_F32) return launch_t<float>(x, dy, dx, w, dw, B, T, C, sg, Kt, s);
    return launch_t<__nv_bfloat16>(x, dy, dx, w, dw, B, T, C, sg, Kt, s);
}

}  // namespace kda
