// Modality-aware short convolution (mShortConv), Chimera paper section 3.4.
//
// Depthwise, per segment of the packed [B, T, C] stream, zero padding inside the
// segment so that no kernel crosses a text/visual (or sample) boundary:
//   text  : 1-D causal, y[t] = sum_{j<Kt} w[c,j] x[t-(Kt-1)+j]
//   image : 3x3 spatial, y[r,s] = sum_{a,e} w[c,a,e] x[r-1+a, s-1+e]
//   video : 3x3x3, causal in time and symmetric in space,
//           y[f,r,s] = sum_{tau,a,e} w[c,tau,a,e] x[f-2+tau, r-1+a, s-1+e]
// Visual tokens are in the time-first raster order of Eq. 12 (m = f*H*W + r*W + s),
// so a spatial neighbour is a fixed token offset (+-1, +-W) and a temporal one is
// -H*W or -2*H*W: the kernel reads the packed buffer in place (no gather/scatter).
//
// Mapping: each thread owns 8 consecutive channels of one token (one 16-byte bf16
// vector), so a warp reads 512 contiguous bytes per tap; taps of neighbouring tokens
// hit L1/L2.  With norm_D > 0 the D/8 threads of one (token, head) are consecutive
// lanes of one warp and reduce the sum of squares with shuffles to L2-normalise the
// head vector before it is stored (the q/k prologue of the fused path).

#include "internal.h"

namespace kda {
namespace {

constexpr int kThreads = 256;

template <typename T> struct Vec8;
template <> struct Vec8<__nv_bfloat16> {
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float* f) {
        const uint4 u = *reinterpret_cast<const uint4*>(p);
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) { float2 t = __bfloat1622float2(h[i]); f[2 * i] = t.x; f[2 * i + 1] = t.y; }
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, const float* f) {
        uint4 u;
        __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
        *reinterpret_cast<uint4*>(p) = u;
    }
};
template <> struct Vec8<__half> {
    static __device__ __forceinline__ void store(__half* p, const float* f) {
        uint4 u;
        __half2* h = reinterpret_cast<__half2*>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) h[i] = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
        *reinterpret_cast<uint4*>(p) = u;
    }
};
template <> struct Vec8<float> {
    static __device__ __forceinline__ void load(const float* p, float* f) {
        const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
        f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    }
    static __device__ __forceinline__ void store(float* p, const float* f) {
        reinterpret_cast<float4*>(p)[0] = make_float4(f[0], f[1], f[2], f[3]);
        reinterpret_cast<float4*>(p)[1] = make_float4(f[4], f[5], f[6], f[7]);
    }
};

// MOD: 0 text, 1 image, 2 video.  NTAP = Kt (text), 9, 27.
template <typename TIn, typename TOut, int MOD>
__global__ void __launch_bounds__(kThreads)
conv_segment_kernel(const TIn* __restrict__ x, TOut* __restrict__ y, int T, int C,
                    int64_t start, int F, int Hh, int W, int Kt,
                    const float* __restrict__ w, int norm_D)
{
    const int groups = C >> 3;                       // 8-channel groups per token
    const int64_t len = (MOD == 0) ? (int64_t)W : (MOD == 1 ? (int64_t)Hh * W : (int64_t)F * Hh * W);
    const int64_t lin = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    const int b = blockIdx.y;
    const int64_t p = lin / groups;                  // token within the segment
    const int c0 = (int)(lin % groups) * 8;
    const bool active = p < len;

    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;

    if (active) {
        const TIn* xb = x + ((int64_t)b * T + start) * C + c0;
        const int ntap = (MOD == 0) ? Kt : (MOD == 1 ? 9 : 27);
        if (MOD == 0) {
            for (int j = 0; j < Kt; ++j) {
                const int64_t src = p - (Kt - 1) + j;
                if (src < 0) continue;
                float xv[8];
                Vec8<TIn>::load(xb + src * C, xv);
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i] = fmaf(w[(int64_t)(c0 + i) * ntap + j], xv[i], acc[i]);
            }
        } else {
            const int64_t HW = (int64_t)Hh * W;
            const int f = (MOD == 2) ? (int)(p / HW) : 0;
            const int r = (int)((p / W) % Hh), s = (int)(p % W);
            const int taus = (MOD == 2) ? 3 : 1;
            for (int tau = 0; tau < taus; ++tau) {
                const int ff = (MOD == 2) ? f - 2 + tau : 0;
                if (ff < 0) continue;
                for (int a = 0; a < 3; ++a) {
                    const int rr = r - 1 + a;
                    if (rr < 0 || rr >= Hh) continue;
                    for (int e = 0; e < 3; ++e) {
                        const int ss = s - 1 + e;
                        if (ss < 0 || ss >= W) continue;
                        const int tap = (MOD == 2) ? (tau * 3 + a) * 3 + e : a * 3 + e;
                        float xv[8];
                        Vec8<TIn>::load(xb + ((int64_t)ff * HW + (int64_t)rr * W + ss) * C, xv);
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            acc[i] = fmaf(w[(int64_t)(c0 + i) * ntap + tap], xv[i], acc[i]);
                    }
                }
            }
        }
    }
    if (norm_D > 0) {
        // sum of squares over the D/8 lanes that hold this (token, head)
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) ss = fmaf(acc[i], acc[i], ss);
        const int lanes = norm_D >> 3;
        for (int off = 1; off < lanes; off <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        const float inv = ss > 0.f ? rsqrtf(ss) : 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] *= inv;
    }
    if (active) Vec8<TOut>::store(y + ((int64_t)b * T + start + p) * C + c0, acc);
}

template <typename TIn, typename TOut>
cudaError_t launch_typed(const void* x, void* y, int B, int T, int C, const ConvSeg& sg, int Kt,
                         const float* w, int norm_D, cudaStream_t s)
{
    const int64_t len = sg.modality == MSC_TEXT ? (int64_t)sg.Wid
                      : sg.modality == MSC_IMAGE ? (int64_t)sg.Hgt * sg.Wid
                                                 : (int64_t)sg.F * sg.Hgt * sg.Wid;
    if (len <= 0 || B <= 0) return cudaSuccess;
    const int64_t threads = len * (C / 8);
    dim3 grid((unsigned)((threads + kThreads - 1) / kThreads), B);
    const TIn* xp = (const TIn*)x;
    TOut* yp = (TOut*)y;
    ProfileScope prof("conv", s);
    count_launch();
    switch (sg.modality) {
        case MSC_TEXT:
            conv_segment_kernel<TIn, TOut, 0><<<grid, kThreads, 0, s>>>(xp, yp, T, C, sg.start, 1, 1, sg.Wid, Kt, w, norm_D);
            break;
        case MSC_IMAGE:
            conv_segment_kernel<TIn, TOut, 1><<<grid, kThreads, 0, s>>>(xp, yp, T, C, sg.start, 1, sg.Hgt, sg.Wid, Kt, w, norm_D);
            break;
        default:
            conv_segment_kernel<TIn, TOut, 2><<<grid, kThreads, 0, s>>>(xp, yp, T, C, sg.start, sg.F, sg.Hgt, sg.Wid, Kt, w, norm_D);
            break;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_conv_segment(const void* x, void* y, int B, int T, int C, ElemType in_t,
                                ElemType out_t, const ConvSeg& seg, int Kt, const float* w,
                                int norm_D, cudaStream_t s)
{
    if (in_t == ET_F32 && out_t == ET_F32) return launch_typed<float, float>(x, y, B, T, C, seg, Kt, w, norm_D, s);
    if (in_t == ET_BF16 && out_t == ET_BF16)
        return launch_typed<__nv_bfloat16, __nv_bfloat16>(x, y, B, T, C, seg, Kt, w, norm_D, s);
    if (in_t == ET_BF16 && out_t == ET_F16)
        return launch_typed<__nv_bfloat16, __half>(x, y, B, T, C, seg, Kt, w, norm_D, s);
    if (in_t == ET_F32 && out_t == ET_F16) return launch_typed<float, __half>(x, y, B, T, C, seg, Kt, w, norm_D, s);
    return cudaErrorInvalidValue;
}

}  // namespace kda
