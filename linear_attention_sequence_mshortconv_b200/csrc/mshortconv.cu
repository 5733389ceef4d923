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
// vector), so a warp reads two 256-byte token rows per tap; taps of neighbouring
// tokens hit L1/L2.  With norm_D > 0 the D/8 threads of one (token, head) are
// consecutive lanes of one warp and reduce the sum of squares with shuffles to
// L2-normalise the head vector before it is stored (the q/k prologue of the fused path).

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

// One block = 16 consecutive tokens of a segment x 128 channels (when C is a
// multiple of 128; else 64 or 8 x ...).  Thread (token t >> 4, channel group t & 15)
// owns 8 channels.  The block's weights are staged in shared memory as [tap][channel]
// so the 16 threads of one channel group read them as two broadcast float4 loads per
// tap; the 16 lanes of one token hold a whole 128-channel head for the L2 norm.
constexpr int kCB = 128;                  // channels per block
constexpr int kTokPerBlk = kThreads / (kCB / 8);   // 16

template <typename TIn, typename TOut, int MOD>
__global__ void __launch_bounds__(kThreads)
conv_segment_kernel(const TIn* __restrict__ x, TOut* __restrict__ y, int T, int C,
                    int64_t start, int F, int Hh, int W, int Kt,
                    const float* __restrict__ w, int norm_D)
{
    __shared__ __align__(16) float sw_[27 * kCB];
    const int ntap = (MOD == 0) ? Kt : (MOD == 1 ? 9 : 27);
    const int cbase = blockIdx.y * kCB;
    const int ncb = min(kCB, C - cbase);          // channels in this block (multiple of 8)
    for (int i = threadIdx.x; i < ntap * kCB; i += kThreads) {
        const int tap = i / kCB, cc = i % kCB;
        sw_[i] = (cc < ncb) ? w[(int64_t)(cbase + cc) * ntap + tap] : 0.f;
    }
    __syncthreads();

    const int64_t len = (MOD == 0) ? (int64_t)W : (MOD == 1 ? (int64_t)Hh * W : (int64_t)F * Hh * W);
    const int g = threadIdx.x & 15, tk = threadIdx.x >> 4;
    const int64_t p = (int64_t)blockIdx.x * kTokPerBlk + tk;    // token within the segment
    const int b = blockIdx.z;
    const int cl = g * 8;                                       // channel offset in the block
    const bool active = p < len && cl < ncb;

    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    auto tap_fma = [&](int64_t src, int tap) {
        float xv[8];
        Vec8<TIn>::load(x + ((int64_t)b * T + start + src) * C + cbase + cl, xv);
        const float4 w0 = *reinterpret_cast<const float4*>(sw_ + tap * kCB + cl);
        const float4 w1 = *reinterpret_cast<const float4*>(sw_ + tap * kCB + cl + 4);
        acc[0] = fmaf(w0.x, xv[0], acc[0]); acc[1] = fmaf(w0.y, xv[1], acc[1]);
        acc[2] = fmaf(w0.z, xv[2], acc[2]); acc[3] = fmaf(w0.w, xv[3], acc[3]);
        acc[4] = fmaf(w1.x, xv[4], acc[4]); acc[5] = fmaf(w1.y, xv[5], acc[5]);
        acc[6] = fmaf(w1.z, xv[6], acc[6]); acc[7] = fmaf(w1.w, xv[7], acc[7]);
    };
    if (active) {
        if (MOD == 0) {
            for (int j = 0; j < Kt; ++j) {
                const int64_t src = p - (Kt - 1) + j;
                if (src >= 0) tap_fma(src, j);
            }
        } else {
            const int64_t HW = (int64_t)Hh * W;
            const int f = (MOD == 2) ? (int)(p / HW) : 0;
            const int r = (int)((p / W) % Hh), s = (int)(p % W);
#pragma unroll
            for (int tau = 0; tau < ((MOD == 2) ? 3 : 1); ++tau) {
                const int ff = (MOD == 2) ? f - 2 + tau : 0;
                if (ff < 0) continue;
#pragma unroll
                for (int a = 0; a < 3; ++a) {
                    const int rr = r - 1 + a;
                    if (rr < 0 || rr >= Hh) continue;
#pragma unroll
                    for (int e = 0; e < 3; ++e) {
                        const int ss = s - 1 + e;
                        if (ss < 0 || ss >= W) continue;
                        const int tap = (MOD == 2) ? (tau * 3 + a) * 3 + e : a * 3 + e;
                        tap_fma((int64_t)ff * HW + (int64_t)rr * W + ss, tap);
                    }
                }
            }
        }
    }
    if (norm_D > 0) {
        // sum of squares over the norm_D/8 lanes that hold this (token, head)
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) ss = fmaf(acc[i], acc[i], ss);
        for (int off = 1; off < (norm_D >> 3); off <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        const float inv = ss > 0.f ? rsqrtf(ss) : 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] *= inv;
    }
    if (active) Vec8<TOut>::store(y + ((int64_t)b * T + start + p) * C + cbase + cl, acc);
}

template <typename TIn, typename TOut>
cudaError_t launch_typed(const void* x, void* y, int B, int T, int C, const ConvSeg& sg, int Kt,
                         const float* w, int norm_D, cudaStream_t s)
{
    const int64_t len = sg.modality == MSC_TEXT ? (int64_t)sg.Wid
                      : sg.modality == MSC_IMAGE ? (int64_t)sg.Hgt * sg.Wid
                                                 : (int64_t)sg.F * sg.Hgt * sg.Wid;
    if (len <= 0 || B <= 0) return cudaSuccess;
    dim3 grid((unsigned)((len + kTokPerBlk - 1) / kTokPerBlk), (unsigned)((C + kCB - 1) / kCB), B);
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
