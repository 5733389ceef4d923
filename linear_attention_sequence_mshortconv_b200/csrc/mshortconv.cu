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

// ---- tiled kernel for image and video segments (bf16 input, C % 128 == 0) -----------
// One block (512 threads) = one head's 128 channels x a spatial tile of TR x TS
// positions, sweeping the frames of the segment.  Frames (with a one-position halo,
// zero outside the image) stream through a 4-slot ring in shared memory by cp.async:
// frame f+1 loads while frame f is computed from slots f-2, f-1, f (the video kernel is
// causal in time, so a frame is read by three consecutive steps and then recycled).
// Warp w owns channel half w & 1 and tile row w >> 1; lane l owns channels
// 64*(w & 1) + 2l, +1 (one 4-byte bf16 pair: a warp reads 128 contiguous bytes per
// position) for all TS = 16 positions of the row.  Its 27 (or 9) taps x 2 channels of
// weights live in registers; per (tau, a) it reads the 18 halo positions of one row
// once and applies the 3 taps to all 16 outputs with packed fp32 FMAs.  Every input
// element comes from L2/HBM about (TR+2)(TS+2)/(TR*TS) = 1.4 times.  The per-head L2
// norm (q, k) reduces 16 positions per warp with a transposing butterfly and the two
// channel halves through shared memory.
constexpr int kTThreads = 512;
constexpr int TR = 8, TS = 16;
constexpr int HALO_R = TR + 2, HALO_S = TS + 2;
constexpr int kNSlot = 4;
constexpr int kSlotBytes = HALO_R * HALO_S * kCB * 2;     // 46,080 B
constexpr int kTileSmem = kNSlot * kSlotBytes + 2 * TR * TS * 4;

struct TileArgs {
    const void* x[3];
    void* y[3];
    const float* w[3];
    int norm_D[3];
    int T, C, F, Hh, W, ntile_s;
    int64_t start;
};

__device__ __forceinline__ void cp_async16_zfill(void* smem, const void* gmem, bool valid)
{
    const unsigned sa = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    const int n = valid ? 16 : 0;   // src-size 0: the 16 bytes are zero-filled, nothing is read
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(sa), "l"(gmem), "r"(n) : "memory");
}

template <typename TOut> __device__ __forceinline__ void st_pair_out(TOut* p, float2 v);
template <> __device__ __forceinline__ void st_pair_out<__half>(__half* p, float2 v)
{
    *reinterpret_cast<__half2*>(p) = __floats2half2_rn(v.x, v.y);
}
template <> __device__ __forceinline__ void st_pair_out<__nv_bfloat16>(__nv_bfloat16* p, float2 v)
{
    *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(v.x, v.y);
}

template <typename TOut, int MOD>
__global__ void __launch_bounds__(kTThreads, 1)
conv_tile_kernel(const TileArgs args)
{
    extern __shared__ __align__(16) uint8_t csm[];
    constexpr int ntap = MOD == 2 ? 27 : 9;
    float* sRed = reinterpret_cast<float*>(csm + kNSlot * kSlotBytes);   // [2 halves][TR][TS]
    // blockIdx.z = tensor * Bn + b (tensors: the non-null entries of x[]); selects, not
    // a dynamic index into the parameter struct
    const int nt = (args.x[2] ? 3 : (args.x[1] ? 2 : 1));
    const int Bn = gridDim.z / nt;
    const int ti = blockIdx.z / Bn, b = blockIdx.z % Bn;
    const __nv_bfloat16* __restrict__ x =
        reinterpret_cast<const __nv_bfloat16*>(ti == 0 ? args.x[0] : ti == 1 ? args.x[1] : args.x[2]);
    TOut* __restrict__ y = reinterpret_cast<TOut*>(ti == 0 ? args.y[0] : ti == 1 ? args.y[1] : args.y[2]);
    const float* __restrict__ w = ti == 0 ? args.w[0] : ti == 1 ? args.w[1] : args.w[2];
    const int norm_D = ti == 0 ? args.norm_D[0] : ti == 1 ? args.norm_D[1] : args.norm_D[2];
    const int C = args.C, Hh = args.Hh, W = args.W, F = args.F;
    const int cbase = blockIdx.y * kCB;
    const int R0 = (blockIdx.x / args.ntile_s) * TR, S0 = (blockIdx.x % args.ntile_s) * TS;
    const int t = threadIdx.x, lane = t & 31, wp = t >> 5;
    const int hf = wp & 1, r = wp >> 1;                    // channel half, tile row
    const int c0 = hf * 64 + 2 * lane;                     // this thread's first channel in the block

    float2 wr[ntap];                                       // taps x (c0, c0 + 1)
#pragma unroll
    for (int tap = 0; tap < ntap; ++tap)
        wr[tap] = make_float2(w[(int64_t)(cbase + c0) * ntap + tap], w[(int64_t)(cbase + c0 + 1) * ntap + tap]);

    const int64_t HW = (int64_t)Hh * W;
    const __nv_bfloat16* xb = x + ((int64_t)b * args.T + args.start) * C + cbase;
    auto load_frame = [&](int f) {
        uint8_t* slot = csm + (f % kNSlot) * kSlotBytes;
        for (int i = t; i < HALO_R * HALO_S * 16; i += kTThreads) {
            const int oc = i & 15, pos = i >> 4;
            const int hr = pos / HALO_S, hs = pos % HALO_S;
            const int gr = R0 - 1 + hr, gs = S0 - 1 + hs;
            const bool valid = gr >= 0 && gr < Hh && gs >= 0 && gs < W;
            const __nv_bfloat16* src = valid ? xb + ((int64_t)f * HW + (int64_t)gr * W + gs) * C + oc * 8 : xb;
            cp_async16_zfill(slot + (pos * 16 + oc) * 16, src, valid);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    load_frame(0);
    for (int f = 0; f < F; ++f) {
        if (f + 1 < F) load_frame(f + 1);
        else asm volatile("cp.async.commit_group;" ::: "memory");   // keep the group count
        asm volatile("cp.async.wait_group 1;" ::: "memory");
        __syncthreads();
        float2 acc[TS];
#pragma unroll
        for (int j = 0; j < TS; ++j) acc[j] = make_float2(0.f, 0.f);
#pragma unroll
        for (int tau = 0; tau < (MOD == 2 ? 3 : 1); ++tau) {
            const int ff = (MOD == 2) ? f - 2 + tau : f;
            if (ff < 0) continue;
            const uint8_t* slot = csm + (ff % kNSlot) * kSlotBytes;
#pragma unroll
            for (int a = 0; a < 3; ++a) {
                const uint32_t* row = reinterpret_cast<const uint32_t*>(slot + (r + a) * HALO_S * 256) + (c0 >> 1);
                const int tap0 = (MOD == 2) ? (tau * 3 + a) * 3 : a * 3;
                // each halo position is converted once and feeds up to 3 outputs
#pragma unroll
                for (int k = 0; k < HALO_S; ++k) {
                    const uint32_t u = row[k * 64];
                    const float2 xv = make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
#pragma unroll
                    for (int e = 0; e < 3; ++e) {
                        const int j = k - e;
                        if (j >= 0 && j < TS) acc[j] = __ffma2_rn(wr[tap0 + e], xv, acc[j]);
                    }
                }
            }
        }
        if (norm_D > 0) {
            // sum of squares per position over this warp's 64 channels: a transposing
            // butterfly leaves position lane >> 1 in lanes 2p, 2p+1
            float v[TS];
#pragma unroll
            for (int j = 0; j < TS; ++j) v[j] = acc[j].x * acc[j].x + acc[j].y * acc[j].y;
#pragma unroll
            for (int m = 16, n = TS / 2; m >= 2; m >>= 1, n >>= 1) {
                const bool up = (lane & m) != 0;
#pragma unroll
                for (int k = 0; k < n; ++k) {
                    const float send = up ? v[k] : v[k + n];
                    const float keep = up ? v[k + n] : v[k];
                    v[k] = keep + __shfl_xor_sync(0xffffffffu, send, m);
                }
            }
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
            if ((lane & 1) == 0) sRed[(hf * TR + r) * TS + (lane >> 1)] = v[0];
            __syncthreads();
#pragma unroll
            for (int j = 0; j < TS; ++j) {
                const float ss = sRed[(0 * TR + r) * TS + j] + sRed[(1 * TR + r) * TS + j];
                const float inv = ss > 0.f ? rsqrtf(ss) : 0.f;
                acc[j] = make_float2(acc[j].x * inv, acc[j].y * inv);
            }
        }
        const int gr = R0 + r;
        if (gr < Hh) {
#pragma unroll
            for (int j = 0; j < TS; ++j) {
                const int gs = S0 + j;
                if (gs < W) {
                    const int64_t tok = args.start + (int64_t)f * HW + (int64_t)gr * W + gs;
                    st_pair_out<TOut>(y + ((int64_t)b * args.T + tok) * C + cbase + c0, acc[j]);
                }
            }
        }
        __syncthreads();   // slot (f+2) % 4 = (f-2) % 4 is refilled by the next step; sRed reused
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
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

template <typename TOut>
cudaError_t launch_tiled(int nt, const void* const* xs, void* const* ys, const float* const* ws,
                         const int* norm_Ds, int B, int T, int C, const ConvSeg& sg, cudaStream_t s)
{
    TileArgs a{};
    for (int i = 0; i < nt; ++i) {
        a.x[i] = xs[i];
        a.y[i] = ys[i];
        a.w[i] = ws[i];
        a.norm_D[i] = norm_Ds[i];
    }
    const bool video = sg.modality == MSC_VIDEO;
    a.T = T;
    a.C = C;
    a.F = video ? sg.F : 1;
    a.Hh = sg.Hgt;
    a.W = sg.Wid;
    a.start = sg.start;
    a.ntile_s = (sg.Wid + TS - 1) / TS;
    const int ntile_r = (sg.Hgt + TR - 1) / TR;
    if (a.F <= 0 || sg.Hgt <= 0 || sg.Wid <= 0 || B <= 0) return cudaSuccess;
    const dim3 grid((unsigned)(ntile_r * a.ntile_s), (unsigned)(C / kCB), (unsigned)(nt * B));
    ProfileScope prof("conv", s);
    count_launch();
    auto k = video ? conv_tile_kernel<TOut, 2> : conv_tile_kernel<TOut, 1>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kTileSmem);
    if (e != cudaSuccess) return e;
    k<<<grid, kTThreads, kTileSmem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_conv_segment_multi(int nt, const void* const* xs, void* const* ys, int B, int T, int C,
                                      ElemType in_t, ElemType out_t, const ConvSeg& seg, int Kt,
                                      const float* const* ws, const int* norm_Ds, cudaStream_t s)
{
    // image and video segments of bf16 input with whole 128-channel heads: the tiled
    // kernel, all tensors in one launch
    if (seg.modality != MSC_TEXT && in_t == ET_BF16 && C % kCB == 0 && nt >= 1 && nt <= 3) {
        if (out_t == ET_F16) return launch_tiled<__half>(nt, xs, ys, ws, norm_Ds, B, T, C, seg, s);
        if (out_t == ET_BF16) return launch_tiled<__nv_bfloat16>(nt, xs, ys, ws, norm_Ds, B, T, C, seg, s);
    }
    for (int i = 0; i < nt; ++i) {
        const cudaError_t e = launch_conv_segment(xs[i], ys[i], B, T, C, in_t, out_t, seg, Kt, ws[i], norm_Ds[i], s);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

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
