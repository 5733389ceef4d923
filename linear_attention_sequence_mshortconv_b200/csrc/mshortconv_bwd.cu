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
// dx: every (position, channel) is written by one thread (no atomics).  dw: each thread
// sums its rows in registers (one accumulator per tap), a block reduces its 8 warps in
// shared memory and adds its sums with one atomic per (channel, tap).  fp32 arithmetic;
// x, dy in fp32 or bf16.

#include "internal.h"

namespace kda {
namespace {

// Both kernels walk raster rows: a thread owns one row (f, r) of the segment box and
// two adjacent channels, and steps along s keeping, for every row the taps reach, a
// window of NS consecutive values in registers, so each step loads one new value per
// reached row (NF*NR of them) instead of one per tap.
//   NF = 3 (video: df = tau - 2) or 1;  NR = 3 (image, video: dr = a - 1) or 1;
//   NS = Kt (text: ds = j - (Kt-1)) or 3 (ds = e - 1).
// Tap numbering follows the weight layout: tap = (tau*NR + a)*NS + e.
template <typename TIn> struct Pair;
template <> struct Pair<float> {
    static __device__ __forceinline__ float2 ld(const float* p) { return *reinterpret_cast<const float2*>(p); }
};
template <> struct Pair<__nv_bfloat16> {
    static __device__ __forceinline__ float2 ld(const __nv_bfloat16* p)
    {
        const uint32_t u = *reinterpret_cast<const uint32_t*>(p);
        return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
    }
};

constexpr int SCH = 16;             // positions of a row per work item
constexpr int DX_ITEMS = 2;    // work items (row, run of SCH positions) per warp: dx
constexpr int DW_ITEMS = 2;

// dx: grid (ceil(items / (8*DX_ITEMS)), ceil(C / 64), B), 256 threads = 8 warps x
// 32 lanes; a work item is a run of SCH positions of one row (items = F*Hg*ceil(Wd/SCH));
// lane owns channels c, c + 1.  w: this segment's weight set [C][taps].
template <int NF, int NR, int NS, typename TIn>
__global__ void __launch_bounds__(256)
conv_dx_rows_kernel(const TIn* __restrict__ dy, const float* __restrict__ w, float* __restrict__ dx, int T, int C,
                    int64_t start, int F, int Hg, int Wd)
{
    constexpr int NT = NF * NR * NS;
    constexpr int M0 = NR == 3 ? -1 : 0;   // window origin: dy[s + M0 + m]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int c = (blockIdx.y * 32 + lane) * 2;
    if (c >= C) return;
    const int64_t rowbase = (int64_t)blockIdx.z * T + start;
    float2 wr[NT];
#pragma unroll
    for (int tp = 0; tp < NT; ++tp) wr[tp] = make_float2(w[(int64_t)c * NT + tp], w[(int64_t)(c + 1) * NT + tp]);
    const int nsc = (Wd + SCH - 1) / SCH, nitems = F * Hg * nsc;
    for (int q = 0; q < DX_ITEMS; ++q) {
        const int item = (blockIdx.x * 8 + warp) * DX_ITEMS + q;
        if (item >= nitems) break;
        const int row = item / nsc, s0 = (item % nsc) * SCH, s1 = min(Wd, s0 + SCH);
        const int f = row / Hg, r = row % Hg;
        // source rows of dy: (f + 2 - tau, r + 1 - a) for video, (f, r + 1 - a) for image
        const TIn* src[NF][NR];
#pragma unroll
        for (int tau = 0; tau < NF; ++tau)
#pragma unroll
            for (int a = 0; a < NR; ++a) {
                const int ff = NF == 3 ? f + 2 - tau : f, rr = NR == 3 ? r + 1 - a : r;
                src[tau][a] = (ff >= 0 && ff < F && rr >= 0 && rr < Hg)
                                  ? dy + (rowbase + ((int64_t)ff * Hg + rr) * Wd) * C + c : nullptr;
            }
        float2 win[NF][NR][NS];
#pragma unroll
        for (int tau = 0; tau < NF; ++tau)
#pragma unroll
            for (int a = 0; a < NR; ++a)
#pragma unroll
                for (int m = 0; m < NS; ++m) {
                    const int ss = s0 - 1 + M0 + m;   // the window of s = s0 - 1, shifted in at s0
                    win[tau][a][m] = (src[tau][a] && ss >= 0 && ss < Wd) ? Pair<TIn>::ld(src[tau][a] + (int64_t)ss * C)
                                                                         : make_float2(0.f, 0.f);
                }
        float* out = dx + (rowbase + ((int64_t)f * Hg + r) * Wd) * C + c;
#pragma unroll 4
        for (int s = s0; s < s1; ++s) {
            const int sn = s + M0 + NS - 1;   // the value entering the window
#pragma unroll
            for (int tau = 0; tau < NF; ++tau)
#pragma unroll
                for (int a = 0; a < NR; ++a) {
#pragma unroll
                    for (int m = 0; m < NS - 1; ++m) win[tau][a][m] = win[tau][a][m + 1];
                    win[tau][a][NS - 1] = (src[tau][a] && sn < Wd) ? Pair<TIn>::ld(src[tau][a] + (int64_t)sn * C)
                                                                   : make_float2(0.f, 0.f);
                }
            float2 acc = make_float2(0.f, 0.f);
#pragma unroll
            for (int tau = 0; tau < NF; ++tau)
#pragma unroll
                for (int a = 0; a < NR; ++a)
#pragma unroll
                    for (int e = 0; e < NS; ++e) {
                        const float2 wv = wr[(tau * NR + a) * NS + e], d = win[tau][a][NS - 1 - e];
                        acc.x = fmaf(wv.x, d.x, acc.x);
                        acc.y = fmaf(wv.y, d.y, acc.y);
                    }
            *reinterpret_cast<float2*>(out + (int64_t)s * C) = acc;
        }
    }
}

// dw: grid (ceil(items / (8*DW_ITEMS)), ceil(C / 64), B), the same work items.  Window
// over x rows (f - 2 + tau, r - 1 + a):
// x[s + D0 + m], m < NS, with D0 = -(NS-1) (text) or -1.
template <int NF, int NR, int NS, typename TIn>
__global__ void __launch_bounds__(256)
conv_dw_rows_kernel(const TIn* __restrict__ x, const TIn* __restrict__ dy, float* __restrict__ dw, int T, int C,
                    int64_t start, int F, int Hg, int Wd)
{
    constexpr int NT = NF * NR * NS;
    constexpr int D0 = NR == 3 ? -1 : -(NS - 1);
    extern __shared__ float red[];   // [8][NT][64]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int c = (blockIdx.y * 32 + lane) * 2;
    const bool live = c < C;
    const int64_t rowbase = (int64_t)blockIdx.z * T + start;
    float2 acc[NT];
#pragma unroll
    for (int tp = 0; tp < NT; ++tp) acc[tp] = make_float2(0.f, 0.f);
    const int nsc = (Wd + SCH - 1) / SCH, nitems = F * Hg * nsc;
    for (int q = 0; q < DW_ITEMS && live; ++q) {
        const int item = (blockIdx.x * 8 + warp) * DW_ITEMS + q;
        if (item >= nitems) break;
        const int row = item / nsc, s0 = (item % nsc) * SCH, s1 = min(Wd, s0 + SCH);
        const int f = row / Hg, r = row % Hg;
        const TIn* src[NF][NR];
#pragma unroll
        for (int tau = 0; tau < NF; ++tau)
#pragma unroll
            for (int a = 0; a < NR; ++a) {
                const int ff = NF == 3 ? f - 2 + tau : f, rr = NR == 3 ? r - 1 + a : r;
                src[tau][a] = (ff >= 0 && ff < F && rr >= 0 && rr < Hg)
                                  ? x + (rowbase + ((int64_t)ff * Hg + rr) * Wd) * C + c : nullptr;
            }
        float2 win[NF][NR][NS];
#pragma unroll
        for (int tau = 0; tau < NF; ++tau)
#pragma unroll
            for (int a = 0; a < NR; ++a)
#pragma unroll
                for (int m = 0; m < NS; ++m) {
                    const int ss = s0 - 1 + D0 + m;
                    win[tau][a][m] = (src[tau][a] && ss >= 0 && ss < Wd) ? Pair<TIn>::ld(src[tau][a] + (int64_t)ss * C)
                                                                         : make_float2(0.f, 0.f);
                }
        const TIn* g = dy + (rowbase + ((int64_t)f * Hg + r) * Wd) * C + c;
#pragma unroll 4
        for (int s = s0; s < s1; ++s) {
            const int sn = s + D0 + NS - 1;
#pragma unroll
            for (int tau = 0; tau < NF; ++tau)
#pragma unroll
                for (int a = 0; a < NR; ++a) {
#pragma unroll
                    for (int m = 0; m < NS - 1; ++m) win[tau][a][m] = win[tau][a][m + 1];
                    win[tau][a][NS - 1] = (src[tau][a] && sn >= 0 && sn < Wd)
                                              ? Pair<TIn>::ld(src[tau][a] + (int64_t)sn * C) : make_float2(0.f, 0.f);
                }
            const float2 gv = Pair<TIn>::ld(g + (int64_t)s * C);
#pragma unroll
            for (int tau = 0; tau < NF; ++tau)
#pragma unroll
                for (int a = 0; a < NR; ++a)
#pragma unroll
                    for (int e = 0; e < NS; ++e) {
                        float2& ac = acc[(tau * NR + a) * NS + e];
                        const float2 xv = win[tau][a][e];
                        ac.x = fmaf(gv.x, xv.x, ac.x);
                        ac.y = fmaf(gv.y, xv.y, ac.y);
                    }
        }
    }
#pragma unroll
    for (int tp = 0; tp < NT; ++tp) {
        red[(warp * NT + tp) * 64 + 2 * lane] = acc[tp].x;
        red[(warp * NT + tp) * 64 + 2 * lane + 1] = acc[tp].y;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < NT * 64; e += 256) {
        const int tp = e / 64, ch = e % 64;
        const int cc = blockIdx.y * 64 + ch;
        if (cc >= C) continue;
        float sum = 0.f;
#pragma unroll
        for (int l = 0; l < 8; ++l) sum += red[(l * NT + tp) * 64 + ch];
        atomicAdd(dw + (int64_t)cc * NT + tp, sum);
    }
}

// ---- image and video segments: shared-memory tiles ----------------------------------------
// A block owns 8 rows x 16 positions of one frame and 64 channels (8 warps = rows, lane =
// channel pair).  It stages the tile it reads, with its halo, by 16-byte loads from all
// threads (zero outside the box): NF frames x 10 rows x 18 positions x 64 channels.
// Each warp then walks its row along s with a 3-value register window per reached
// (frame, row), 9 shared loads per step for 27 taps.
constexpr int TR = 8, TS = 16, HR = TR + 2, HS = TS + 2;

template <typename TIn> struct PairT;
template <> struct PairT<float> {
    using type = float2;
    static __device__ __forceinline__ float2 f2(float2 v) { return v; }
};
template <> struct PairT<__nv_bfloat16> {
    using type = uint32_t;
    static __device__ __forceinline__ float2 f2(uint32_t u)
    {
        return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
    }
};

// tile[(j*HR + i)*HS + m][32] <- src frame f0 + j, row r0 + i, position s0 + m (64 channels
// from c0), for j < nf
template <typename TIn>
__device__ __forceinline__ void stage_tile(typename PairT<TIn>::type* tile, const TIn* src, int64_t rowbase, int C,
                                           int c0, int F, int Hg, int Wd, int f0, int r0, int s0, int nf)
{
    constexpr int VPP = 64 * (int)sizeof(TIn) / 16;   // 16-byte vectors per position
    const int n = nf * HR * HS * VPP;
    for (int e = threadIdx.x; e < n; e += 256) {
        const int v = e % VPP, pos = e / VPP;
        const int m = pos % HS, i = (pos / HS) % HR, j = pos / (HS * HR);
        const int ff = f0 + j, rr = r0 + i, ss = s0 + m;
        const int cc = c0 + v * (16 / (int)sizeof(TIn));
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        if (ff >= 0 && ff < F && rr >= 0 && rr < Hg && ss >= 0 && ss < Wd && cc < C)
            val = *reinterpret_cast<const uint4*>(src + (rowbase + ((int64_t)ff * Hg + rr) * Wd + ss) * C + cc);
        reinterpret_cast<uint4*>(tile + (size_t)pos * 32)[v] = val;
    }
}

template <int NF, typename TIn>
__host__ __device__ constexpr int tile_bytes() { return NF * HR * HS * 32 * (int)sizeof(typename PairT<TIn>::type); }

// dx[f, r, s] = sum_{tau,a,e} w[tau,a,e] dy[f + 2 - tau, r + 1 - a, s + 1 - e] (video;
// image: tau = 2 only).  grid (ceil(Wd/16) * ceil(Hg/8) * F, ceil(C/64), B).
template <int NF, typename TIn>
__global__ void __launch_bounds__(256, 2)
conv_dx_tile_kernel(const TIn* __restrict__ dy, const float* __restrict__ w, float* __restrict__ dx, int T, int C,
                    int64_t start, int F, int Hg, int Wd)
{
    using PT = typename PairT<TIn>::type;
    constexpr int NT = NF * 9;
    extern __shared__ __align__(16) unsigned char tsm[];
    PT* tile = reinterpret_cast<PT*>(tsm);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nsx = (Wd + TS - 1) / TS, nrx = (Hg + TR - 1) / TR;
    const int bx = blockIdx.x;
    const int sx = bx % nsx, rx = (bx / nsx) % nrx, f = bx / (nsx * nrx);
    const int s0 = sx * TS, r0 = rx * TR, c0 = blockIdx.y * 64;
    const int64_t rowbase = (int64_t)blockIdx.z * T + start;
    // dy frames f .. f + NF - 1 (tile frame j = 2 - tau), rows r0-1 .., positions s0-1 ..
    stage_tile<TIn>(tile, dy, rowbase, C, c0, F, Hg, Wd, f, r0 - 1, s0 - 1, NF);
    const int c = c0 + 2 * lane;
    float2 wr[NT];
#pragma unroll
    for (int tp = 0; tp < NT; ++tp)
        wr[tp] = c < C ? make_float2(w[(int64_t)c * NT + tp], w[(int64_t)(c + 1) * NT + tp]) : make_float2(0.f, 0.f);
    __syncthreads();
    const int r = r0 + warp;
    if (r >= Hg || c >= C) return;
    // window over tile positions m = (s - s0) + 2 - e, e = 0..2 -> win[.][k] = tile m = (s - s0) + k
    float2 win[NF][3][3];
#pragma unroll
    for (int j = 0; j < NF; ++j)
#pragma unroll
        for (int a = 0; a < 3; ++a)
#pragma unroll
            for (int k = 0; k < 2; ++k)
                win[j][a][k + 1] = PairT<TIn>::f2(tile[((j * HR + warp + 2 - a) * HS + k) * 32 + lane]);
    float* out = dx + (rowbase + ((int64_t)f * Hg + r) * Wd) * C + c;
    const int s1 = min(TS, Wd - s0);
#pragma unroll 4
    for (int ls = 0; ls < s1; ++ls) {
        float2 acc = make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < NF; ++j)
#pragma unroll
            for (int a = 0; a < 3; ++a) {
                win[j][a][0] = win[j][a][1];
                win[j][a][1] = win[j][a][2];
                win[j][a][2] = PairT<TIn>::f2(tile[((j * HR + warp + 2 - a) * HS + ls + 2) * 32 + lane]);
                const int tau = NF == 3 ? 2 - j : 2;   // image: the single frame is tau = 2's slot
#pragma unroll
                for (int e = 0; e < 3; ++e) {
                    const float2 wv = wr[((NF == 3 ? tau : 0) * 3 + a) * 3 + e], d = win[j][a][2 - e];
                    acc.x = fmaf(wv.x, d.x, acc.x);
                    acc.y = fmaf(wv.y, d.y, acc.y);
                }
            }
        *reinterpret_cast<float2*>(out + (int64_t)(s0 + ls) * C) = acc;
    }
}

// dw[c, tau, a, e] += sum dy[f, r, s] x[f - 2 + tau, r - 1 + a, s - 1 + e]; a block sweeps
// all frames of its (8 x 16) spatial tile and 64 channels, then reduces its 8 warps and
// adds with one atomic per (channel, tap).  grid (ceil(Wd/16) * ceil(Hg/8), ceil(C/64), B).
template <int NF, typename TIn>
__global__ void __launch_bounds__(256)
conv_dw_tile_kernel(const TIn* __restrict__ x, const TIn* __restrict__ dy, float* __restrict__ dw, int T, int C,
                    int64_t start, int F, int Hg, int Wd)
{
    using PT = typename PairT<TIn>::type;
    constexpr int NT = NF * 9;
    extern __shared__ __align__(16) unsigned char tsm[];
    PT* tile = reinterpret_cast<PT*>(tsm);                                   // x: NF frames
    PT* gt = reinterpret_cast<PT*>(tsm + tile_bytes<NF, TIn>());           // dy: 1 frame
    float* red = reinterpret_cast<float*>(tsm);                             // reused at the end
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nsx = (Wd + TS - 1) / TS;
    const int sx = blockIdx.x % nsx, rx = blockIdx.x / nsx;
    const int s0 = sx * TS, r0 = rx * TR, c0 = blockIdx.y * 64;
    const int64_t rowbase = (int64_t)blockIdx.z * T + start;
    const int c = c0 + 2 * lane, r = r0 + warp;
    const bool live = c < C && r < Hg;
    const int s1 = min(TS, Wd - s0);
    float2 acc[NT];
#pragma unroll
    for (int tp = 0; tp < NT; ++tp) acc[tp] = make_float2(0.f, 0.f);
    for (int f = 0; f < F; ++f) {
        __syncthreads();   // the previous frame's reads are done
        stage_tile<TIn>(tile, x, rowbase, C, c0, F, Hg, Wd, f - (NF - 1), r0 - 1, s0 - 1, NF);
        stage_tile<TIn>(gt, dy, rowbase, C, c0, F, Hg, Wd, f, r0 - 1, s0 - 1, 1);
        __syncthreads();
        if (!live) continue;
        // x window: win[j][a][k] = tile position m = ls + k (s - 1 + e with e = k)
        float2 win[NF][3][3];
#pragma unroll
        for (int j = 0; j < NF; ++j)
#pragma unroll
            for (int a = 0; a < 3; ++a)
#pragma unroll
                for (int k = 0; k < 2; ++k)
                    win[j][a][k + 1] = PairT<TIn>::f2(tile[((j * HR + warp + a) * HS + k) * 32 + lane]);
#pragma unroll 2
        for (int ls = 0; ls < s1; ++ls) {
            const float2 g = PairT<TIn>::f2(gt[((warp + 1) * HS + ls + 1) * 32 + lane]);
#pragma unroll
            for (int j = 0; j < NF; ++j)
#pragma unroll
                for (int a = 0; a < 3; ++a) {
                    win[j][a][0] = win[j][a][1];
                    win[j][a][1] = win[j][a][2];
                    win[j][a][2] = PairT<TIn>::f2(tile[((j * HR + warp + a) * HS + ls + 2) * 32 + lane]);
#pragma unroll
                    for (int e = 0; e < 3; ++e) {
                        float2& ac = acc[(j * 3 + a) * 3 + e];
                        ac.x = fmaf(g.x, win[j][a][e].x, ac.x);
                        ac.y = fmaf(g.y, win[j][a][e].y, ac.y);
                    }
                }
        }
    }
    __syncthreads();
#pragma unroll
    for (int tp = 0; tp < NT; ++tp) {
        red[(warp * NT + tp) * 64 + 2 * lane] = live ? acc[tp].x : 0.f;
        red[(warp * NT + tp) * 64 + 2 * lane + 1] = live ? acc[tp].y : 0.f;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < NT * 64; e += 256) {
        const int tp = e / 64, ch = e % 64;
        if (c0 + ch >= C) continue;
        float sum = 0.f;
#pragma unroll
        for (int l = 0; l < 8; ++l) sum += red[(l * NT + tp) * 64 + ch];
        // image: tap (a, e) is tp; video: tile frame j = tau
        atomicAdd(dw + (int64_t)(c0 + ch) * NT + tp, sum);
    }
}

template <int NF, typename TIn>
cudaError_t launch_tiles(const void* x, const void* dy, float* dx, const float* w, float* dw, int B, int T, int C,
                         int64_t start, int F, int Hg, int Wd, cudaStream_t s)
{
    const int nsx = (Wd + TS - 1) / TS, nrx = (Hg + TR - 1) / TR;
    const unsigned cb = (unsigned)((C + 63) / 64);
    {
        auto kern = conv_dx_tile_kernel<NF, TIn>;
        const int smem = tile_bytes<NF, TIn>();
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        count_launch();
        kern<<<dim3((unsigned)(nsx * nrx * F), cb, B), 256, smem, s>>>((const TIn*)dy, w, dx, T, C, start, F, Hg, Wd);
        e = cudaGetLastError();
        if (e != cudaSuccess || !dw) return e;
    }
    auto kern = conv_dw_tile_kernel<NF, TIn>;
    const int smem = max(tile_bytes<NF, TIn>() + tile_bytes<1, TIn>(), 8 * NF * 9 * 64 * (int)sizeof(float));
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    count_launch();
    kern<<<dim3((unsigned)(nsx * nrx), cb, B), 256, smem, s>>>((const TIn*)x, (const TIn*)dy, dw, T, C, start, F, Hg, Wd);
    return cudaGetLastError();
}

template <int NF, int NR, int NS, typename TIn>
cudaError_t launch_rows(const void* x, const void* dy, float* dx, const float* w, float* dw, int B, int T, int C,
                        int64_t start, int F, int Hg, int Wd, cudaStream_t s)
{
    const int64_t nitems = (int64_t)F * Hg * ((Wd + SCH - 1) / SCH);
    const dim3 grid((unsigned)((nitems + 8 * DX_ITEMS - 1) / (8 * DX_ITEMS)), (unsigned)((C + 63) / 64), B);
    const dim3 grid_w((unsigned)((nitems + 8 * DW_ITEMS - 1) / (8 * DW_ITEMS)), (unsigned)((C + 63) / 64), B);
    count_launch();
    conv_dx_rows_kernel<NF, NR, NS, TIn><<<grid, 256, 0, s>>>((const TIn*)dy, w, dx, T, C, start, F, Hg, Wd);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || !dw) return e;
    constexpr int NT = NF * NR * NS;
    const int smem = 8 * NT * 64 * (int)sizeof(float);
    auto kern = conv_dw_rows_kernel<NF, NR, NS, TIn>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    count_launch();
    kern<<<grid_w, 256, smem, s>>>((const TIn*)x, (const TIn*)dy, dw, T, C, start, F, Hg, Wd);
    return cudaGetLastError();
}

template <typename TIn>
cudaError_t launch_t(const void* x, const void* dy, float* dx, const float* w, float* dw, int B, int T, int C,
                     const ConvSeg& sg, int Kt, cudaStream_t s)
{
    ProfileScope prof("conv_bwd", s);
    if (sg.modality == MSC_VIDEO)
        return launch_tiles<3, TIn>(x, dy, dx, w, dw, B, T, C, sg.start, sg.F, sg.Hgt, sg.Wid, s);
    if (sg.modality == MSC_IMAGE)
        return launch_tiles<1, TIn>(x, dy, dx, w, dw, B, T, C, sg.start, 1, sg.Hgt, sg.Wid, s);
    switch (Kt) {
        case 1: return launch_rows<1, 1, 1, TIn>(x, dy, dx, w, dw, B, T, C, sg.start, 1, 1, sg.Wid, s);
        case 2: return launch_rows<1, 1, 2, TIn>(x, dy, dx, w, dw, B, T, C, sg.start, 1, 1, sg.Wid, s);
        case 3: return launch_rows<1, 1, 3, TIn>(x, dy, dx, w, dw, B, T, C, sg.start, 1, 1, sg.Wid, s);
        case 4: return launch_rows<1, 1, 4, TIn>(x, dy, dx, w, dw, B, T, C, sg.start, 1, 1, sg.Wid, s);
        case 5: return launch_rows<1, 1, 5, TIn>(x, dy, dx, w, dw, B, T, C, sg.start, 1, 1, sg.Wid, s);
        case 6: return launch_rows<1, 1, 6, TIn>(x, dy, dx, w, dw, B, T, C, sg.start, 1, 1, sg.Wid, s);
        case 7: return launch_rows<1, 1, 7, TIn>(x, dy, dx, w, dw, B, T, C, sg.start, 1, 1, sg.Wid, s);
        case 8: return launch_rows<1, 1, 8, TIn>(x, dy, dx, w, dw, B, T, C, sg.start, 1, 1, sg.Wid, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_conv_backward_segment(const void* x, const void* dy, float* dx, const float* w, float* dw, int B,
                                         int T, int C, ElemType in_t, const ConvSeg& sg, int Kt, cudaStream_t s)
{
    if (in_t == ET_F32) return launch_t<float>(x, dy, dx, w, dw, B, T, C, sg, Kt, s);
    return launch_t<__nv_bfloat16>(x, dy, dx, w, dw, B, T, C, sg, Kt, s);
}

}  // namespace kda
