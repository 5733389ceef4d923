// Chunkwise KDA forward on CUDA cores, fp32 arithmetic throughout.
//
// This is the path for fp32 inputs (where tensor-core operands would not meet an
// fp32 accuracy bar) and for every shape the tensor-core path does not cover.
//
// Chunkwise form of Eq. 14 (Chimera paper, section 3.3).  The paper only says the KDA
// kernel is "chunked"; the algebra below is derived from Eq. 14 itself.  Inside a
// chunk of C tokens with state S0 on entry, let b_i = sum_{r<=i} g_r (per channel,
// fp32) and u_i = beta_i (v_i - (D_i S_{i-1})^T k_i), so S_i = D_i S_{i-1} + k_i u_i^T.
// Unrolling:
//   u_i + beta_i sum_{j<i} (k_i . (e^{b_i - b_j} k_j)) u_j = beta_i (v_i - S0^T (e^{b_i} k_i))
//   o_i = S0^T (e^{b_i} q_i) + sum_{j<=i} (q_i . (e^{b_i - b_j} k_j)) u_j
//   S_C = Diag(e^{b_C}) S0 + sum_j (e^{b_C - b_j} k_j) u_j^T
// Every exponent above is <= 0 (b is non-increasing along the chunk), so no factor
// can overflow whatever the gates are.  The pairwise exponentials are formed
// directly, which costs C*C*Dk/2 exp() per chunk but keeps the fp32 path exact to
// rounding for any g.
//
// Grid: (Dv/32, H, B); each CTA owns 32 state columns of one (b, h): the columns of
// S evolve independently under Eq. 14 (every term acts on S from the left or adds
// k v^T), so no cross-CTA exchange is needed.

#include "internal.h"

namespace kda {
namespace {

constexpr int kThreads = 256;
constexpr int kDvt = 32;  // state columns per CTA

template <typename TIn, typename TG, typename TOut, int DK>
__global__ void __launch_bounds__(kThreads)
kda_generic_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k,
                   const TIn* __restrict__ v, const TG* __restrict__ g,
                   const TG* __restrict__ beta, const float* __restrict__ S0,
                   TOut* __restrict__ o, float* __restrict__ ST, int T, int H, int Dv, int C)
{
    const int col0 = blockIdx.x * kDvt;
    const int h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x;
    constexpr int LD = DK + 1;
    const int LDC = C + 1;

    extern __shared__ float sm[];
    float* sQ = sm;                   // [C][LD]  q, then e^{b} q
    float* sK = sQ + C * LD;          // [C][LD]  k, then e^{b} k
    float* sB = sK + C * LD;          // [C][LD]  g -> b (cumulative), then e^{b_C - b} k
    float* sA = sB + C * LD;          // [C][LDC] beta_i k_i.(e^{b_i-b_j} k_j), j < i
    float* sP = sA + C * LDC;         // [C][LDC] q_i.(e^{b_i-b_j} k_j), j <= i
    float* sV = sP + C * LDC;         // [C][kDvt+1] v, then rhs, then u
    float* sO = sV + C * (kDvt + 1);  // [C][kDvt]
    float* sS = sO + C * kDvt;        // [DK][kDvt] state columns
    float* sBeta = sS + DK * kDvt;    // [C]
    float* sBC = sBeta + C;           // [DK]  b at the chunk's last token

    const int64_t strk = (int64_t)H * DK, strv = (int64_t)H * Dv;
    const int64_t sbase = ((int64_t)b * H + h) * DK * Dv + col0;

    for (int idx = tid; idx < DK * kDvt; idx += kThreads) {
        const int c = idx / kDvt, j = idx % kDvt;
        sS[idx] = S0 ? S0[sbase + (int64_t)c * Dv + j] : 0.f;
    }

    for (int t0 = 0; t0 < T; t0 += C) {
        const int Ct = min(C, T - t0);
        __syncthreads();
        // 1. load the chunk (rows past the end act as k = q = v = g = beta = 0)
        for (int idx = tid; idx < C * DK; idx += kThreads) {
            const int i = idx / DK, c = idx % DK;
            float qq = 0.f, kk = 0.f, gg = 0.f;
            if (i < Ct) {
                const int64_t off = ((int64_t)b * T + t0 + i) * strk + (int64_t)h * DK + c;
                qq = to_f32(q[off]); kk = to_f32(k[off]); gg = to_f32(g[off]);
            }
            sQ[i * LD + c] = qq; sK[i * LD + c] = kk; sB[i * LD + c] = gg;
        }
        for (int idx = tid; idx < C * kDvt; idx += kThreads) {
            const int i = idx / kDvt, j = idx % kDvt;
            float vv = 0.f;
            if (i < Ct) vv = to_f32(v[((int64_t)b * T + t0 + i) * strv + (int64_t)h * Dv + col0 + j]);
            sV[i * (kDvt + 1) + j] = vv;
        }
        for (int i = tid; i < C; i += kThreads)
            sBeta[i] = (i < Ct) ? to_f32(beta[((int64_t)b * T + t0 + i) * H + h]) : 0.f;
        __syncthreads();
        // 2. per-channel cumulative log-decay
        for (int c = tid; c < DK; c += kThreads) {
            float run = 0.f;
            for (int i = 0; i < C; ++i) { run += sB[i * LD + c]; sB[i * LD + c] = run; }
            sBC[c] = run;
        }
        __syncthreads();
        // 3. pairwise decayed key/query products
        for (int idx = tid; idx < C * C; idx += kThreads) {
            const int i = idx / C, j = idx % C;
            float aa = 0.f, pp = 0.f;
            if (j <= i) {
                const float* ki = sK + i * LD; const float* qi = sQ + i * LD;
                const float* kj = sK + j * LD;
                const float* bi = sB + i * LD; const float* bj = sB + j * LD;
                for (int c = 0; c < DK; ++c) {
                    const float kd = kj[c] * expf(bi[c] - bj[c]);
                    aa = fmaf(ki[c], kd, aa);
                    pp = fmaf(qi[c], kd, pp);
                }
            }
            sA[i * LDC + j] = (j < i) ? sBeta[i] * aa : 0.f;
            sP[i * LDC + j] = pp;
        }
        __syncthreads();
        // 4. e^{b} q, e^{b} k and e^{b_C - b} k
        for (int idx = tid; idx < C * DK; idx += kThreads) {
            const int i = idx / DK, c = idx % DK;
            const float bb = sB[i * LD + c];
            const float e = expf(bb), et = expf(sBC[c] - bb);
            const float kk = sK[i * LD + c];
            sQ[i * LD + c] *= e;
            sK[i * LD + c] = kk * e;
            sB[i * LD + c] = kk * et;
        }
        __syncthreads();
        // 5. rhs = beta (v - (e^b k) S0) and the inter-chunk part of the output
        for (int idx = tid; idx < C * kDvt; idx += kThreads) {
            const int i = idx / kDvt, j = idx % kDvt;
            float ks = 0.f, qs = 0.f;
            for (int c = 0; c < DK; ++c) {
                const float s = sS[c * kDvt + j];
                ks = fmaf(sK[i * LD + c], s, ks);
                qs = fmaf(sQ[i * LD + c], s, qs);
            }
            float* vp = sV + i * (kDvt + 1) + j;
            *vp = sBeta[i] * (*vp - ks);
            sO[i * kDvt + j] = qs;
        }
        __syncthreads();
        // 6. forward substitution (I + A) u = rhs, one row at a time
        {
            const int part = tid & 7, j = tid >> 3;  // 8 partial sums per column
            for (int i = 1; i < C; ++i) {
                float s = 0.f;
                for (int m = part; m < i; m += 8)
                    s = fmaf(sA[i * LDC + m], sV[m * (kDvt + 1) + j], s);
                s += __shfl_xor_sync(0xffffffffu, s, 1);
                s += __shfl_xor_sync(0xffffffffu, s, 2);
                s += __shfl_xor_sync(0xffffffffu, s, 4);
                if (part == 0) sV[i * (kDvt + 1) + j] -= s;
                __syncthreads();
            }
        }
        // 7. outputs: o_i = (e^b q_i) S0 + sum_{m<=i} P_im u_m
        for (int idx = tid; idx < C * kDvt; idx += kThreads) {
            const int i = idx / kDvt, j = idx % kDvt;
            if (i >= Ct) continue;
            float acc = sO[i * kDvt + j];
            for (int m = 0; m <= i; ++m) acc = fmaf(sP[i * LDC + m], sV[m * (kDvt + 1) + j], acc);
            o[((int64_t)b * T + t0 + i) * strv + (int64_t)h * Dv + col0 + j] = from_f32<TOut>(acc);
        }
        // 8. state to the chunk end: Diag(e^{b_C}) S0 + sum_i (e^{b_C - b_i} k_i) u_i^T
        for (int idx = tid; idx < DK * kDvt; idx += kThreads) {
            const int c = idx / kDvt, j = idx % kDvt;
            float acc = expf(sBC[c]) * sS[idx];
            for (int i = 0; i < C; ++i) acc = fmaf(sB[i * LD + c], sV[i * (kDvt + 1) + j], acc);
            sS[idx] = acc;
        }
    }
    __syncthreads();
    if (ST) {
        for (int idx = tid; idx < DK * kDvt; idx += kThreads) {
            const int c = idx / kDvt, j = idx % kDvt;
            ST[sbase + (int64_t)c * Dv + j] = sS[idx];
        }
    }
}

// Chunks of 128 tokens.  The two C x C pair matrices alone would take 128 KB in fp32, so
// A and P share one array (A_ij below the diagonal, P_ij at [j][i] above it, P_ii apart)
// and the key channels are taken in blocks of KB = 32: each block adds its share of A, P
// and of the inter-chunk terms (e^b k) S0 and (e^b q) S0; after the substitution the state
// update reads each block's k and g once more (from L2) for e^{b_C - b} k.
constexpr int kWideC = 128;
constexpr int kKB = 32;
static_assert(kThreads == 8 * kKB, "the cumulative sum takes 8 threads per channel");

template <typename TIn, typename TG, typename TOut, int DK>
__global__ void __launch_bounds__(kThreads)
kda_generic_wide_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k,
                        const TIn* __restrict__ v, const TG* __restrict__ g,
                        const TG* __restrict__ beta, const float* __restrict__ S0,
                        TOut* __restrict__ o, float* __restrict__ ST, int T, int H, int Dv)
{
    constexpr int C = kWideC, KB = kKB, LDB = KB + 1, LDC = C + 1, LDV = kDvt + 1;
    const int col0 = blockIdx.x * kDvt;
    const int h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x;

    extern __shared__ float sm[];
    float* sAP = sm;                  // [C][LDC] A_ij (j < i) and P_ij at [j][i] (j < i)
    float* sPd = sAP + C * LDC;       // [C]      P_ii
    float* sQ = sPd + C;              // [C][LDB] q of the channel block, then e^b q
    float* sK = sQ + C * LDB;         // [C][LDB] k, then e^b k (or e^{b_C - b} k)
    float* sB = sK + C * LDB;         // [C][LDB] g -> b (cumulative)
    float* sV = sB + C * LDB;         // [C][LDV] v, then v - (e^b k) S0, then rhs, then u
    float* sO = sV + C * LDV;         // [C][kDvt] (e^b q) S0
    float* sS = sO + C * kDvt;        // [DK][kDvt] state columns
    float* sBeta = sS + DK * kDvt;    // [C]
    float* sBC = sBeta + C;           // [DK] b at the chunk's last token

    const int64_t strk = (int64_t)H * DK, strv = (int64_t)H * Dv;
    const int64_t sbase = ((int64_t)b * H + h) * DK * Dv + col0;

    for (int idx = tid; idx < DK * kDvt; idx += kThreads) {
        const int c = idx / kDvt, j = idx % kDvt;
        sS[idx] = S0 ? S0[sbase + (int64_t)c * Dv + j] : 0.f;
    }

    // k, g (and q) of channels [c0, c0 + KB) for the chunk's rows (zero past its end), g
    // turned into the cumulative b; ends with the block synchronised.  The two calls per
    // chunk and block sum in the same order, so they give the same b.
    auto load_block = [&](int t0, int Ct, int c0, bool with_q) {
        for (int idx = tid; idx < C * KB; idx += kThreads) {
            const int i = idx / KB, c = idx % KB;
            float qq = 0.f, kk = 0.f, gg = 0.f;
            if (i < Ct) {
                const int64_t off = ((int64_t)b * T + t0 + i) * strk + (int64_t)h * DK + c0 + c;
                if (with_q) qq = to_f32(q[off]);
                kk = to_f32(k[off]);
                gg = to_f32(g[off]);
            }
            if (with_q) sQ[i * LDB + c] = qq;
            sK[i * LDB + c] = kk;
            sB[i * LDB + c] = gg;
        }
        __syncthreads();
        {   // 8 threads per channel (lanes 8m .. 8m+7 of a warp), 16 rows each
            const int c = tid >> 3, part = tid & 7;
            float* col = sB + c;
            float tot = 0.f;
            for (int i = 16 * part; i < 16 * part + 16; ++i) tot += col[i * LDB];
            float incl = tot;   // inclusive scan of the 8 row groups' totals
#pragma unroll
            for (int d = 1; d < 8; d <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, incl, d, 8);
                if (part >= d) incl += y;
            }
            float run = __shfl_up_sync(0xffffffffu, incl, 1, 8);
            if (part == 0) run = 0.f;
            for (int i = 16 * part; i < 16 * part + 16; ++i) {
                run += col[i * LDB];
                col[i * LDB] = run;
            }
            if (part == 7) sBC[c0 + c] = run;
        }
        __syncthreads();
    };

    for (int t0 = 0; t0 < T; t0 += C) {
        const int Ct = min(C, T - t0);
        __syncthreads();
        // 1. v and beta of the chunk (zero past its end); accumulators cleared
        for (int idx = tid; idx < C * LDC; idx += kThreads) sAP[idx] = 0.f;
        for (int i = tid; i < C; i += kThreads) {
            sPd[i] = 0.f;
            sBeta[i] = (i < Ct) ? to_f32(beta[((int64_t)b * T + t0 + i) * H + h]) : 0.f;
        }
        for (int idx = tid; idx < C * kDvt; idx += kThreads) {
            const int i = idx / kDvt, j = idx % kDvt;
            float vv = 0.f;
            if (i < Ct) vv = to_f32(v[((int64_t)b * T + t0 + i) * strv + (int64_t)h * Dv + col0 + j]);
            sV[i * LDV + j] = vv;
            sO[i * kDvt + j] = 0.f;
        }
        // 2. per channel block: its share of A, P, (e^b k) S0 and (e^b q) S0
        for (int c0 = 0; c0 < DK; c0 += KB) {
            if (c0) __syncthreads();
            load_block(t0, Ct, c0, true);
            for (int idx = tid; idx < C * C; idx += kThreads) {
                const int i = idx / C, j = idx % C;
                if (j > i) continue;
                const float* ki = sK + i * LDB; const float* qi = sQ + i * LDB;
                const float* kj = sK + j * LDB;
                const float* bi = sB + i * LDB; const float* bj = sB + j * LDB;
                float aa = 0.f, pp = 0.f;
#pragma unroll 8
                for (int c = 0; c < KB; ++c) {
                    const float kd = kj[c] * expf(bi[c] - bj[c]);
                    aa = fmaf(ki[c], kd, aa);
                    pp = fmaf(qi[c], kd, pp);
                }
                if (j < i) {
                    sAP[i * LDC + j] += aa;
                    sAP[j * LDC + i] += pp;
                } else {
                    sPd[i] += pp;
                }
            }
            __syncthreads();
            for (int idx = tid; idx < C * KB; idx += kThreads) {
                const int i = idx / KB, c = idx % KB;
                const float e = expf(sB[i * LDB + c]);
                sQ[i * LDB + c] *= e;
                sK[i * LDB + c] *= e;
            }
            __syncthreads();
            for (int idx = tid; idx < C * kDvt; idx += kThreads) {
                const int i = idx / kDvt, j = idx % kDvt;
                float ks = 0.f, qs = 0.f;
#pragma unroll 8
                for (int c = 0; c < KB; ++c) {
                    const float st = sS[(c0 + c) * kDvt + j];
                    ks = fmaf(sK[i * LDB + c], st, ks);
                    qs = fmaf(sQ[i * LDB + c], st, qs);
                }
                sV[i * LDV + j] -= ks;
                sO[i * kDvt + j] += qs;
            }
        }
        __syncthreads();
        // 3. rhs = beta (v - (e^b k) S0)
        for (int idx = tid; idx < C * kDvt; idx += kThreads) {
            const int i = idx / kDvt, j = idx % kDvt;
            sV[i * LDV + j] *= sBeta[i];
        }
        __syncthreads();
        // 4. forward substitution u_i = rhs_i - beta_i sum_{m<i} A_im u_m, one row at a time
        {
            const int part = tid & 7, j = tid >> 3;
            for (int i = 1; i < C; ++i) {
                float s = 0.f;
                for (int m = part; m < i; m += 8) s = fmaf(sAP[i * LDC + m], sV[m * LDV + j], s);
                s += __shfl_xor_sync(0xffffffffu, s, 1);
                s += __shfl_xor_sync(0xffffffffu, s, 2);
                s += __shfl_xor_sync(0xffffffffu, s, 4);
                if (part == 0) sV[i * LDV + j] -= sBeta[i] * s;
                __syncthreads();
            }
        }
        // 5. outputs o_i = (e^b q_i) S0 + P_ii u_i + sum_{m<i} P_im u_m
        for (int idx = tid; idx < C * kDvt; idx += kThreads) {
            const int i = idx / kDvt, j = idx % kDvt;
            if (i >= Ct) continue;
            float acc = fmaf(sPd[i], sV[i * LDV + j], sO[i * kDvt + j]);
            for (int m = 0; m < i; ++m) acc = fmaf(sAP[m * LDC + i], sV[m * LDV + j], acc);
            o[((int64_t)b * T + t0 + i) * strv + (int64_t)h * Dv + col0 + j] = from_f32<TOut>(acc);
        }
        // 6. state to the chunk end, per channel block: Diag(e^{b_C}) S0 + sum_i (e^{b_C - b_i} k_i) u_i^T
        for (int c0 = 0; c0 < DK; c0 += KB) {
            __syncthreads();
            load_block(t0, Ct, c0, false);
            for (int idx = tid; idx < C * KB; idx += kThreads) {
                const int i = idx / KB, c = idx % KB;
                sK[i * LDB + c] *= expf(sBC[c0 + c] - sB[i * LDB + c]);
            }
            __syncthreads();
            for (int idx = tid; idx < KB * kDvt; idx += kThreads) {
                const int c = idx / kDvt, j = idx % kDvt;
                float acc = expf(sBC[c0 + c]) * sS[(c0 + c) * kDvt + j];
                for (int i = 0; i < C; ++i) acc = fmaf(sK[i * LDB + c], sV[i * LDV + j], acc);
                sS[(c0 + c) * kDvt + j] = acc;
            }
        }
    }
    __syncthreads();
    if (ST) {
        for (int idx = tid; idx < DK * kDvt; idx += kThreads) {
            const int c = idx / kDvt, j = idx % kDvt;
            ST[sbase + (int64_t)c * Dv + j] = sS[idx];
        }
    }
}

size_t wide_smem_bytes(int DK)
{
    constexpr int C = kWideC;
    const size_t f = (size_t)C * (C + 1) + C + 3ull * C * (kKB + 1) + (size_t)C * (kDvt + 1) +
                     (size_t)C * kDvt + (size_t)DK * kDvt + C + DK;
    return f * sizeof(float);
}

size_t generic_smem_bytes(int DK, int C)
{
    const size_t f = 3ull * C * (DK + 1) + 2ull * C * (C + 1) + (size_t)C * (kDvt + 1) +
                     (size_t)C * kDvt + (size_t)DK * kDvt + C + DK;
    return f * sizeof(float);
}

template <typename TIn, typename TG, typename TOut, int DK>
cudaError_t launch_typed(const KdaArgs& a, cudaStream_t s)
{
    const int C = a.chunk;
    dim3 grid(a.Dv / kDvt, a.H, a.B);
    if (C == kWideC) {
        const size_t smem = wide_smem_bytes(DK);
        auto kern = kda_generic_wide_kernel<TIn, TG, TOut, DK>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        ProfileScope prof("kda_generic", s);
        count_launch();
        kern<<<grid, kThreads, smem, s>>>((const TIn*)a.q, (const TIn*)a.k, (const TIn*)a.v,
                                          (const TG*)a.g, (const TG*)a.beta, a.S0, (TOut*)a.o,
                                          a.ST, a.T, a.H, a.Dv);
        return cudaGetLastError();
    }
    const size_t smem = generic_smem_bytes(DK, C);
    auto kern = kda_generic_kernel<TIn, TG, TOut, DK>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    ProfileScope prof("kda_generic", s);
    count_launch();
    kern<<<grid, kThreads, smem, s>>>((const TIn*)a.q, (const TIn*)a.k, (const TIn*)a.v,
                                      (const TG*)a.g, (const TG*)a.beta, a.S0, (TOut*)a.o,
                                      a.ST, a.T, a.H, a.Dv, C);
    return cudaGetLastError();
}

template <typename TIn, typename TG, typename TOut>
cudaError_t launch_dk(const KdaArgs& a, cudaStream_t s)
{
    switch (a.Dk) {
        case 32: return launch_typed<TIn, TG, TOut, 32>(a, s);
        case 64: return launch_typed<TIn, TG, TOut, 64>(a, s);
        case 128: return launch_typed<TIn, TG, TOut, 128>(a, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_kda_generic(const KdaArgs& a, cudaStream_t s)
{
    using bf = __nv_bfloat16;
    const bool of = a.out_t == ET_F32;
    if (a.in_t == ET_F32 && a.gb_t == ET_F32)
        return of ? launch_dk<float, float, float>(a, s) : launch_dk<float, float, bf>(a, s);
    if (a.in_t == ET_BF16 && a.gb_t == ET_BF16)
        return of ? launch_dk<bf, bf, float>(a, s) : launch_dk<bf, bf, bf>(a, s);
    if (a.in_t == ET_F16 && a.gb_t == ET_BF16)
        return of ? launch_dk<__half, bf, float>(a, s) : launch_dk<__half, bf, bf>(a, s);
    return cudaErrorInvalidValue;
}

}  // namespace kda
