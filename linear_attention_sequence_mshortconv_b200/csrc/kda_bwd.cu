// Backward of the KDA forward scan (Eq. 14 of the Chimera paper, section 3.3, with the
// readout o_t = S_t^T q_t of Eq. 15): given dL/do and dL/dS_T, the gradients of q, k, v,
// g = log(alpha), beta and S0.  The paper gives only the forward; this is its
// reverse-mode derivative, taken through the chunk form of the scan.
//
// Chunk form (C = 32 tokens, entry state S, b_i = sum_{r<=i} g_r per key channel, b_C
// the chunk's last b, r = b at row 15 a per-channel reference):
//   K+ = k e^{b-r},  K- = k e^{r-b},  Q+ = q e^{b-r},  Se = Diag(e^r) S
//   Kd = K+ K-^T (used strictly below the diagonal),  A = Diag(beta) Kd,  T = (I + A)^{-1}
//   P  = lower(Q+ K-^T)                      (diagonal included)
//   VX = V - K+ Se,  Rb = Diag(beta) VX,  U = T Rb
//   O  = Q+ Se + P U,   S' = Diag(e^{b_C - r}) (Se + K-^T U)
// Reverse, with G' = dL/dS' and Gc = Diag(e^{b_C - r}) G':
//   dU  = P^T dO + K- Gc           dR = T^T dU            dv = Diag(beta) dR
//   dbeta_i = VX_i . dR_i + sum_{j<i} dA_ij Kd_ij        (dRb = Diag(beta) dR)
//   dT  = dU Rb^T,  dA = -T^T dT T^T (strictly lower),   dAb = Diag(beta) dA
//   dP  = lower(dO U^T)
//   dQ+ = dO Se^T + dP K-          dK+ = -dRb Se^T + dAb K-
//   dK- = U Gc^T + dAb^T K+ + dP^T Q+
//   G   = Diag(e^r) (Gc + Q+^T dO - K+^T dRb)             (dL/dS, to the previous chunk)
//   dq  = dQ+ e^{b-r},  dk = dK+ e^{b-r} + dK- e^{r-b}
//   db  = dQ+ Q+ + dK+ K+ - dK- K-,  plus at b_C: sum_j (U Gc^T)_j K-_j + rowsum(Gc Se)
//   dg  = reverse cumulative sum of db over the chunk's rows
// r cancels out of the loss, so it is held fixed.  Every exponent that reaches a used
// value is <= 0 or within e^{|b_C|}: per key channel the decay over each 32-token chunk
// must stay below 80 (|sum g| < 80, mean g > -2.5 per token).  A chunk beyond that is
// reported on the device status word (DEV_RANGE) and its gradients are not finite.
//
// Every matrix product runs on the tensor cores as 3xTF32 warp MMAs (fp32 accuracy).
// Parallel split: the state's value columns evolve independently, so one CTA owns 16
// value columns of one (b, h).  It first runs the forward over all chunks and stores
// each chunk's entry state (its 16 columns), T and Kd in the workspace, then walks the chunks in
// reverse.  dv and dS0 columns belong to one CTA; dq, dk, dg and dbeta are sums over
// the value columns and are accumulated with atomic adds (the outputs are zeroed first).
// Everything else is fp32 on CUDA cores.

#include <type_traits>

#include "internal.h"

namespace kda {
namespace {

constexpr int BC = 32;        // chunk length
constexpr int BVC = 16;       // value columns per CTA
constexpr int BT = 512;       // threads per CTA
// Largest decay -sum(g) of one key channel over one 32-token chunk (natural-log units)
// that the exponent factorisation around the chunk's row 15 keeps finite in fp32.
constexpr float kBwdDecayLimit = 80.f;
// Row strides (floats) are 4 mod 32, so the 8 x 4 lane pattern of a warp MMA fragment
// load touches 32 different banks for row-major operands.
constexpr int LDV = BVC + 4;  // row stride of [BC][BVC] tiles
constexpr int LDC = BC + 4;   // row stride of [BC][BC] tiles
// one chunk's checkpoint record per CTA: its entry state (DK x BVC), then T and Kd (BC x BC)
template <int DK> __host__ __device__ constexpr int ck_floats() { return DK * BVC + 2 * BC * BC; }

template <int DK> struct BwdPlan {
    static constexpr int LDK = DK + 4;    // [BC][DK] tiles
    static constexpr int LDS = BVC + 4;   // [DK][BVC] tiles
    static constexpr int KP = 0, KM = KP + BC * LDK, QP = KM + BC * LDK;
    static constexpr int DQP = QP + BC * LDK, DKP = DQP + BC * LDK, DKM = DKP + BC * LDK;
    static constexpr int SE = DKM + BC * LDK, GP = SE + DK * LDS;
    static constexpr int VX = GP + DK * LDS, RB = VX + BC * LDV, UU = RB + BC * LDV, DU = UU + BC * LDV,
                         DR = DU + BC * LDV, DO = DR + BC * LDV;
    static constexpr int KD = DO + BC * LDV, PP = KD + BC * LDC, TT = PP + BC * LDC, X1 = TT + BC * LDC,
                         X2 = X1 + BC * LDC, DP = X2 + BC * LDC;
    static constexpr int BB = DP + BC * LDC;   // b = cumsum(g) of the chunk, [BC][DK]
    static constexpr int BETA = BB + BC * LDK, RR = BETA + BC, BCC = RR + DK, DBC = BCC + DK, DBETA = DBC + DK;
    static constexpr int TOTAL = DBETA + BC;
    static constexpr int BYTES = TOTAL * (int)sizeof(float);
};

enum { MM_SET = 0, MM_ADD = 1, MM_SUB = 2, MM_NEG = 3 };

// out(i, j) op= sum_{k<K} A(i, k) B(k, j) for i < M, j < N, on the tensor cores, by the
// warps of threads [tid0, tid0 + nthr) (other warps return at once, so two independent
// products can run side by side on two halves of the block).  A(i, k) = A[i*ai + k*ak], B(k, j) = B[k*bk + j*bj],
// out(i, j) = O[i*oi + j], all in shared memory.  Warp MMAs m16n8k8 with tf32 operands:
// each fp32 operand is split as hi + lo (hi = tf32(x), lo = tf32(x - hi)) and the product
// taken as lo*hi + hi*lo + hi*hi ("3xTF32"), which keeps fp32 accuracy.  16 x 8 output
// tiles are dealt to the warps in turn.
__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo)
{
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(hi) : "f"(x));
    const float r = x - __uint_as_float(hi);
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(lo) : "f"(r));
}

__device__ __forceinline__ void mma_tf32(float (&c)[4], const uint32_t (&a)[4], const uint32_t (&b)[2])
{
    asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

template <int M, int N, int K, int OP>
__device__ __forceinline__ void mmt(float* O, int oi, const float* A, int ai, int ak, const float* B, int bk, int bj,
                                    int tid0 = 0, int nthr = BT)
{
    static_assert(M % 16 == 0 && N % 8 == 0 && K % 8 == 0, "warp MMA tiles");
    constexpr int TN = N / 8, NTILE = (M / 16) * TN;
    const int w0 = tid0 >> 5, nw = nthr >> 5;
    const int wi = (int)(threadIdx.x >> 5) - w0;
    if (wi < 0 || wi >= nw) return;   // not one of this product's warps
    const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    for (int tile = wi; tile < NTILE; tile += nw) {
        const int i0 = (tile / TN) * 16, j0 = (tile % TN) * 8;
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        const float* a0 = A + (i0 + g) * ai + q * ak;
        const float* b0 = B + q * bk + (j0 + g) * bj;
#pragma unroll 4
        for (int k0 = 0; k0 < K; k0 += 8) {
            uint32_t ah[4], al[4], bh[2], bl[2];
            split_tf32(a0[k0 * ak], ah[0], al[0]);
            split_tf32(a0[8 * ai + k0 * ak], ah[1], al[1]);
            split_tf32(a0[(k0 + 4) * ak], ah[2], al[2]);
            split_tf32(a0[8 * ai + (k0 + 4) * ak], ah[3], al[3]);
            split_tf32(b0[k0 * bk], bh[0], bl[0]);
            split_tf32(b0[(k0 + 4) * bk], bh[1], bl[1]);
            mma_tf32(c, al, bh);
            mma_tf32(c, ah, bl);
            mma_tf32(c, ah, bh);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float* o = O + (i0 + g + (e >> 1) * 8) * oi + j0 + 2 * q + (e & 1);
            if (OP == MM_SET) *o = c[e];
            else if (OP == MM_ADD) *o += c[e];
            else if (OP == MM_SUB) *o -= c[e];
            else *o = -c[e];
        }
    }
}

template <typename T> __device__ __forceinline__ float ld(const T* p) { return to_f32(*p); }

// 16 bytes of fp32 or bf16 values -> floats
__device__ __forceinline__ void unpack16(const uint4& u, float (&f)[4], const float*)
{
    f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y); f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
}
__device__ __forceinline__ void unpack16(const uint4& u, float (&f)[8], const __nv_bfloat16*)
{
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

// T = (I + Diag(beta) Kd_strictlower)^{-1} by forward substitution on one warp: lane j
// holds column j of T in registers; row i needs only rows < i.
__device__ __forceinline__ void invert_warp(float* Tm, const float* Kd, const float* beta, int lane)
{
    float col[BC];
#pragma unroll
    for (int i = 0; i < BC; ++i) {
        const float bi = beta[i];
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int m = 0; m < i; ++m) {
            const float a = bi * Kd[i * LDC + m];
            if (m & 1) a1 = fmaf(a, col[m], a1);
            else a0 = fmaf(a, col[m], a0);
        }
        col[i] = (i == lane ? 1.f : 0.f) - (a0 + a1);
    }
#pragma unroll
    for (int i = 0; i < BC; ++i) Tm[i * LDC + lane] = col[i];
}

template <int DK, typename TIn, typename TDo>
__global__ void __launch_bounds__(BT, 1)
kda_bwd_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k, const TIn* __restrict__ v,
               const TIn* __restrict__ g, const TIn* __restrict__ beta, const float* __restrict__ S0,
               const TDo* __restrict__ dout, const float* __restrict__ dST, float* __restrict__ dq,
               float* __restrict__ dk, float* __restrict__ dv, float* __restrict__ dg, float* __restrict__ dbeta,
               float* __restrict__ dS0, float* __restrict__ ckpt, int T, int H, int Dv, int* __restrict__ status)
{
    using PL = BwdPlan<DK>;
    constexpr int LDK = PL::LDK, LDS = PL::LDS;
    extern __shared__ __align__(16) float sm[];
    float *sKP = sm + PL::KP, *sKM = sm + PL::KM, *sQP = sm + PL::QP;
    float *sDQP = sm + PL::DQP, *sDKP = sm + PL::DKP, *sDKM = sm + PL::DKM;
    float *sSe = sm + PL::SE, *sGp = sm + PL::GP;
    float *sVX = sm + PL::VX, *sRb = sm + PL::RB, *sU = sm + PL::UU, *sDU = sm + PL::DU, *sDR = sm + PL::DR,
          *sDO = sm + PL::DO;
    float *sKd = sm + PL::KD, *sP = sm + PL::PP, *sT = sm + PL::TT, *sX1 = sm + PL::X1, *sX2 = sm + PL::X2,
          *sDP = sm + PL::DP;
    float* sB = sm + PL::BB;
    float *sBeta = sm + PL::BETA, *sR = sm + PL::RR, *sBC = sm + PL::BCC, *sDbC = sm + PL::DBC,
          *sDbeta = sm + PL::DBETA;

    const int t = threadIdx.x, w = t >> 5, lane = t & 31;
    const int cb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int col0 = cb * BVC;
    const int NC = (T + BC - 1) / BC;
    const size_t rowH = (size_t)H;                 // tokens -> rows of [B, T, H, *]
    const size_t tok0 = (size_t)b * T;             // first token row of this sequence
    constexpr int CK = ck_floats<DK>();
    float* ck = ckpt + ((size_t)(b * H + h) * (Dv / BVC) + cb) * (size_t)NC * CK;

    // rows [t0, t0 + BC) of a [B, T, H, W] tensor, columns [c0, c0 + NCOL), into an fp32
    // tile with row stride ld (16-byte vector loads, zero past T)
    auto stage = [&](float* dst, int ld, auto src, int W, int c0, auto ncol_tag, int n) {
        using TS = typename std::remove_cv<typename std::remove_pointer<decltype(src)>::type>::type;
        constexpr int NCOL = decltype(ncol_tag)::value;
        constexpr int VE = 16 / (int)sizeof(TS), VPR = NCOL / VE;
        const int t0 = n * BC;
        for (int e = t; e < BC * VPR; e += BT) {
            const int i = e / VPR, cv = (e % VPR) * VE;
            float f[VE];
            if (t0 + i < T) {
                const uint4 u = *reinterpret_cast<const uint4*>(src + ((tok0 + t0 + i) * rowH + h) * W + c0 + cv);
                unpack16(u, f, src);
            } else {
#pragma unroll
                for (int j = 0; j < VE; ++j) f[j] = 0.f;
            }
            // 16-byte stores (rows are 16-byte aligned): a warp's stores spread over all banks
#pragma unroll
            for (int j = 0; j < VE; j += 4)
                *reinterpret_cast<float4*>(dst + i * ld + cv + j) = make_float4(f[j], f[j + 1], f[j + 2], f[j + 3]);
        }
    };
    using KCols = std::integral_constant<int, DK>;
    using VCols = std::integral_constant<int, BVC>;
    // chunk n's k (-> K+ / K-), q (-> Q+), g (-> b), beta, v (and do) staged; then per
    // channel: b = cumsum(g), r, b_C and the decay-scaled operands, in place
    auto prologue = [&](int n, bool bwd) {
        const int t0 = n * BC;
        if (t < BC) sBeta[t] = (t0 + t < T) ? ld(beta + (tok0 + t0 + t) * rowH + h) : 0.f;
        stage(sKP, LDK, k, DK, 0, KCols{}, n);
        stage(sB, LDK, g, DK, 0, KCols{}, n);
        stage(sVX, LDV, v, Dv, col0, VCols{}, n);
        if (bwd) {
            stage(sQP, LDK, q, DK, 0, KCols{}, n);
            stage(sDO, LDV, dout, Dv, col0, VCols{}, n);
        }
        __syncthreads();
        if (t < DK) {
            const int c = t;
            float run = 0.f;
#pragma unroll 8
            for (int i = 0; i < BC; ++i) {
                run += sB[i * LDK + c];
                sB[i * LDK + c] = run;
            }
            const float r = sB[15 * LDK + c];
            sR[c] = r;
            sBC[c] = run;
            // the factorisation around row 15 needs e^{b_0 - r} and e^{r - b_C} finite: the
            // chunk's decay -b_C (b is non-increasing) below kBwdDecayLimit, else the
            // gradients are reported as out of domain
            if (!bwd && !(run > -kBwdDecayLimit)) atomicCAS(status, DEV_OK, DEV_RANGE);
#pragma unroll 4
            for (int i = 0; i < BC; ++i) {
                const float bi = sB[i * LDK + c];
                const float ep = expf(bi - r), em = expf(r - bi);
                const float kk = sKP[i * LDK + c];
                sKP[i * LDK + c] = kk * ep;
                sKM[i * LDK + c] = kk * em;
                if (bwd) sQP[i * LDK + c] *= ep;
            }
        }
    };

    // ---------------- forward sweep: entry state of every chunk -> workspace ----------------
    for (int e = t; e < DK * BVC; e += BT) {
        const int c = e / BVC, j = e % BVC;
        sSe[c * LDS + j] = S0 ? S0[((size_t)(b * H + h) * DK + c) * Dv + col0 + j] : 0.f;
    }
    __syncthreads();
    for (int n = 0; n < NC; ++n) {
        float* ckn = ck + (size_t)n * CK;
        for (int e = t; e < DK * BVC / 4; e += BT) {
            const float* d = sSe + (4 * e / BVC) * LDS + (4 * e) % BVC;
            reinterpret_cast<float4*>(ckn)[e] = make_float4(d[0], d[1], d[2], d[3]);
        }
        prologue(n, false);
        __syncthreads();
        mmt<BC, BC, DK, MM_SET>(sKd, LDC, sKP, LDK, 1, sKM, 1, LDK);
        for (int e = t; e < DK * BVC; e += BT) {
            const int c = e / BVC, j = e % BVC;
            sSe[c * LDS + j] *= expf(sR[c]);
        }
        __syncthreads();
        if (w == 0) invert_warp(sT, sKd, sBeta, lane);
        else mmt<BC, BVC, DK, MM_SUB>(sVX, LDV, sKP, LDK, 1, sSe, LDS, 1, 32, BT - 32);
        __syncthreads();
        for (int e = t; e < BC * BVC; e += BT) {
            const int i = e / BVC, j = e % BVC;
            sRb[i * LDV + j] = sBeta[i] * sVX[i * LDV + j];
        }
        for (int e = t; e < 2 * BC * BC / 4; e += BT) {   // T and Kd for the reverse sweep
            const int m = e / (BC * BC / 4), r = (e % (BC * BC / 4)) * 4 / BC, c4 = (4 * e) % BC;
            const float* src = (m ? sKd : sT) + r * LDC + c4;
            reinterpret_cast<float4*>(ckn + DK * BVC)[e] = make_float4(src[0], src[1], src[2], src[3]);
        }
        __syncthreads();
        mmt<BC, BVC, BC, MM_SET>(sU, LDV, sT, LDC, 1, sRb, LDV, 1);
        __syncthreads();
        mmt<DK, BVC, BC, MM_ADD>(sSe, LDS, sKM, 1, LDK, sU, LDV, 1);
        __syncthreads();
        for (int e = t; e < DK * BVC; e += BT) {
            const int c = e / BVC, j = e % BVC;
            sSe[c * LDS + j] *= expf(sBC[c] - sR[c]);
        }
        __syncthreads();
    }

    // ---------------- reverse sweep ----------------
    for (int e = t; e < DK * BVC; e += BT) {
        const int c = e / BVC, j = e % BVC;
        sGp[c * LDS + j] = dST ? dST[((size_t)(b * H + h) * DK + c) * Dv + col0 + j] : 0.f;
    }
    for (int n = NC - 1; n >= 0; --n) {
        const int t0 = n * BC;
        const float* ckn = ck + (size_t)n * CK;
        __syncthreads();   // the previous chunk is done with every tile
        for (int e = t; e < DK * BVC / 4; e += BT) {
            const float4 c4 = reinterpret_cast<const float4*>(ckn)[e];
            float* d = sSe + (4 * e / BVC) * LDS + (4 * e) % BVC;
            d[0] = c4.x; d[1] = c4.y; d[2] = c4.z; d[3] = c4.w;
        }
        for (int e = t; e < 2 * BC * BC / 4; e += BT) {   // T and Kd from the forward sweep
            const int m = e / (BC * BC / 4), r = (e % (BC * BC / 4)) * 4 / BC, c4 = (4 * e) % BC;
            const float4 v4 = reinterpret_cast<const float4*>(ckn + DK * BVC)[e];
            float* d = (m ? sKd : sT) + r * LDC + c4;
            d[0] = v4.x; d[1] = v4.y; d[2] = v4.z; d[3] = v4.w;
        }
        prologue(n, true);
        __syncthreads();
        // P (T and Kd come from the forward sweep); Se = Diag(e^r) S; Gc = Diag(e^{b_C - r}) G'
        mmt<BC, BC, DK, MM_SET>(sP, LDC, sQP, LDK, 1, sKM, 1, LDK, 0, BT / 2);
        for (int e = t; e < DK * BVC; e += BT) {
            const int c = e / BVC, j = e % BVC;
            sSe[c * LDS + j] *= expf(sR[c]);
            sGp[c * LDS + j] *= expf(sBC[c] - sR[c]);
        }
        __syncthreads();
        // VX = V - K+ Se | dU = K- Gc; P masked
        mmt<BC, BVC, DK, MM_SUB>(sVX, LDV, sKP, LDK, 1, sSe, LDS, 1, 0, BT / 2);
        mmt<BC, BVC, DK, MM_SET>(sDU, LDV, sKM, LDK, 1, sGp, LDS, 1, BT / 2, BT / 2);
        for (int e = t; e < BC * BC; e += BT) {
            const int i = e / BC, j = e % BC;
            if (j > i) sP[i * LDC + j] = 0.f;
        }
        __syncthreads();
        for (int e = t; e < BC * BVC; e += BT) {
            const int i = e / BVC, j = e % BVC;
            sRb[i * LDV + j] = sBeta[i] * sVX[i * LDV + j];
        }
        mmt<BC, BVC, BC, MM_ADD>(sDU, LDV, sP, 1, LDC, sDO, LDV, 1);   // dU += P^T dO
        __syncthreads();
        mmt<BC, BVC, BC, MM_SET>(sU, LDV, sT, LDC, 1, sRb, LDV, 1, 0, BT / 2);         // U = T Rb
        mmt<BC, BVC, BC, MM_SET>(sDR, LDV, sT, 1, LDC, sDU, LDV, 1, BT / 2, BT / 2);   // dR = T^T dU
        __syncthreads();
        if (t < BC) {
            float s = 0.f;
            for (int j = 0; j < BVC; ++j) s = fmaf(sVX[t * LDV + j], sDR[t * LDV + j], s);
            sDbeta[t] = s;
        }
        for (int e = t; e < BC * BVC; e += BT) {
            const int i = e / BVC, j = e % BVC;
            if (t0 + i < T) dv[((tok0 + t0 + i) * rowH + h) * Dv + col0 + j] = sBeta[i] * sDR[i * LDV + j];
        }
        mmt<BC, BC, BVC, MM_SET>(sX1, LDC, sDU, LDV, 1, sRb, 1, LDV, 0, BT / 2);       // dT = dU Rb^T
        mmt<BC, BC, BVC, MM_SET>(sDP, LDC, sDO, LDV, 1, sU, 1, LDV, BT / 2, BT / 2);   // dO U^T
        __syncthreads();
        for (int e = t; e < BC * BVC; e += BT) {                        // dRb = Diag(beta) dR
            const int i = e / BVC, j = e % BVC;
            sDR[i * LDV + j] *= sBeta[i];
        }
        for (int e = t; e < BC * BC; e += BT) {                         // dP = lower(dO U^T)
            const int i = e / BC, j = e % BC;
            if (j > i) sDP[i * LDC + j] = 0.f;
        }
        mmt<BC, BC, BC, MM_SET>(sX2, LDC, sX1, LDC, 1, sT, 1, LDC);    // dT T^T
        __syncthreads();
        mmt<BC, BC, BC, MM_NEG>(sX1, LDC, sT, 1, LDC, sX2, LDC, 1);    // dA = -T^T dT T^T
        __syncthreads();
        if (t < BC) {   // strictly lower part; dbeta from A; dAb = Diag(beta) dA
            const int i = t;
            float s = sDbeta[i];
            for (int j = 0; j < BC; ++j) {
                const float da = (j < i) ? sX1[i * LDC + j] : 0.f;
                s = fmaf(da, sKd[i * LDC + j], s);
                sX1[i * LDC + j] = sBeta[i] * da;
            }
            sDbeta[i] = s;
        }
        mmt<BC, DK, BVC, MM_SET>(sDQP, LDK, sDO, LDV, 1, sSe, 1, LDS);  // dQ+ = dO Se^T
        mmt<BC, DK, BVC, MM_NEG>(sDKP, LDK, sDR, LDV, 1, sSe, 1, LDS);  // dK+ = -dRb Se^T
        mmt<BC, DK, BVC, MM_SET>(sDKM, LDK, sU, LDV, 1, sGp, 1, LDS);   // dK- = U Gc^T
        __syncthreads();
        if (t < DK) {   // the b_C terms: sum_j (U Gc^T)_j K-_j + rowsum(Gc Se)
            const int c = t;
            float s = 0.f;
            for (int i = 0; i < BC; ++i) s = fmaf(sDKM[i * LDK + c], sKM[i * LDK + c], s);
            for (int j = 0; j < BVC; ++j) s = fmaf(sGp[c * LDS + j], sSe[c * LDS + j], s);
            sDbC[c] = s;
        }
        mmt<BC, DK, BC, MM_ADD>(sDQP, LDK, sDP, LDC, 1, sKM, LDK, 1);   // dQ+ += dP K-
        mmt<BC, DK, BC, MM_ADD>(sDKP, LDK, sX1, LDC, 1, sKM, LDK, 1);   // dK+ += dAb K-
        __syncthreads();
        mmt<BC, DK, BC, MM_ADD>(sDKM, LDK, sX1, 1, LDC, sKP, LDK, 1);   // dK- += dAb^T K+
        mmt<BC, DK, BC, MM_ADD>(sDKM, LDK, sDP, 1, LDC, sQP, LDK, 1);   // dK- += dP^T Q+
        mmt<DK, BVC, BC, MM_ADD>(sGp, LDS, sQP, 1, LDK, sDO, LDV, 1);   // Gc + Q+^T dO
        mmt<DK, BVC, BC, MM_SUB>(sGp, LDS, sKP, 1, LDK, sDR, LDV, 1);   //    - K+^T dRb
        __syncthreads();
        if (t < DK) {   // per channel: dq, dk, db -> dg (reverse cumulative sum), in place; G row scale
            const int c = t;
            const float r = sR[c];
            float acc = sDbC[c];
#pragma unroll 4
            for (int i = BC - 1; i >= 0; --i) {
                const float bi = sB[i * LDK + c];
                const float ep = expf(bi - r), em = expf(r - bi);
                const float dqp = sDQP[i * LDK + c], dkp = sDKP[i * LDK + c], dkm = sDKM[i * LDK + c];
                acc += dqp * sQP[i * LDK + c] + dkp * sKP[i * LDK + c] - dkm * sKM[i * LDK + c];
                sDQP[i * LDK + c] = dqp * ep;
                sDKP[i * LDK + c] = dkp * ep + dkm * em;
                sDKM[i * LDK + c] = acc;
            }
            const float er = expf(r);
            for (int j = 0; j < BVC; ++j) sGp[c * LDS + j] *= er;
        }
        __syncthreads();
        for (int e = t; e < BC * DK / 4; e += BT) {   // dq, dk, dg += this CTA's part, 16 bytes at a time
            const int i = e / (DK / 4), c = (e % (DK / 4)) * 4;
            if (t0 + i >= T) continue;
            const size_t idx = ((tok0 + t0 + i) * rowH + h) * DK + c;
            atomicAdd(reinterpret_cast<float4*>(dq + idx), *reinterpret_cast<const float4*>(sDQP + i * LDK + c));
            atomicAdd(reinterpret_cast<float4*>(dk + idx), *reinterpret_cast<const float4*>(sDKP + i * LDK + c));
            atomicAdd(reinterpret_cast<float4*>(dg + idx), *reinterpret_cast<const float4*>(sDKM + i * LDK + c));
        }
        if (t < BC && t0 + t < T) atomicAdd(dbeta + (tok0 + t0 + t) * rowH + h, sDbeta[t]);
    }
    __syncthreads();
    if (dS0)
        for (int e = t; e < DK * BVC; e += BT) {
            const int c = e / BVC, j = e % BVC;
            dS0[((size_t)(b * H + h) * DK + c) * Dv + col0 + j] = sGp[c * LDS + j];
        }
}

template <int DK, typename TIn, typename TDo>
cudaError_t launch_t(const KdaBwdArgs& a, void* ws, cudaStream_t s)
{
    auto kern = kda_bwd_kernel<DK, TIn, TDo>;
    const int smem = BwdPlan<DK>::BYTES;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    ProfileScope prof("kda_bwd", s);
    count_launch();
    kern<<<dim3(a.Dv / BVC, a.H, a.B), BT, smem, s>>>(
        (const TIn*)a.q, (const TIn*)a.k, (const TIn*)a.v, (const TIn*)a.g, (const TIn*)a.beta, a.S0,
        (const TDo*)a.dout, a.dST, a.dq, a.dk, a.dv, a.dg, a.dbeta, a.dS0, reinterpret_cast<float*>(ws), a.T, a.H,
        a.Dv, a.status);
    return cudaGetLastError();
}

template <int DK>
cudaError_t launch_d(const KdaBwdArgs& a, void* ws, cudaStream_t s)
{
    const bool in_f32 = a.in_t == ET_F32, do_f32 = a.do_t == ET_F32;
    if (in_f32 && do_f32) return launch_t<DK, float, float>(a, ws, s);
    if (in_f32) return launch_t<DK, float, __nv_bfloat16>(a, ws, s);
    if (do_f32) return launch_t<DK, __nv_bfloat16, float>(a, ws, s);
    return launch_t<DK, __nv_bfloat16, __nv_bfloat16>(a, ws, s);
}

}  // namespace

size_t kda_bwd_workspace_bytes(int B, int T, int H, int Dk, int Dv)
{
    if (B <= 0 || T <= 0) return 0;
    const size_t NC = (size_t)(T + BC - 1) / BC;
    // per CTA (B*H*Dv/BVC of them) and chunk: its state columns, T and Kd
    return (size_t)B * H * NC * ((size_t)Dk * Dv + (size_t)(Dv / BVC) * 2 * BC * BC) * sizeof(float);
}

cudaError_t launch_kda_bwd(const KdaBwdArgs& a, void* ws, cudaStream_t s)
{
    const size_t tok = (size_t)a.B * a.T * a.H;
    cudaError_t e = cudaMemsetAsync(a.dq, 0, tok * a.Dk * sizeof(float), s);
    if (e == cudaSuccess) e = cudaMemsetAsync(a.dk, 0, tok * a.Dk * sizeof(float), s);
    if (e == cudaSuccess) e = cudaMemsetAsync(a.dg, 0, tok * a.Dk * sizeof(float), s);
    if (e == cudaSuccess) e = cudaMemsetAsync(a.dbeta, 0, tok * sizeof(float), s);
    if (e != cudaSuccess) return e;
    switch (a.Dk) {
        case 32: return launch_d<32>(a, ws, s);
        case 64: return launch_d<64>(a, ws, s);
        case 128: return launch_d<128>(a, ws, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace kda
