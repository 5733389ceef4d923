// Tensor-core (tcgen05 / TMEM / TMA) chunkwise KDA forward for Dk = Dv = 128, chunk 64.
//
// What it computes is Eq. 14 of the Chimera paper (section 3.3) with the readout
// o_t = S_t^T q_t (Eq. 15, inner term).  The pages only say the kernel is "chunked";
// the chunk algebra is derived from Eq. 14.  Inside a chunk of C = 64 tokens with
// entry state S0, b_i = sum_{r<=i} g_r (fp32, per key channel), a reference point
// r = b_31 (the middle of the chunk) keeps every exponential within e^{+-|b|/2}:
//   K+ = k e^{b - r},  Q+ = q e^{b - r},  K- = k e^{r - b},  Kt = k e^{b_C - b}
//   A  = diag(beta) strict_lower(K+ K-^T),   P = lower(Q+ K-^T)      (incl. diagonal)
//   T' = (I + A)^{-1} diag(beta)                                  (blocked, fp32)
//   S^ = diag(e^{r}) S0                                           (state seen by K+, Q+)
//   U  = T' V - (T' K+) S^              O = Q+ S^ + P U
//   S_C = diag(e^{b_C}) S0 + Kt^T U
// Every MMA operand is fp16 in shared memory (11-bit significand: bf16 operands
// would cost ~3% of RMS(o) in max error), accumulation is fp32 in TMEM, and the
// state's master copy stays fp32 in TMEM across chunks.
//
// Parallelism.  A head's scan is sequential over chunks, and one B200 workload has
// only B*H = 16 heads for 148 SMs, so each head's chunk sequence is cut into P
// segments of L chunks.  Eq. 14 is affine in the state, so a segment maps its entry
// state S to M S + N.
//   pass 1 (MODE_STATE, segments 0..P-2): run the recurrence on the augmented state
//          [S | Phi] starting from [0 | I] with the values of the segment: the result
//          is [N | M] (the identity columns carry no values).
//   combine: S_start(p+1) = M_p S_start(p) + N_p in fp32 (CUDA cores).
//   pass 2 (MODE_OUTPUT, all segments): run the recurrence from S_start(p) and write
//          o (and S_T from the last segment).
// Each pass is one CTA per (b, h, segment), 256 threads, ~200 KB of shared memory.
//
// Shared-memory operand tiles use the no-swizzle core-matrix layout: 8 rows x 16 B
// blocks of 128 contiguous bytes.  A thread that owns one key channel writes 8
// consecutive chunk positions as one 16-byte store, so the channel-major tiles serve
// both as MN-major operands (chunk position = M/N) and K-major ones (position = K).
//
// All waits are bounded (kWaitNs); on expiry the kernel records DEV_TIMEOUT in the
// device status word, drains its own copies and MMAs, frees TMEM and returns.

#include <mutex>
#include <type_traits>

#include "internal.h"
#include "sm100.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int C = 64;         // chunk length
constexpr int D = 128;        // Dk = Dv
constexpr int NT = 256;       // threads per CTA
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s bound on every wait
enum { MODE_STATE = 0, MODE_OUTPUT = 1 };

// ---- shared-memory plan (bytes) --------------------------------------------------
template <int MODE> struct Plan;
template <> struct Plan<MODE_OUTPUT> {
    static constexpr int NS = 128;                 // state columns (values only)
    static constexpr int STG = 0;                  // q,k,v,g staging: 4 x [64][128] bf16
    static constexpr int stQ = 0, stK = 16384, stV = 32768, stG = 49152;
    static constexpr int X = 65536;                // K+ | V interleaved (i-group stride 4096); later W
    static constexpr int QP = 98304;               // Q+ (channel-major, i-group stride 2048)
    static constexpr int KM = 114688;              // K-, then fp32 T (16 KB), then T' (8 KB) | P (8 KB)
    static constexpr int KT = 131072;              // Kt
    static constexpr int U = 147456;               // fp32 A during the inverse, then U (64 x 128 fp16)
    static constexpr int S = 163840;               // S^ (128 x 128 fp16)
    static constexpr int MISC = 196608;
    static constexpr int TMA_BYTES = 4 * 16384;
};
template <> struct Plan<MODE_STATE> {
    static constexpr int NS = 256;                 // [S | Phi]
    static constexpr int STG = 0;
    static constexpr int stQ = -1, stK = 0, stV = 16384, stG = 32768;
    static constexpr int X = 49152;
    static constexpr int QP = -1;
    static constexpr int KM = 81920;
    static constexpr int KT = 98304;
    static constexpr int U = 114688;               // 64 x 256 fp16
    static constexpr int S = 147456;               // 128 x 256 fp16
    static constexpr int MISC = 212992;
    static constexpr int TMA_BYTES = 3 * 16384;
};
// MISC sub-layout
constexpr int M_BETA = 0;        // float[64]
constexpr int M_REF = 256;       // float[128]  b at row 31 (reference)
constexpr int M_BC = 768;        // float[128]  b at row 63
constexpr int M_XS = 1280;       // float[3][256] block products of the inverse
constexpr int M_BAR = 4352;      // 2 x uint64 mbarriers
constexpr int M_TMEM = 4368;     // uint32 TMEM base
constexpr int M_ABORT = 4372;    // int
constexpr int MISC_BYTES = 4384;

template <int MODE> constexpr int smem_bytes() { return Plan<MODE>::MISC + MISC_BYTES; }

// TMEM columns
constexpr uint32_t TM_S = 0;       // state master (fp32), 128 or 256 columns
// MODE_OUTPUT
constexpr uint32_t TO_U = 128, TO_A = 256, TO_P = 320, TO_W = 256, TO_O = 384;
// MODE_STATE
constexpr uint32_t TS_A = 256, TS_R = 256, TS_W = 384;

// ---- helpers ------------------------------------------------------------------------
__device__ __forceinline__ float ld_in(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ float ld_in(const __half* p) { return __half2float(*p); }

__device__ __forceinline__ uint4 pack8_f16(const float* f)
{
    uint4 u;
    __half2* h = reinterpret_cast<__half2*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
    return u;
}

// fp32 64x64 with an XOR swizzle on 4-column groups (conflict-free row and column use)
__device__ __forceinline__ int sw(int i, int j) { return i * 64 + (j ^ ((i & 7) << 2)); }

struct Ctl {
    uint64_t* tma_bar;
    uint64_t* mma_bar;
    int* abort_flag;
    int* status;
    uint32_t tma_phase, mma_phase;
};

// Bounded wait on the MMA barrier; every thread calls it, and the CTA agrees on the
// outcome at the following __syncthreads.
__device__ __forceinline__ void wait_mma(Ctl& c)
{
    if (!mbar_wait_bounded(c.mma_bar, c.mma_phase, kWaitNs)) {
        *c.abort_flag = 1;
        atomicCAS(c.status, DEV_OK, DEV_TIMEOUT);
    }
    c.mma_phase ^= 1;
    tc_fence_after();
}
__device__ __forceinline__ void wait_tma(Ctl& c)
{
    if (!mbar_wait_bounded(c.tma_bar, c.tma_phase, kWaitNs)) {
        *c.abort_flag = 1;
        atomicCAS(c.status, DEV_OK, DEV_TIMEOUT);
    }
    c.tma_phase ^= 1;
}

// The kernel ---------------------------------------------------------------------------
template <int MODE, typename TQ>
__global__ void __launch_bounds__(NT, 1)
kda_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
              const __nv_bfloat16* __restrict__ beta, void* __restrict__ o, int o_f32,
              const float* __restrict__ S_in, int s_in_per_segment, float* __restrict__ maps,
              float* __restrict__ S_T, int B, int T, int H, int P, int L, int* status)
{
    using PL = Plan<MODE>;
    constexpr int NS = PL::NS;
    extern __shared__ __align__(1024) uint8_t sm[];

    const int t = threadIdx.x, w = t >> 5, lane = t & 31;
    const int q4 = w & 3, hf = w >> 2;        // TMEM lane quarter, column half
    const int c = t & 127, rb = t >> 7;       // channel / TMEM row, row block of the prologue
    const int nseg = (MODE == MODE_STATE) ? P - 1 : P;
    const int bh = blockIdx.x / nseg, p = blockIdx.x % nseg;
    const int b = bh / H, h = bh % H;
    const int NC = (T + C - 1) / C;
    const int n0 = p * L, n1 = min(NC, n0 + L);

    float* sBeta = reinterpret_cast<float*>(sm + PL::MISC + M_BETA);
    float* sRef = reinterpret_cast<float*>(sm + PL::MISC + M_REF);
    float* sBC = reinterpret_cast<float*>(sm + PL::MISC + M_BC);
    float* sXs = reinterpret_cast<float*>(sm + PL::MISC + M_XS);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + PL::MISC + M_BAR);
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(sm + PL::MISC + M_TMEM);
    int* sAbort = reinterpret_cast<int*>(sm + PL::MISC + M_ABORT);
    float* Afp = reinterpret_cast<float*>(sm + PL::U);    // during the inverse
    float* Tfp = reinterpret_cast<float*>(sm + PL::KM);   // during the inverse
    const uint32_t sbase = smem_addr(sm);

    Ctl ctl{&bars[0], &bars[1], sAbort, status, 0u, 0u};
    if (t == 0) {
        mbar_init(ctl.tma_bar, 1);
        mbar_init(ctl.mma_bar, 1);
        *sAbort = 0;
        fence_mbar_init();
    }
    if (w == 0) {
        tmem_alloc(sTmem, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *sTmem;
    const uint32_t tl = tmem + ((uint32_t)(32 * q4) << 16);   // this warp's lane quarter
    bool tma_in_flight = false;
    bool mma_in_flight = false;

    auto issue_tma = [&](int n) {
        const int row = b * T + n * C;
        mbar_arrive_expect_tx(ctl.tma_bar, PL::TMA_BYTES);
        if (MODE == MODE_OUTPUT) tma_load_3d(sm + PL::stQ, &tm_q, ctl.tma_bar, 0, h, row);
        tma_load_3d(sm + PL::stK, &tm_k, ctl.tma_bar, 0, h, row);
        tma_load_3d(sm + PL::stV, &tm_v, ctl.tma_bar, 0, h, row);
        tma_load_3d(sm + PL::stG, &tm_g, ctl.tma_bar, 0, h, row);
    };
    if (t == 0 && n0 < n1) issue_tma(n0);
    tma_in_flight = n0 < n1;

    // ---- initial state in TMEM ------------------------------------------------------
    {
        const int col0 = hf * (NS / 2);
        for (int cc = 0; cc < NS / 2; cc += 32) {
            float v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int col = col0 + cc + j;
                float x = 0.f;
                if (MODE == MODE_STATE) {
                    x = (col >= D && col - D == c) ? 1.f : 0.f;
                } else if (S_in) {
                    const size_t idx = s_in_per_segment ? (size_t)bh * P + p : (size_t)bh;
                    x = S_in[(idx * D + c) * D + col];
                }
                v[j] = x;
            }
            tmem_st32(tl + TM_S + col0 + cc, v);
        }
    }
    tc_fence_before();
    __syncthreads();

    for (int n = n0; n < n1 && !*sAbort; ++n) {
        const int t0 = n * C;
        // ---- 1. prologue: staging -> fp16 operand tiles --------------------------------
        wait_tma(ctl);
        __syncthreads();
        if (*sAbort) break;
        tma_in_flight = false;
        if (t < C) sBeta[t] = (t0 + t < T) ? __bfloat162float(beta[((size_t)b * T + t0 + t) * H + h]) : 0.f;
        float bl[32];
        {
            const __nv_bfloat16* stg = reinterpret_cast<const __nv_bfloat16*>(sm + PL::stG);
            float run = 0.f;
#pragma unroll
            for (int r = 0; r < 32; ++r) {
                const int i = 32 * rb + r;
                run += (t0 + i < T) ? __bfloat162float(stg[i * D + c]) : 0.f;
                bl[r] = run;
            }
            if (rb == 0) sRef[c] = run;
        }
        __syncthreads();
        const float rc = sRef[c];
        if (rb == 1) {
#pragma unroll
            for (int r = 0; r < 32; ++r) bl[r] += rc;
            sBC[c] = bl[31];
        }
        __syncthreads();
        const float bC = sBC[c];
        {
            const float eCr = __expf(bC - rc);
            const TQ* sk = reinterpret_cast<const TQ*>(sm + PL::stK);
            const TQ* sv = reinterpret_cast<const TQ*>(sm + PL::stV);
            const TQ* sq = reinterpret_cast<const TQ*>(sm + (MODE == MODE_OUTPUT ? PL::stQ : PL::stK));
            const int cofs = (c >> 3) * 128 + (c & 7) * 16;
#pragma unroll
            for (int grp = 0; grp < 4; ++grp) {
                float kp[8], km[8], kt[8], vh[8], qp[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int r = grp * 8 + j, i = 32 * rb + r;
                    const bool valid = t0 + i < T;
                    const float kk = valid ? ld_in(sk + i * D + c) : 0.f;
                    const float vv = valid ? ld_in(sv + i * D + c) : 0.f;
                    const float x = bl[r] - rc;
                    const float ep = __expf(x), em = __expf(-x);
                    kp[j] = kk * ep;
                    km[j] = kk * em;
                    kt[j] = km[j] * eCr;
                    vh[j] = vv;
                    if (MODE == MODE_OUTPUT) qp[j] = (valid ? ld_in(sq + i * D + c) : 0.f) * ep;
                }
                const int ig = 4 * rb + grp;   // 8-row group of chunk positions
                *reinterpret_cast<uint4*>(sm + PL::X + ig * 4096 + cofs) = pack8_f16(kp);
                *reinterpret_cast<uint4*>(sm + PL::X + ig * 4096 + 2048 + cofs) = pack8_f16(vh);
                *reinterpret_cast<uint4*>(sm + PL::KM + ig * 2048 + cofs) = pack8_f16(km);
                *reinterpret_cast<uint4*>(sm + PL::KT + ig * 2048 + cofs) = pack8_f16(kt);
                if (MODE == MODE_OUTPUT)
                    *reinterpret_cast<uint4*>(sm + PL::QP + ig * 2048 + cofs) = pack8_f16(qp);
            }
        }
        // ---- 2. state: S^ = diag(e^r) S (fp16 tile), master *= e^{b_C} ----------------
        {
            const float er = __expf(rc), eC = __expf(bC);
            const int col0 = hf * (NS / 2);
            for (int cc = 0; cc < NS / 2; cc += 32) {
                float v[32];
                tmem_ld32(tl + TM_S + col0 + cc, v);
#pragma unroll
                for (int g8 = 0; g8 < 4; ++g8) {
                    float f[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) f[j] = v[g8 * 8 + j] * er;
                    const int col = col0 + cc + g8 * 8;
                    *reinterpret_cast<uint4*>(sm + PL::S + (col >> 3) * 2048 + (c >> 3) * 128 + (c & 7) * 16) =
                        pack8_f16(f);
                }
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] *= eC;
                tmem_st32(tl + TM_S + col0 + cc, v);
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        // next chunk's inputs can stream in while this one computes
        if (t == 0 && n + 1 < n1) issue_tma(n + 1);
        tma_in_flight = n + 1 < n1;

        // ---- 3. A = K+ K-^T (and P = Q+ K-^T) ------------------------------------------
        if (t == 0) {
            tc_fence_after();
            const uint32_t id = idesc_f16(64, 64, true, true);
            const uint32_t tA = (MODE == MODE_OUTPUT) ? TO_A : TS_A;
            for (int kk = 0; kk < 8; ++kk) {
                const uint64_t bd = sdesc(sbase + PL::KM + 256 * kk, 128, 2048);
                umma_f16(tmem + tA, sdesc(sbase + PL::X + 256 * kk, 128, 4096), bd, id, kk > 0);
                if (MODE == MODE_OUTPUT)
                    umma_f16(tmem + TO_P, sdesc(sbase + PL::QP + 256 * kk, 128, 2048), bd, id, kk > 0);
            }
            umma_commit(ctl.mma_bar);
        }
        mma_in_flight = true;
        wait_mma(ctl);
        mma_in_flight = false;
        // A rows -> fp32 (beta-scaled, strictly lower)
        {
            float v[32];
            const uint32_t tA = (MODE == MODE_OUTPUT) ? TO_A : TS_A;
            tmem_ld32(tl + tA + 32 * hf, v);
            if (lane < 16) {
                const int i = 16 * q4 + lane;
                const float bi = sBeta[i];
#pragma unroll
                for (int j4 = 0; j4 < 8; ++j4) {
                    float4 f;
                    const int j = 32 * hf + 4 * j4;
                    f.x = (j + 0 < i) ? bi * v[4 * j4 + 0] : 0.f;
                    f.y = (j + 1 < i) ? bi * v[4 * j4 + 1] : 0.f;
                    f.z = (j + 2 < i) ? bi * v[4 * j4 + 2] : 0.f;
                    f.w = (j + 3 < i) ? bi * v[4 * j4 + 3] : 0.f;
                    *reinterpret_cast<float4*>(Afp + sw(i, j)) = f;
                }
            }
        }
        __syncthreads();
        if (*sAbort) break;
        // ---- 4. T = (I + A)^{-1}: 16x16 diagonal blocks by substitution, then the
        //         off-diagonal blocks T_IJ = -T_II sum_{K=J}^{I-1} A_IK T_KJ -------------
        if (t < 64) {
            const int blk = t >> 4, m = t & 15, base = 16 * blk;
            float tc_[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float s = (r == m) ? 1.f : 0.f;
#pragma unroll
                for (int j = 0; j < r; ++j) s = fmaf(-Afp[sw(base + r, base + j)], tc_[j], s);
                tc_[r] = s;
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) Tfp[sw(base + r, base + m)] = tc_[r];
        }
        __syncthreads();
        for (int d = 1; d < 4; ++d) {
            const int nb = 4 - d;
            for (int idx = t; idx < nb * 256; idx += NT) {
                const int J = idx >> 8, I = J + d, r = (idx >> 4) & 15, cc = idx & 15;
                float s = 0.f;
                for (int K = J; K < I; ++K)
#pragma unroll
                    for (int k = 0; k < 16; ++k)
                        s = fmaf(Afp[sw(16 * I + r, 16 * K + k)], Tfp[sw(16 * K + k, 16 * J + cc)], s);
                sXs[idx] = s;
            }
            __syncthreads();
            for (int idx = t; idx < nb * 256; idx += NT) {
                const int J = idx >> 8, I = J + d, r = (idx >> 4) & 15, cc = idx & 15;
                float s = 0.f;
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    s = fmaf(Tfp[sw(16 * I + r, 16 * I + k)], sXs[(J << 8) + k * 16 + cc], s);
                Tfp[sw(16 * I + r, 16 * J + cc)] = -s;
            }
            __syncthreads();
        }
        // T' = T diag(beta), lower part only, fp16 K-major tile [i][j] at KM
        {
            float vals[2][8];
            int ii[2], jg[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int idx = t + u * NT;       // 512 (row, 8-column group) pairs
                ii[u] = idx >> 3;
                jg[u] = idx & 7;
                const float4 a0 = *reinterpret_cast<const float4*>(Tfp + sw(ii[u], 8 * jg[u]));
                const float4 a1 = *reinterpret_cast<const float4*>(Tfp + sw(ii[u], 8 * jg[u] + 4));
                const float f[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int col = 8 * jg[u] + j;
                    vals[u][j] = (col <= ii[u]) ? f[j] * sBeta[col] : 0.f;
                }
            }
            __syncthreads();
#pragma unroll
            for (int u = 0; u < 2; ++u)
                *reinterpret_cast<uint4*>(sm + PL::KM + jg[u] * 1024 + (ii[u] >> 3) * 128 + (ii[u] & 7) * 16) =
                    pack8_f16(vals[u]);
        }
        // P (masked, fp16 K-major) next to T'
        if (MODE == MODE_OUTPUT) {
            float v[32];
            tmem_ld32(tl + TO_P + 32 * hf, v);
            if (lane < 16) {
                const int i = 16 * q4 + lane;
#pragma unroll
                for (int g8 = 0; g8 < 4; ++g8) {
                    float f[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int col = 32 * hf + 8 * g8 + j;
                        f[j] = (col <= i) ? v[8 * g8 + j] : 0.f;
                    }
                    const int jgp = 4 * hf + g8;
                    *reinterpret_cast<uint4*>(sm + PL::KM + 8192 + jgp * 1024 + (i >> 3) * 128 + (i & 7) * 16) =
                        pack8_f16(f);
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        // ---- 5. U~ = T' V,  W = T' K+  (and O = Q+ S^) ---------------------------------
        if (t == 0) {
            tc_fence_after();
            const uint32_t id128 = idesc_f16(64, 128, false, false);
            const uint32_t tU = (MODE == MODE_OUTPUT) ? TO_U : TS_R;
            const uint32_t tW = (MODE == MODE_OUTPUT) ? TO_W : TS_W;
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t ad = sdesc(sbase + PL::KM + 2048 * kk, 1024, 128);
                umma_f16(tmem + tU, ad, sdesc(sbase + PL::X + 2048 + 8192 * kk, 4096, 128), id128, kk > 0);
                umma_f16(tmem + tW, ad, sdesc(sbase + PL::X + 8192 * kk, 4096, 128), id128, kk > 0);
            }
            if (MODE == MODE_OUTPUT) {
                const uint32_t idq = idesc_f16(64, 128, true, true);
                for (int kk = 0; kk < 8; ++kk)
                    umma_f16(tmem + TO_O, sdesc(sbase + PL::QP + 256 * kk, 128, 2048),
                             sdesc(sbase + PL::S + 256 * kk, 128, 2048), idq, kk > 0);
            }
            umma_commit(ctl.mma_bar);
        }
        mma_in_flight = true;
        wait_mma(ctl);
        mma_in_flight = false;
        // W -> fp16 K-major tile [i][c] at X (K+ | V are no longer needed)
        {
            const uint32_t tW = (MODE == MODE_OUTPUT) ? TO_W : TS_W;
            for (int cc = 0; cc < 64; cc += 32) {
                float v[32];
                tmem_ld32(tl + tW + 64 * hf + cc, v);
                if (lane < 16) {
                    const int i = 16 * q4 + lane;
#pragma unroll
                    for (int g8 = 0; g8 < 4; ++g8) {
                        const int cg = (64 * hf + cc) / 8 + g8;
                        *reinterpret_cast<uint4*>(sm + PL::X + cg * 1024 + (i >> 3) * 128 + (i & 7) * 16) =
                            pack8_f16(&v[8 * g8]);
                    }
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (*sAbort) break;
        // ---- 6. U = U~ - W S^  (critical path) -----------------------------------------
        if (t == 0) {
            tc_fence_after();
            const uint32_t idn = idesc_f16(64, 128, false, true, true);
            const uint32_t tU = (MODE == MODE_OUTPUT) ? TO_U : TS_R;
            for (int kk = 0; kk < 8; ++kk)
                umma_f16(tmem + tU, sdesc(sbase + PL::X + 2048 * kk, 1024, 128),
                         sdesc(sbase + PL::S + 256 * kk, 128, 2048), idn, 1);
            if (MODE == MODE_STATE) {
                // identity columns carry no values: their U starts at -W Phi^
                for (int kk = 0; kk < 8; ++kk)
                    umma_f16(tmem + TS_W, sdesc(sbase + PL::X + 2048 * kk, 1024, 128),
                             sdesc(sbase + PL::S + 32768 + 256 * kk, 128, 2048), idn, kk > 0);
            }
            umma_commit(ctl.mma_bar);
        }
        mma_in_flight = true;
        wait_mma(ctl);
        mma_in_flight = false;
        // U -> fp16 MN-major tile [i][col] at U
        {
            const uint32_t tU = (MODE == MODE_OUTPUT) ? TO_U : TS_R;
            constexpr int NU = NS;                 // 128 or 256 columns (contiguous in TMEM)
            for (int cc = 0; cc < NU / 2; cc += 32) {
                float v[32];
                tmem_ld32(tl + tU + hf * (NU / 2) + cc, v);
                if (lane < 16) {
                    const int i = 16 * q4 + lane;
#pragma unroll
                    for (int g8 = 0; g8 < 4; ++g8) {
                        const int cg = (hf * (NU / 2) + cc) / 8 + g8;
                        *reinterpret_cast<uint4*>(sm + PL::U + cg * 1024 + (i >> 3) * 128 + (i & 7) * 16) =
                            pack8_f16(&v[8 * g8]);
                    }
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        // ---- 7. S += Kt^T U  (and O += P U) ---------------------------------------------
        if (t == 0) {
            tc_fence_after();
            const uint32_t ids = idesc_f16(128, NS, false, true);
            for (int kk = 0; kk < 4; ++kk)
                umma_f16(tmem + TM_S, sdesc(sbase + PL::KT + 4096 * kk, 2048, 128),
                         sdesc(sbase + PL::U + 256 * kk, 128, 1024), ids, 1);
            if (MODE == MODE_OUTPUT) {
                const uint32_t ido = idesc_f16(64, 128, false, true);
                for (int kk = 0; kk < 4; ++kk)
                    umma_f16(tmem + TO_O, sdesc(sbase + PL::KM + 8192 + 2048 * kk, 1024, 128),
                             sdesc(sbase + PL::U + 256 * kk, 128, 1024), ido, 1);
            }
            umma_commit(ctl.mma_bar);
        }
        mma_in_flight = true;
        wait_mma(ctl);
        mma_in_flight = false;
        // ---- 8. outputs ----------------------------------------------------------------
        if (MODE == MODE_OUTPUT) {
            for (int cc = 0; cc < 64; cc += 32) {
                float v[32];
                tmem_ld32(tl + TO_O + 64 * hf + cc, v);
                const int i = 16 * q4 + lane;
                if (lane < 16 && t0 + i < T) {
                    const size_t off = (((size_t)b * T + t0 + i) * H + h) * D + 64 * hf + cc;
                    if (o_f32) {
                        float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(o) + off);
#pragma unroll
                        for (int j = 0; j < 8; ++j) dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
                    } else {
                        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(o) + off);
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            uint4 u;
                            __nv_bfloat162* hh = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
                            for (int e = 0; e < 4; ++e) hh[e] = __floats2bfloat162_rn(v[8 * j + 2 * e], v[8 * j + 2 * e + 1]);
                            dst[j] = u;
                        }
                    }
                }
            }
        }
        tc_fence_before();
        __syncthreads();
    }

    // ---- end of segment: write the state ------------------------------------------------
    if (!*sAbort) {
        float* dst = nullptr;
        if (MODE == MODE_STATE) dst = maps + (size_t)(bh * (P - 1) + p) * 2 * D * D;  // [N | M]
        else if (S_T && p == P - 1) dst = S_T + (size_t)bh * D * D;
        if (dst) {
            const int col0 = hf * (NS / 2);
            for (int cc = 0; cc < NS / 2; cc += 32) {
                float v[32];
                tmem_ld32(tl + TM_S + col0 + cc, v);
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int col = col0 + cc + j;
                    // maps: N block (value columns) then M block (identity columns)
                    const size_t idx = (col < D) ? ((size_t)c * D + col) : ((size_t)D * D + (size_t)c * D + (col - D));
                    dst[idx] = v[j];
                }
            }
        }
    }
    // ---- teardown: drain what is in flight, free TMEM ---------------------------------
    if (*sAbort) {
        if (mma_in_flight) mbar_wait_bounded(ctl.mma_bar, ctl.mma_phase, kWaitNs);
        if (tma_in_flight) mbar_wait_bounded(ctl.tma_bar, ctl.tma_phase, kWaitNs);
    }
    tc_fence_before();
    __syncthreads();
    if (w == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// S_start(p+1) = M_p S_start(p) + N_p, fp32 on CUDA cores.  Grid (D/8, H, B), 128
// threads: thread c owns row c of an 8-column slice of the state.
__global__ void __launch_bounds__(128)
kda_combine_kernel(const float* __restrict__ maps, const float* __restrict__ S0,
                   float* __restrict__ starts, int H, int P)
{
    __shared__ float sS[D][8];
    const int c = threadIdx.x, col0 = blockIdx.x * 8;
    const int bh = blockIdx.z * H + blockIdx.y;
    float s[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) s[j] = S0 ? S0[((size_t)bh * D + c) * D + col0 + j] : 0.f;
    for (int p = 0; p < P; ++p) {
        float* out = starts + ((size_t)bh * P + p) * D * D + (size_t)c * D + col0;
#pragma unroll
        for (int j = 0; j < 8; ++j) out[j] = s[j];
        if (p == P - 1) break;
        __syncthreads();
#pragma unroll
        for (int j = 0; j < 8; ++j) sS[c][j] = s[j];
        __syncthreads();
        const float* Nm = maps + ((size_t)bh * (P - 1) + p) * 2 * D * D;
        const float* Mm = Nm + D * D;
        float acc[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] = Nm[(size_t)c * D + col0 + j];
        const float4* mrow = reinterpret_cast<const float4*>(Mm + (size_t)c * D);
        for (int k4 = 0; k4 < D / 4; ++k4) {
            const float4 m = mrow[k4];
            const float mk[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[j] = fmaf(mk[u], sS[4 * k4 + u][j], acc[j]);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) s[j] = acc[j];
    }
}

// ---- host side ----------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// [B*T, H, 128] tensor of 2-byte elements, box = 64 tokens x 1 head x 128 channels.
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int B, int T, int H)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)B * (cuuint64_t)T};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
    const cuuint32_t box[3] = {(cuuint32_t)D, 1u, (cuuint32_t)C};
    const cuuint32_t es[3] = {1u, 1u, 1u};
    return fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct Split {
    int P, L;
};
Split split_for(int B, int T, int H, int num_sms)
{
    const int NC = (T + C - 1) / C;
    int P = num_sms / max(1, B * H);
    P = max(1, min(P, NC));
    const int L = (NC + P - 1) / P;
    P = (NC + L - 1) / L;  // no empty segment
    return {P, L};
}

template <int MODE, typename TQ>
cudaError_t launch_pass(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                        const CUtensorMap& mg, const KdaArgs& a, const float* S_in, int per_seg,
                        float* maps, int P, int L, int* status, cudaStream_t s)
{
    auto kern = kda_tc_kernel<MODE, TQ>;
    const int smem = smem_bytes<MODE>();
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int nseg = MODE == MODE_STATE ? P - 1 : P;
    const unsigned grid = (unsigned)(a.B * a.H * nseg);
    ProfileScope prof(MODE == MODE_STATE ? "kda_tc_state" : "kda_tc_output", s);
    count_launch();
    kern<<<grid, NT, smem, s>>>(mq, mk, mv, mg, (const __nv_bfloat16*)a.beta, a.o, a.out_t == ET_F32 ? 1 : 0,
                                S_in, per_seg, maps, a.ST, a.B, a.T, a.H, P, L, status);
    return cudaGetLastError();
}

template <typename TQ>
cudaError_t launch_all(const KdaArgs& a, void* ws, int* status, cudaStream_t s)
{
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const Split sp = split_for(a.B, a.T, a.H, sms);
    const CUtensorMapDataType dq =
        std::is_same<TQ, __half>::value ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    CUtensorMap mq, mk, mv, mg;
    if (!make_map(&mq, a.q, dq, a.B, a.T, a.H) || !make_map(&mk, a.k, dq, a.B, a.T, a.H) ||
        !make_map(&mv, a.v, dq, a.B, a.T, a.H) ||
        !make_map(&mg, a.g, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.B, a.T, a.H))
        return cudaErrorInvalidValue;
    if (sp.P == 1)
        return launch_pass<MODE_OUTPUT, TQ>(mq, mk, mv, mg, a, a.S0, 0, nullptr, 1, sp.L, status, s);
    float* maps = reinterpret_cast<float*>(ws);
    float* starts = maps + (size_t)a.B * a.H * (sp.P - 1) * 2 * D * D;
    cudaError_t e = launch_pass<MODE_STATE, TQ>(mq, mk, mv, mg, a, nullptr, 0, maps, sp.P, sp.L, status, s);
    if (e != cudaSuccess) return e;
    {
        ProfileScope prof("kda_tc_combine", s);
        count_launch();
        kda_combine_kernel<<<dim3(D / 8, a.H, a.B), 128, 0, s>>>(maps, a.S0, starts, a.H, sp.P);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return launch_pass<MODE_OUTPUT, TQ>(mq, mk, mv, mg, a, starts, 1, maps, sp.P, sp.L, status, s);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

bool kda_tc_supported(const KdaArgs& a)
{
    if (a.Dk != D || a.Dv != D || a.chunk != C || a.T < 1) return false;
    if (a.in_t != ET_BF16 && a.in_t != ET_F16) return false;
    if (a.gb_t != ET_BF16) return false;
    if (a.out_t != ET_BF16 && a.out_t != ET_F32) return false;
    if (!aligned16(a.q) || !aligned16(a.k) || !aligned16(a.v) || !aligned16(a.g) || !aligned16(a.o)) return false;
    return encode_fn() != nullptr;
}

size_t kda_tc_workspace_bytes(int B, int T, int H, int chunk, int num_sms)
{
    if (chunk != C || T < 1) return 0;
    const Split sp = split_for(B, T, H, num_sms);
    if (sp.P == 1) return 0;
    return (size_t)B * H * ((size_t)(sp.P - 1) * 2 + sp.P) * D * D * sizeof(float);
}

cudaError_t launch_kda_tc(const KdaArgs& a, void* ws, size_t ws_bytes, int* status, cudaStream_t s)
{
    (void)ws_bytes;
    if (a.in_t == ET_F16) return launch_all<__half>(a, ws, status, s);
    return launch_all<__nv_bfloat16>(a, ws, status, s);
}

}  // namespace kda
