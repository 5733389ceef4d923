// Tensor-core (tcgen05 / TMEM / TMA) chunkwise KDA forward for Dk = Dv = 128, chunk 64.
//
// What it computes is Eq. 14 of the Chimera paper (section 3.3) with the readout
// o_t = S_t^T q_t (Eq. 15, inner term).  The pages only say the kernel is "chunked";
// the chunk algebra is derived from Eq. 14.  Inside a chunk of C = 64 tokens with
// entry state S0, b_i = sum_{r<=i} g_r (fp32, per key channel), a reference point
// r = b_31 (the middle of the chunk) keeps every exponential within e^{+-|b|/2}:
//   K+ = k e^{b - r},  Q+ = q e^{b - r},  K- = k e^{r - b}
//   A  = strict_lower((diag(beta) K+) K-^T),   P = lower(Q+ K-^T)  (incl. diagonal)
//   T  = (I + A)^{-1}                     (16x16 blocks on warp MMAs, fp16 operands)
//   S^ = diag(e^{r}) S0,   Y = (diag(beta) K+) S^
//   U  = T (beta V) - T Y                 O = Q+ S^ + P U
//   S_C = diag(e^{b_C - r}) (S^ + K-^T U)     (k e^{b_C - b} = K- diag(e^{b_C - r}))
// The state's fp32 master copy lives in TMEM in the scaled form S^ + K-^T U: the row
// scale e^{b_C - r} of one chunk and e^{r'} of the next are applied together, once,
// when the next chunk reads it.  Every MMA operand is fp16 in shared memory (11-bit
// significand: bf16 operands would cost ~3% of RMS(o) in max error); accumulation is
// fp32 in TMEM.  Exponents are kept in base 2 (g log2(e) summed in fp32).
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
// Each pass is one CTA per (b, h, segment), 512 threads, ~200 KB of shared memory.
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
constexpr int NT = 512;       // threads per CTA
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s bound on every wait
constexpr float kLog2e = 1.4426950408889634f;
enum { MODE_STATE = 0, MODE_OUTPUT = 1 };

// ---- shared-memory plan (bytes) --------------------------------------------------
// Channel-major fp16 tiles (K+ beta, Q+, K-, beta V): 8-position group ig at
// tile + ig*2048, channel c at (c >> 3)*128 + (c & 7)*16 inside it.  Q+ follows K+ beta
// directly, so [beta K+; Q+] is one M = 128 operand.  After the Y MMA the S^ region
// holds Y (position-major: 8-position group j at j*NS*16, 8 columns per 16 bytes).
template <int MODE> struct Plan;
template <> struct Plan<MODE_OUTPUT> {
    static constexpr int NS = 128;                 // state columns (values only)
    static constexpr int stQ = 0, stK = 16384, stV = 32768, stG = 49152;  // TMA staging, [64][128]
    static constexpr int KP = 65536;               // beta K+
    static constexpr int QP = 81920;               // Q+
    static constexpr int KM = 98304;               // K-
    static constexpr int VB = 114688;              // beta V
    static constexpr int TF = 131072;              // T (64 x 64 fp16, K-major, 8-column groups 2 KB
                                                   // apart) interleaved with P in the other 1 KB halves
    static constexpr int U = 147456;               // fp16 A during the inverse, then U (64 x 128)
    static constexpr int S = 163840;               // S^ (128 x 128 fp16), then Y
    static constexpr int MISC = 196608;
    static constexpr int TMA_BYTES = 4 * 16384;
};
template <> struct Plan<MODE_STATE> {
    static constexpr int NS = 256;                 // [S | Phi]
    static constexpr int stQ = -1, stK = 0, stV = 16384, stG = 32768;
    static constexpr int KP = 49152;
    static constexpr int QP = -1;
    static constexpr int KM = 65536;
    static constexpr int VB = 81920;
    static constexpr int TF = -1;                  // T lives at U + 8192
    static constexpr int U = 98304;                // fp16 A and T during the inverse, then U (64 x 256)
    static constexpr int S = 131072;               // [S^ | Phi^] (128 x 256 fp16), then Y
    static constexpr int MISC = 196608;
    static constexpr int TMA_BYTES = 3 * 16384;
};
// MISC sub-layout
constexpr int M_BETA = 0;        // float[64]
constexpr int M_TOT = 256;       // float[8][128] per-8-row-block sums of g log2(e)
constexpr int M_XS = 4352;       // 8 x 512 B per-warp 16x16 fp16 scratch of the inverse
constexpr int M_BAR = 8448;      // 4 x uint64 mbarriers (TMA, MMA, second issuer, A read)
constexpr int M_TMEM = 8480;     // uint32 TMEM base
constexpr int M_ABORT = 8484;    // int
constexpr int MISC_BYTES = 8496;

template <int MODE> constexpr int smem_bytes() { return Plan<MODE>::MISC + MISC_BYTES; }

// TMEM columns.
constexpr uint32_t TM_S = 0;     // state master (fp32), 128 or 256 columns
constexpr uint32_t T_AP = 256;   // A (and P below it in MODE_OUTPUT), 64 columns
// MODE_OUTPUT: [Y; O] (M = 128) at 128, U (M = 64) at 384.
// MODE_STATE:  Y, then U (M = 64, 256 columns) at 256, once A has been read.
template <int MODE> struct Tm;
template <> struct Tm<MODE_OUTPUT> { static constexpr uint32_t Y = 128, UU = 384; };
template <> struct Tm<MODE_STATE> { static constexpr uint32_t Y = 256, UU = 256; };

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

// Byte offset of (row i, column j), j % 8 == 0, in a 64 x 64 fp16 tile in the
// K-major core-matrix layout the tensor-core MMA reads (8-column groups 1 KB apart).
__device__ __forceinline__ uint32_t cm64(int i, int j) { return (j >> 3) * 1024 + (i >> 3) * 128 + (i & 7) * 16; }
// Same for a 16 x 16 scratch block (8-column groups 256 B apart).
__device__ __forceinline__ uint32_t cm16(int i, int j) { return (j >> 3) * 256 + (i >> 3) * 128 + (i & 7) * 16; }

// Warp-MMA helpers on 16x16 blocks.  A C fragment pair (two n-halves) is exactly the
// A fragment of the next product; B fragments go through a per-warp scratch block.
__device__ __forceinline__ void c_to_a(uint32_t (&a)[4], const float (&c0)[4], const float (&c1)[4])
{
    a[0] = pack_f16x2(c0[0], c0[1]);
    a[1] = pack_f16x2(c0[2], c0[3]);
    a[2] = pack_f16x2(c1[0], c1[1]);
    a[3] = pack_f16x2(c1[2], c1[3]);
}
// C fragments (rows g, g+8; columns 2q, 2q+1 of each n-half) -> 16x16 fp16 scratch
__device__ __forceinline__ void c_to_scr(uint32_t scr, int lane, const float (&c0)[4], const float (&c1)[4])
{
    const int g = lane >> 2, q = lane & 3;
    st_shared_b32(scr + cm16(g, 0) + 4 * q, pack_f16x2(c0[0], c0[1]));
    st_shared_b32(scr + cm16(g + 8, 0) + 4 * q, pack_f16x2(c0[2], c0[3]));
    st_shared_b32(scr + cm16(g, 8) + 4 * q, pack_f16x2(c1[0], c1[1]));
    st_shared_b32(scr + cm16(g + 8, 8) + 4 * q, pack_f16x2(c1[2], c1[3]));
}
// B fragments (both n-halves) of a 16x16 block stored [k][n] in the scratch
__device__ __forceinline__ void scr_to_b(uint32_t (&b)[4], uint32_t scr, int lane)
{
    ldsm_x4_t(b, scr + cm16((lane & 7) + 8 * ((lane >> 3) & 1), 8 * (lane >> 4)));
}
__device__ __forceinline__ void mma_16x16(float (&c0)[4], float (&c1)[4], const uint32_t (&a)[4], const uint32_t (&b)[4])
{
    const uint32_t b0[2] = {b[0], b[1]}, b1[2] = {b[2], b[3]};
    mma16816(c0, a, b0);
    mma16816(c1, a, b1);
}

__device__ __forceinline__ void named_sync(int id, int nthreads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

struct Ctl {
    uint64_t* tma_bar;
    uint64_t* mma_bar;
    int* abort_flag;
    int* status;
    uint32_t tma_phase, mma_phase;
};

// Bounded waits.  One thread polls the mbarrier; the others wait at a barrier (no
// issue slots spent polling): the whole CTA (bar_id 0) or one 256-thread group.  The
// CTA agrees on a timeout through the shared abort flag.  After an MMA wait every
// thread orders its TMEM reads behind it.
__device__ __forceinline__ void wait_bar(uint64_t* bar, uint32_t& phase, Ctl& c, bool poller, int bar_id)
{
    if (poller && !mbar_wait_bounded(bar, phase, kWaitNs)) {
        *c.abort_flag = 1;
        atomicCAS(c.status, DEV_OK, DEV_TIMEOUT);
    }
    if (bar_id == 0) __syncthreads();
    else named_sync(bar_id, NT / 2);
    phase ^= 1;
    tc_fence_after();
}
__device__ __forceinline__ void wait_mma(Ctl& c, int t) { wait_bar(c.mma_bar, c.mma_phase, c, t == 0, 0); }
__device__ __forceinline__ void wait_tma(Ctl& c, int t) { wait_bar(c.tma_bar, c.tma_phase, c, t == 0, 0); }

// Two adjacent 2-byte input elements -> fp32
__device__ __forceinline__ float2 in2(uint32_t u, const __nv_bfloat16*)
{
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}
__device__ __forceinline__ float2 in2(uint32_t u, const __half*) { return unpack_f16x2(u); }

// Output rows of one chunk from TMEM to global memory.  O is rows 64-127 of the
// M = 128 accumulator [Y; O]: output row i sits in lane 64 + i, so warps of lane
// quarters 2 and 3 store it; this warp stores columns col0 .. col0 + 32*nld - 1.
__device__ __forceinline__ void store_o(uint32_t tl, int q4, int col0, int nld, int lane, void* o, int o_f32,
                                        int b, int T, int H, int h, int t0)
{
    for (int u = 0; u < nld; ++u) {
        float v[32];
        const int cc = col0 + 32 * u;
        tmem_ld32(tl + Tm<MODE_OUTPUT>::Y + cc, v);
        const int i = 32 * (q4 - 2) + lane;
        if (t0 + i < T) {
            const size_t off = (((size_t)b * T + t0 + i) * H + h) * D + cc;
            if (o_f32) {
                float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(o) + off);
#pragma unroll
                for (int j = 0; j < 8; ++j) dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
            } else {
                uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(o) + off);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    uint4 uu;
                    __nv_bfloat162* hh = reinterpret_cast<__nv_bfloat162*>(&uu);
#pragma unroll
                    for (int e = 0; e < 4; ++e) hh[e] = __floats2bfloat162_rn(v[8 * j + 2 * e], v[8 * j + 2 * e + 1]);
                    dst[j] = uu;
                }
            }
        }
    }
}

// The kernel ---------------------------------------------------------------------------
// 512 threads.  Prologue: thread t owns key channels 2*(t & 63) + {0, 1} and chunk rows
// 8*(t >> 6) .. +7.  TMEM: warp w reads lane quarter w & 3.  While warps 0-7 read A and
// invert (I + A), warps 8-15 store the previous chunk's output, rescale the state,
// issue Y (and O) from S^, and read P and Y.
template <int MODE, typename TQ>
__global__ void __launch_bounds__(NT, 1)
kda_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
              const __nv_bfloat16* __restrict__ beta, void* __restrict__ o, int o_f32,
              const float* __restrict__ S_in, int s_in_per_segment, float* __restrict__ maps,
              float* __restrict__ S_T, int B, int T, int H, int P, int L, int* status)
{
    using PL = Plan<MODE>;
    constexpr bool OUT = MODE == MODE_OUTPUT;
    constexpr int NS = PL::NS;
    constexpr int NQ = NS / 4;                // state columns per column quarter (all 16 warps)
    constexpr int YJ = NS * 16;               // Y tile: bytes per 8-position group
    constexpr uint32_t T_Y = Tm<MODE>::Y, T_UU = Tm<MODE>::UU;
    constexpr int TT = OUT ? PL::TF : PL::U + 8192;   // T tile base
    constexpr int T_LBO = OUT ? 2048 : 1024;          // T's 8-column group stride
    auto cmT = [](int i, int j) -> uint32_t { return (j >> 3) * T_LBO + (i >> 3) * 128 + (i & 7) * 16; };
    extern __shared__ __align__(1024) uint8_t sm[];

    const int t = threadIdx.x, w = t >> 5, lane = t & 31;
    const int q4 = w & 3, cq = w >> 2;        // TMEM lane quarter, column quarter
    const bool grpY = w >= 8;                 // second 256-thread group
    const int hg = (w >> 2) & 1;              // column half inside a group
    const int c = t & 127;                    // channel / TMEM row of the state steps
    const int cp = t & 63, rb = t >> 6;       // prologue: channel pair, 8-row block
    const int nseg = (MODE == MODE_STATE) ? P - 1 : P;
    const int bh = blockIdx.x / nseg, p = blockIdx.x % nseg;
    const int b = bh / H, h = bh % H;
    const int NC = (T + C - 1) / C;
    const int n0 = p * L, n1 = min(NC, n0 + L);

    float* sBeta = reinterpret_cast<float*>(sm + PL::MISC + M_BETA);
    float* sTot = reinterpret_cast<float*>(sm + PL::MISC + M_TOT);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + PL::MISC + M_BAR);
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(sm + PL::MISC + M_TMEM);
    int* sAbort = reinterpret_cast<int*>(sm + PL::MISC + M_ABORT);
    const uint32_t sbase = smem_addr(sm);

    Ctl ctl{&bars[0], &bars[1], sAbort, status, 0u, 0u};
    uint64_t* y_bar = &bars[2];       // MMAs issued by thread NT/2 (Y, and O in MODE_OUTPUT)
    uint64_t* a_bar = &bars[3];       // MODE_STATE: A has been read out of TMEM
    uint32_t y_phase = 0, a_phase = 0;
    bool y_in_flight = false;
    if (t == 0) {
        mbar_init(ctl.tma_bar, 1);
        mbar_init(ctl.mma_bar, 1);
        mbar_init(y_bar, 1);
        mbar_init(a_bar, 1);
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
        if (OUT) tma_load_3d(sm + PL::stQ, &tm_q, ctl.tma_bar, 0, h, row);
        tma_load_3d(sm + PL::stK, &tm_k, ctl.tma_bar, 0, h, row);
        tma_load_3d(sm + PL::stV, &tm_v, ctl.tma_bar, 0, h, row);
        tma_load_3d(sm + PL::stG, &tm_g, ctl.tma_bar, 0, h, row);
    };
    // beta is prefetched one chunk ahead as raw bf16 bits (no use until the next chunk,
    // so the load never stalls the thread); the index is clamped to stay in bounds.
    auto load_beta_bits = [&](int n) -> uint32_t {
        const int tt = n * C + t;
        const int ts = (n < n1 && tt < T) ? tt : 0;
        return *reinterpret_cast<const unsigned short*>(beta + ((size_t)b * T + ts) * H + h);
    };
    if (t == 0 && n0 < n1) issue_tma(n0);
    tma_in_flight = n0 < n1;
    uint32_t beta_bits = (t < C) ? load_beta_bits(n0) : 0u;

    // ---- initial state in TMEM ------------------------------------------------------
    {
        const int col0 = cq * NQ;
        for (int cc = 0; cc < NQ; cc += 32) {
            float v[32];
            if (MODE == MODE_STATE) {
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int col = col0 + cc + j;
                    v[j] = (col >= D && col - D == c) ? 1.f : 0.f;
                }
            } else if (S_in) {
                const size_t idx = s_in_per_segment ? (size_t)bh * P + p : (size_t)bh;
                const float4* s4 = reinterpret_cast<const float4*>(S_in + (idx * D + c) * D + col0 + cc);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float4 x = s4[j];
                    v[4 * j] = x.x; v[4 * j + 1] = x.y; v[4 * j + 2] = x.z; v[4 * j + 3] = x.w;
                }
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = 0.f;
            }
            tmem_st32(tl + TM_S + col0 + cc, v);
        }
    }
    tc_fence_before();
    __syncthreads();

    // The master holds diag(2^{-carry}) S for channel c (log2 units; 0 before any chunk).
    float carry = 0.f;
    int prev_t0 = -1;   // chunk whose output still sits in TMEM (MODE_OUTPUT)
    for (int n = n0; n < n1 && !*sAbort; ++n) {
        const int t0 = n * C;
        // ---- 1. prologue: staging -> fp16 operand tiles --------------------------------
        wait_tma(ctl, t);
        if (*sAbort) break;
        tma_in_flight = false;
        if (t < C) {
            sBeta[t] = (t0 + t < T) ? __uint_as_float(beta_bits << 16) : 0.f;
            beta_bits = load_beta_bits(n + 1);    // in flight during this chunk
        }
        const bool full = t0 + C <= T;   // no ragged rows in this chunk
        const int nvalid = T - t0;       // rows i < nvalid are tokens
        float2 bl[8];                    // b log2(e) for this thread's two channels, rows 8*rb + r
        {
            const uint32_t* stg = reinterpret_cast<const uint32_t*>(sm + PL::stG) + cp;
            float2 run = make_float2(0.f, 0.f);
            const float2 l2e = make_float2(kLog2e, kLog2e);
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const int i = 8 * rb + r;
                float2 gv = in2(stg[i * (D / 2)], (const __nv_bfloat16*)nullptr);
                if (!full && i >= nvalid) gv = make_float2(0.f, 0.f);
                run = __ffma2_rn(gv, l2e, run);
                bl[r] = run;
            }
            *reinterpret_cast<float2*>(sTot + rb * D + 2 * cp) = run;
        }
        __syncthreads();
        float2 xo;              // (sum of the earlier row blocks) - r, this thread's channel pair
        float s_scale;          // state row scale for channel c: 2^{r + carry}
        {
            float2 off = make_float2(0.f, 0.f), r2 = make_float2(0.f, 0.f);
            float rc = 0.f, bc = 0.f;
#pragma unroll
            for (int qb = 0; qb < 8; ++qb) {
                const float2 v = *reinterpret_cast<const float2*>(sTot + qb * D + 2 * cp);
                if (qb < rb) off = __fadd2_rn(off, v);
                if (qb < 4) r2 = __fadd2_rn(r2, v);
                bc += sTot[qb * D + c];
                if (qb == 3) rc = bc;
            }
            xo = make_float2(off.x - r2.x, off.y - r2.y);
            s_scale = ex2_approx(rc + carry);
            carry = bc - rc;
        }
        {
            const TQ* tq = nullptr;
            const uint32_t* sk = reinterpret_cast<const uint32_t*>(sm + PL::stK) + cp;
            const uint32_t* sv = reinterpret_cast<const uint32_t*>(sm + PL::stV) + cp;
            const uint32_t* sq = reinterpret_cast<const uint32_t*>(sm + (OUT ? PL::stQ : PL::stK)) + cp;
            // packed fp16 pairs (rows 2m, 2m+1) per channel: [channel][m]
            uint32_t pk[2][4], pm[2][4], pv[2][4], pq[2][4];
            float2 lk, lm, lv, lq;   // even row, waiting for its odd partner
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const int i = 8 * rb + r;
                const bool valid = full || i < nvalid;
                float2 kk = in2(sk[i * (D / 2)], tq), vv = in2(sv[i * (D / 2)], tq);
                float2 qq = OUT ? in2(sq[i * (D / 2)], tq) : make_float2(0.f, 0.f);
                if (!valid) kk = vv = qq = make_float2(0.f, 0.f);
                const float bi = sBeta[i];
                const float2 b2 = make_float2(bi, bi);
                const float2 x = __fadd2_rn(bl[r], xo);
                const float2 ep = make_float2(ex2_approx(x.x), ex2_approx(x.y));
                const float2 em = make_float2(ex2_approx(-x.x), ex2_approx(-x.y));
                const float2 kp = __fmul2_rn(__fmul2_rn(kk, b2), ep);   // beta K+
                const float2 km = __fmul2_rn(kk, em);                   // K-
                const float2 vb = __fmul2_rn(vv, b2);                   // beta V
                const float2 qp = __fmul2_rn(qq, ep);                   // Q+
                if (r & 1) {
                    const int m = r >> 1;
                    pk[0][m] = pack_f16x2(lk.x, kp.x); pk[1][m] = pack_f16x2(lk.y, kp.y);
                    pm[0][m] = pack_f16x2(lm.x, km.x); pm[1][m] = pack_f16x2(lm.y, km.y);
                    pv[0][m] = pack_f16x2(lv.x, vb.x); pv[1][m] = pack_f16x2(lv.y, vb.y);
                    pq[0][m] = pack_f16x2(lq.x, qp.x); pq[1][m] = pack_f16x2(lq.y, qp.y);
                } else {
                    lk = kp; lm = km; lv = vb; lq = qp;
                }
            }
            // Threads with (cp & 4) store their odd channel first: each 8-thread phase of a
            // 16-byte store then covers all 32 banks once.
            const bool sw = (cp & 4) != 0;
            const int c_first = 2 * cp + (sw ? 1 : 0), c_second = 2 * cp + (sw ? 0 : 1);
            const uint32_t o1 = rb * 2048 + (c_first >> 3) * 128 + (c_first & 7) * 16;
            const uint32_t o2 = rb * 2048 + (c_second >> 3) * 128 + (c_second & 7) * 16;
            auto st2 = [&](int tile, const uint32_t (&pp)[2][4]) {
                const uint4 a0 = make_uint4(pp[0][0], pp[0][1], pp[0][2], pp[0][3]);
                const uint4 a1 = make_uint4(pp[1][0], pp[1][1], pp[1][2], pp[1][3]);
                *reinterpret_cast<uint4*>(sm + tile + o1) = sw ? a1 : a0;
                *reinterpret_cast<uint4*>(sm + tile + o2) = sw ? a0 : a1;
            };
            st2(PL::KP, pk);
            st2(PL::KM, pm);
            st2(PL::VB, pv);
            if (OUT) st2(PL::QP, pq);
        }
        fence_async_smem();
        __syncthreads();
        // ---- 2. A (and P) on the tensor core ----------------------------------------------
        if (t == 0) {
            tc_fence_after();
            // [beta K+; Q+] (M = 128) x K-^T: rows 0-63 give A, rows 64-127 give P
            const uint32_t id = idesc_f16(OUT ? 128 : 64, 64, true, true);
            for (int kk = 0; kk < 8; ++kk)
                umma_f16(tmem + T_AP, sdesc(sbase + PL::KP + 256 * kk, 128, 2048),
                         sdesc(sbase + PL::KM + 256 * kk, 128, 2048), id, kk > 0);
            umma_commit(ctl.mma_bar);
        }
        tma_in_flight = n + 1 < n1;
        mma_in_flight = true;
        if (!grpY) {
            // ---- 3X. warps 0-7: A -> fp16 tile, then T = (I + A)^{-1} ---------------------------
            // A = diag(beta) strict_lower(K+ K-^T) (beta is already in K+).
            wait_bar(ctl.mma_bar, ctl.mma_phase, ctl, t == 0, 1);
            const uint32_t Ah = sbase + PL::U;       // A, fp16 K-major core-matrix tile
            const uint32_t Tt = sbase + TT;          // T: the next MMA's operand
            {
                float v[32];
                int i = -1;
                if (OUT) {
                    // M = 128 layout: row i in lane i; rows 0-63 (quarters 0, 1) are A
                    if (q4 < 2) {
                        tmem_ld32(tl + T_AP + 32 * hg, v);
                        i = 32 * q4 + lane;
                    }
                } else {
                    // M = 64 layout: row 16*q4 + l in lane 32*q4 + l (l < 16)
                    tmem_ld32(tl + T_AP + 32 * hg, v);
                    if (lane < 16) i = 16 * q4 + lane;
                }
                if (i >= 0) {
#pragma unroll
                    for (int g8 = 0; g8 < 4; ++g8) {
                        float f[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const int col = 32 * hg + 8 * g8 + j;
                            f[j] = (col < i) ? v[8 * g8 + j] : 0.f;
                        }
                        *reinterpret_cast<uint4*>(sm + PL::U + cm64(i, 32 * hg + 8 * g8)) = pack8_f16(f);
                    }
                }
                // the six upper 16x16 blocks of T are zero
                if (t < 192) {
                    const int e = t >> 5, u = t & 31;
                    const int I = (e < 3) ? 0 : (e < 5 ? 1 : 2);
                    const int J = (e < 3) ? e + 1 : (e < 5 ? e - 1 : 3);
                    const int row = 16 * I + 8 * (u >> 4) + (u & 7), col = 16 * J + 8 * ((u >> 3) & 1);
                    *reinterpret_cast<uint4*>(sm + TT + cmT(row, col)) = make_uint4(0u, 0u, 0u, 0u);
                }
            }
            tc_fence_before();
            named_sync(1, NT / 2);
            if (MODE == MODE_STATE && t == 0) mbar_arrive(a_bar);   // Y may now overwrite A's columns
            // diagonal 16x16 blocks (warp w < 4 owns block w): with N = A_ww (strictly lower,
            // N^16 = 0), (I + N)^{-1} = (I - N)(I + N^2)(I + N^4)(I + N^8) on warp MMAs
            if (w < 4) {
                const int b0 = 16 * w, g = lane >> 2, q = lane & 3;
                const uint32_t scr = sbase + PL::MISC + M_XS + 512 * w;
                uint32_t aN[4], bN[4], bP[4], aX[4];
                ldsm_x4(aN, Ah + cm64(b0 + (lane & 15), b0 + 8 * (lane >> 4)));
                ldsm_x4_t(bN, Ah + cm64(b0 + (lane & 7) + 8 * ((lane >> 3) & 1), b0 + 8 * (lane >> 4)));
                float n2a[4] = {0.f, 0.f, 0.f, 0.f}, n2b[4] = {0.f, 0.f, 0.f, 0.f};
                mma_16x16(n2a, n2b, aN, bN);                                   // N^2
                c_to_scr(scr, lane, n2a, n2b);
                __syncwarp();
                scr_to_b(bP, scr, lane);                                       // bP = N^2
                __syncwarp();
                c_to_a(aX, n2a, n2b);
                float n4a[4] = {0.f, 0.f, 0.f, 0.f}, n4b[4] = {0.f, 0.f, 0.f, 0.f};
                float n3a[4] = {0.f, 0.f, 0.f, 0.f}, n3b[4] = {0.f, 0.f, 0.f, 0.f};
                mma_16x16(n4a, n4b, aX, bP);                                   // N^4
                mma_16x16(n3a, n3b, aN, bP);                                   // N^3
                c_to_scr(scr, lane, n4a, n4b);
                __syncwarp();
                scr_to_b(bP, scr, lane);                                       // bP = N^4
                __syncwarp();
                c_to_a(aX, n4a, n4b);
                float n8a[4] = {0.f, 0.f, 0.f, 0.f}, n8b[4] = {0.f, 0.f, 0.f, 0.f};
                mma_16x16(n8a, n8b, aX, bP);                                   // N^8
                // Z = I - N + N^2 - N^3, in the C layout (rows g, g+8; columns 2q, 2q+1 of
                // each 8-column half); N's values come from its A fragment
                float za[4], zb[4];
                {
                    const float2 n00 = unpack_f16x2(aN[0]), n10 = unpack_f16x2(aN[1]);
                    const float2 n01 = unpack_f16x2(aN[2]), n11 = unpack_f16x2(aN[3]);
                    const float d0 = (g == 2 * q) ? 1.f : 0.f, d1 = (g == 2 * q + 1) ? 1.f : 0.f;
                    za[0] = d0 - n00.x + n2a[0] - n3a[0];
                    za[1] = d1 - n00.y + n2a[1] - n3a[1];
                    za[2] = -n10.x + n2a[2] - n3a[2];
                    za[3] = -n10.y + n2a[3] - n3a[3];
                    zb[0] = -n01.x + n2b[0] - n3b[0];
                    zb[1] = -n01.y + n2b[1] - n3b[1];
                    zb[2] = d0 - n11.x + n2b[2] - n3b[2];
                    zb[3] = d1 - n11.y + n2b[3] - n3b[3];
                }
                {   // Z += Z N^4
                    float ta[4] = {0.f, 0.f, 0.f, 0.f}, tb[4] = {0.f, 0.f, 0.f, 0.f};
                    c_to_a(aX, za, zb);
                    mma_16x16(ta, tb, aX, bP);
#pragma unroll
                    for (int k = 0; k < 4; ++k) { za[k] += ta[k]; zb[k] += tb[k]; }
                }
                c_to_scr(scr, lane, n8a, n8b);
                __syncwarp();
                scr_to_b(bP, scr, lane);                                       // bP = N^8
                {   // Z += Z N^8
                    float ta[4] = {0.f, 0.f, 0.f, 0.f}, tb[4] = {0.f, 0.f, 0.f, 0.f};
                    c_to_a(aX, za, zb);
                    mma_16x16(ta, tb, aX, bP);
#pragma unroll
                    for (int k = 0; k < 4; ++k) { za[k] += ta[k]; zb[k] += tb[k]; }
                }
                st_shared_b32(Tt + cmT(b0 + g, b0) + 4 * q, pack_f16x2(za[0], za[1]));
                st_shared_b32(Tt + cmT(b0 + g + 8, b0) + 4 * q, pack_f16x2(za[2], za[3]));
                st_shared_b32(Tt + cmT(b0 + g, b0 + 8) + 4 * q, pack_f16x2(zb[0], zb[1]));
                st_shared_b32(Tt + cmT(b0 + g + 8, b0 + 8) + 4 * q, pack_f16x2(zb[2], zb[3]));
            }
            named_sync(1, NT / 2);
            // block diagonal d: warp (block J, 8-column half) computes
            //   X = sum_{K=J}^{I-1} A_IK T_KJ  and  T_IJ = -T_II X   (I = J + d)
            for (int d = 1; d < 4; ++d) {
                if (w < 2 * (4 - d)) {
                    const int J = w >> 1, I = J + d, N0 = 16 * J + 8 * (w & 1);
                    const int g = lane >> 2, q = lane & 3;
                    const uint32_t scr = sbase + PL::MISC + M_XS + 512 * w;
                    float x[4] = {0.f, 0.f, 0.f, 0.f};
                    for (int K = J; K < I; ++K) {
                        uint32_t aA[4], bT[2];
                        ldsm_x4(aA, Ah + cm64(16 * I + (lane & 15), 16 * K + 8 * (lane >> 4)));
                        ldsm_x2_t(bT, Tt + cmT(16 * K + (lane & 7) + 8 * ((lane >> 3) & 1), N0));
                        mma16816(x, aA, bT);
                    }
                    st_shared_b32(scr + cm16(g, 0) + 4 * q, pack_f16x2(x[0], x[1]));
                    st_shared_b32(scr + cm16(g + 8, 0) + 4 * q, pack_f16x2(x[2], x[3]));
                    __syncwarp();
                    uint32_t bX[2], aT[4];
                    ldsm_x2_t(bX, scr + cm16((lane & 7) + 8 * ((lane >> 3) & 1), 0));
                    ldsm_x4(aT, Tt + cmT(16 * I + (lane & 15), 16 * I + 8 * (lane >> 4)));
                    float tt[4] = {0.f, 0.f, 0.f, 0.f};
                    mma16816(tt, aT, bX);
                    st_shared_b32(Tt + cmT(16 * I + g, N0) + 4 * q, pack_f16x2(-tt[0], -tt[1]));
                    st_shared_b32(Tt + cmT(16 * I + g + 8, N0) + 4 * q, pack_f16x2(-tt[2], -tt[3]));
                }
                named_sync(1, NT / 2);
            }
            fence_async_smem();
        } else {
            // ---- 3Y. warps 8-15: previous output; S^; Y (and O) = [beta K+ (; Q+)] S^; P; Y --
            if (OUT && prev_t0 >= 0 && q4 >= 2)
                store_o(tl, q4, 64 * hg, 2, lane, o, o_f32, b, T, H, h, prev_t0);
            {
                // master (scaled form) -> S^ = 2^{r + carry} master: fp16 operand tile and the
                // fp32 master both take the new scale
                const int col0 = hg * (NS / 2);
                for (int cc = 0; cc < NS / 2; cc += 32) {
                    float v[32];
                    tmem_ld32(tl + TM_S + col0 + cc, v);
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] *= s_scale;
#pragma unroll
                    for (int g8 = 0; g8 < 4; ++g8) {
                        const int col = col0 + cc + g8 * 8;
                        *reinterpret_cast<uint4*>(sm + PL::S + (col >> 3) * 2048 + (c >> 3) * 128 + (c & 7) * 16) =
                            pack8_f16(&v[8 * g8]);
                    }
                    tmem_st32(tl + TM_S + col0 + cc, v);
                }
            }
            fence_async_smem();
            tc_fence_before();
            if (OUT) {
                named_sync(2, NT / 2);
            } else {
                // Y's TMEM columns hold A until warps 0-7 have read it
                wait_bar(a_bar, a_phase, ctl, t == NT / 2, 2);
            }
            if (t == NT / 2) {
                tc_fence_after();
                // OUT:   [Y; O] = [beta K+; Q+] S^   (M = 128, N = 128)
                // STATE: Y = beta K+ [S^ | Phi^]     (M = 64,  N = 256)
                const uint32_t idy = idesc_f16(OUT ? 128 : 64, NS, true, true);
                for (int kk = 0; kk < 8; ++kk)
                    umma_f16(tmem + T_Y, sdesc(sbase + PL::KP + 256 * kk, 128, 2048),
                             sdesc(sbase + PL::S + 256 * kk, 128, 2048), idy, kk > 0);
                umma_commit(y_bar);
                // the next chunk's q, k, v, g land while the inverse runs (the staging
                // buffer was last read by this chunk's prologue)
                if (n + 1 < n1) issue_tma(n + 1);
            }
            y_in_flight = true;
            if (OUT) {
                wait_bar(ctl.mma_bar, ctl.mma_phase, ctl, t == NT / 2, 2);
                if (q4 >= 2) {
                    // P rows: lanes 64-127 of the M = 128 accumulator; P goes to the free 1 KB
                    // halves of the T region, so that [T; P] reads as one M = 128 operand
                    float v[32];
                    tmem_ld32(tl + T_AP + 32 * hg, v);
                    const int i = 32 * (q4 - 2) + lane;
#pragma unroll
                    for (int g8 = 0; g8 < 4; ++g8) {
                        float f[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const int col = 32 * hg + 8 * g8 + j;
                            f[j] = (col <= i) ? v[8 * g8 + j] : 0.f;
                        }
                        *reinterpret_cast<uint4*>(sm + PL::TF + 1024 + cmT(i, 32 * hg + 8 * g8)) = pack8_f16(f);
                    }
                }
            } else {
                ctl.mma_phase ^= 1;   // A's phase: complete, since warps 0-7 have read A
            }
            wait_bar(y_bar, y_phase, ctl, t == NT / 2, 2);
            y_in_flight = false;
            // Y -> fp16 position-major tile in the S^ region (S^ is no longer needed)
            if (OUT) {
                if (q4 < 2) {
                    const int j = 32 * q4 + lane;    // M = 128 layout: row j in lane j
                    for (int cc = 0; cc < 64; cc += 32) {
                        float v[32];
                        tmem_ld32(tl + T_Y + 64 * hg + cc, v);
#pragma unroll
                        for (int g8 = 0; g8 < 4; ++g8) {
                            const int cg = (64 * hg + cc) / 8 + g8;
                            *reinterpret_cast<uint4*>(sm + PL::S + (j >> 3) * YJ + cg * 128 + (j & 7) * 16) =
                                pack8_f16(&v[8 * g8]);
                        }
                    }
                }
            } else {
                const int j = 16 * q4 + lane;        // M = 64 layout: lanes 0-15 of each quarter
                for (int cc = 0; cc < 128; cc += 32) {
                    float v[32];
                    tmem_ld32(tl + T_Y + 128 * hg + cc, v);
                    if (lane < 16) {
#pragma unroll
                        for (int g8 = 0; g8 < 4; ++g8) {
                            const int cg = (128 * hg + cc) / 8 + g8;
                            *reinterpret_cast<uint4*>(sm + PL::S + (j >> 3) * YJ + cg * 128 + (j & 7) * 16) =
                                pack8_f16(&v[8 * g8]);
                        }
                    }
                }
            }
            fence_async_smem();
        }
        tc_fence_before();
        __syncthreads();
        if (*sAbort) break;
        // ---- 4. U = T (beta V) - T Y  (value columns; identity columns: -T Y) -------------
        if (t == 0) {
            tc_fence_after();
            const uint32_t idv = idesc_f16(64, 128, false, false);
            const uint32_t idy = idesc_f16(64, NS, false, true, true);
            if (OUT) {
                for (int kk = 0; kk < 4; ++kk)
                    umma_f16(tmem + T_UU, sdesc(sbase + TT + 2 * T_LBO * kk, T_LBO, 128),
                             sdesc(sbase + PL::VB + 4096 * kk, 2048, 128), idv, kk > 0);
                for (int kk = 0; kk < 4; ++kk)
                    umma_f16(tmem + T_UU, sdesc(sbase + TT + 2 * T_LBO * kk, T_LBO, 128),
                             sdesc(sbase + PL::S + 2 * YJ * kk, YJ, 128), idy, 1);
            } else {
                for (int kk = 0; kk < 4; ++kk)
                    umma_f16(tmem + T_UU, sdesc(sbase + TT + 2 * T_LBO * kk, T_LBO, 128),
                             sdesc(sbase + PL::S + 2 * YJ * kk, YJ, 128), idy, kk > 0);
                for (int kk = 0; kk < 4; ++kk)
                    umma_f16(tmem + T_UU, sdesc(sbase + TT + 2 * T_LBO * kk, T_LBO, 128),
                             sdesc(sbase + PL::VB + 4096 * kk, 2048, 128), idv, 1);
            }
            umma_commit(ctl.mma_bar);
        }
        wait_mma(ctl, t);
        // U -> fp16 MN-major tile [i][col] at U (M = 64 layout: row 16*q4 + l in lane 32*q4 + l)
        {
            for (int cc = 0; cc < NQ; cc += 32) {
                const int col = cq * NQ + cc;            // U tile column
                float v[32];
                tmem_ld32(tl + T_UU + col, v);
                if (lane < 16) {
                    const int i = 16 * q4 + lane;
#pragma unroll
                    for (int g8 = 0; g8 < 4; ++g8) {
                        const int cg = col / 8 + g8;
                        *reinterpret_cast<uint4*>(sm + PL::U + cg * 1024 + (i >> 3) * 128 + (i & 7) * 16) =
                            pack8_f16(&v[8 * g8]);
                    }
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        // ---- 5. master += K-^T U  (and O += P U) ------------------------------------------
        if (t == 0) {
            tc_fence_after();
            const uint32_t ids = idesc_f16(128, NS, false, true);
            for (int kk = 0; kk < 4; ++kk)
                umma_f16(tmem + TM_S, sdesc(sbase + PL::KM + 4096 * kk, 2048, 128),
                         sdesc(sbase + PL::U + 256 * kk, 128, 1024), ids, 1);
            if (OUT) {
                // O += P U as rows 64-127 of an M = 128 MMA whose rows 0-63 read T (their
                // result lands on Y's rows, already consumed)
                const uint32_t ido = idesc_f16(128, 128, false, true);
                for (int kk = 0; kk < 4; ++kk)
                    umma_f16(tmem + T_Y, sdesc(sbase + PL::TF + 4096 * kk, 2048, 128),
                             sdesc(sbase + PL::U + 256 * kk, 128, 1024), ido, 1);
            }
            umma_commit(ctl.mma_bar);
        }
        wait_mma(ctl, t);
        mma_in_flight = false;
        prev_t0 = t0;
    }
    if (OUT && !*sAbort && prev_t0 >= 0 && q4 >= 2)
        store_o(tl, q4, 32 * cq, 1, lane, o, o_f32, b, T, H, h, prev_t0);

    // ---- end of segment: write the state S = diag(2^{carry}) master ---------------------
    if (!*sAbort) {
        float* dst = nullptr;
        if (MODE == MODE_STATE) dst = maps + (size_t)(bh * (P - 1) + p) * 2 * D * D;  // [N | M]
        else if (S_T && p == P - 1) dst = S_T + (size_t)bh * D * D;
        if (dst) {
            const float sc = ex2_approx(carry);
            const int col0 = cq * NQ;
            for (int cc = 0; cc < NQ; cc += 32) {
                float v[32];
                tmem_ld32(tl + TM_S + col0 + cc, v);
                // maps: N block (value columns) then M block (identity columns); a 32-column
                // run never straddles the two
                const int col = col0 + cc;
                const size_t idx = (col < D) ? ((size_t)c * D + col) : ((size_t)D * D + (size_t)c * D + (col - D));
                float4* d4 = reinterpret_cast<float4*>(dst + idx);
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    d4[j] = make_float4(v[4 * j] * sc, v[4 * j + 1] * sc, v[4 * j + 2] * sc, v[4 * j + 3] * sc);
            }
        }
    }
    // ---- teardown: drain what is in flight, free TMEM ---------------------------------
    if (*sAbort) {
        if (mma_in_flight) mbar_wait_bounded(ctl.mma_bar, ctl.mma_phase, kWaitNs);
        if (tma_in_flight) mbar_wait_bounded(ctl.tma_bar, ctl.tma_phase, kWaitNs);
        if (y_in_flight && t == NT / 2) mbar_wait_bounded(y_bar, y_phase, kWaitNs);
    }
    tc_fence_before();
    __syncthreads();
    if (w == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// S_start(p+1) = M_p S_start(p) + N_p in fp32 on CUDA cores.  Grid (D/16, H, B), 256
// threads: thread t owns row t/2 and 8 of the CTA's 16 state columns.  M_{p+1} streams
// into the second shared buffer (cp.async) while step p computes from the first.
constexpr int CB_THREADS = 256;
constexpr int CB_LD = 132;      // row stride in floats (16-byte rows for cp.async)
constexpr int cb_smem_bytes() { return (2 * D * CB_LD + D * 16) * (int)sizeof(float); }

__device__ __forceinline__ void cb_stage(float* dst, const float* M, int t)
{
#pragma unroll
    for (int u = 0; u < D * D / 4 / CB_THREADS; ++u) {
        const int i = t + u * CB_THREADS, row = i >> 5, col = (i & 31) * 4;
        cp_async16(dst + row * CB_LD + col, M + (size_t)row * D + col);
    }
    cp_async_commit();
}

__global__ void __launch_bounds__(CB_THREADS)
kda_combine_kernel(const float* __restrict__ maps, const float* __restrict__ S0,
                   float* __restrict__ starts, int H, int P)
{
    extern __shared__ __align__(16) float csm[];
    float* sS = csm + 2 * D * CB_LD;     // [128][16]
    const int t = threadIdx.x, col0 = blockIdx.x * 16;
    const int bh = blockIdx.z * H + blockIdx.y;
    const int r = t >> 1, c8 = (t & 1) * 8;
    const float* mp = maps + (size_t)bh * (P - 1) * 2 * D * D;   // [P-1][N | M]
    if (P > 1) cb_stage(csm, mp + D * D, t);
    float s[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) s[j] = S0 ? S0[((size_t)bh * D + r) * D + col0 + c8 + j] : 0.f;
    for (int p = 0; p < P; ++p) {
        float* out = starts + ((size_t)bh * P + p) * D * D + (size_t)r * D + col0 + c8;
#pragma unroll
        for (int j = 0; j < 8; ++j) out[j] = s[j];
        if (p == P - 1) break;
        const float* Nm = mp + (size_t)p * 2 * D * D;
        float acc[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] = Nm[(size_t)r * D + col0 + c8 + j];
        __syncthreads();                         // sS and the other buffer are free
#pragma unroll
        for (int j = 0; j < 8; ++j) sS[r * 16 + c8 + j] = s[j];
        if (p + 1 < P - 1) cb_stage(csm + ((p + 1) & 1) * D * CB_LD, mp + (size_t)(p + 1) * 2 * D * D + D * D, t);
        if (p + 1 < P - 1) asm volatile("cp.async.wait_group 1;" ::: "memory");
        else cp_async_wait_all();
        __syncthreads();                         // M_p staged, sS written
        const float* sM = csm + (p & 1) * D * CB_LD;
#pragma unroll 4
        for (int k4 = 0; k4 < D / 4; ++k4) {
            const float4 m = *reinterpret_cast<const float4*>(sM + r * CB_LD + 4 * k4);
            const float mk[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int k = 4 * k4 + u;
                const float4 s0 = *reinterpret_cast<const float4*>(sS + k * 16 + c8);
                const float4 s1 = *reinterpret_cast<const float4*>(sS + k * 16 + c8 + 4);
                acc[0] = fmaf(mk[u], s0.x, acc[0]); acc[1] = fmaf(mk[u], s0.y, acc[1]);
                acc[2] = fmaf(mk[u], s0.z, acc[2]); acc[3] = fmaf(mk[u], s0.w, acc[3]);
                acc[4] = fmaf(mk[u], s1.x, acc[4]); acc[5] = fmaf(mk[u], s1.y, acc[5]);
                acc[6] = fmaf(mk[u], s1.z, acc[6]); acc[7] = fmaf(mk[u], s1.w, acc[7]);
            }
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
        e = cudaFuncSetAttribute(kda_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, cb_smem_bytes());
        if (e != cudaSuccess) return e;
        ProfileScope prof("kda_tc_combine", s);
        count_launch();
        kda_combine_kernel<<<dim3(D / 16, a.H, a.B), CB_THREADS, cb_smem_bytes(), s>>>(maps, a.S0, starts, a.H, sp.P);
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
