// Tensor-core (tcgen05 / TMEM) chunkwise KDA forward for Dk = Dv = 128, chunk 64.
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
//   state pass (MODE_STATE): run the recurrence on the augmented state [S | Phi]
//          starting from [0 | I] with the values of the segment: the result is [N | M]
//          (the identity columns carry no values).
//   combine: S_start(p+1) = M_p S_start(p) + N_p in fp32 (CUDA cores).
//   output pass (MODE_OUTPUT): run the recurrence from S_start(p) and write o (and S_T
//          from the last segment).
// A uniform batch runs in two waves (host side, below): segment 0's output pass beside
// the state pass of segments 1..P-2, then the combine and the output pass of segments
// 1..P-1.  The gated epilogue, packed samples and sequence shards use one state pass over
// segments 0..P-2 (or all P) and one output pass over every segment.
//
// Inside a CTA (one per (b, h, segment), 512 threads) two warp groups form a
// two-stage pipeline over the segment's chunks:
//   producer (warps 0-7): forms beta K+, Q+, K- (fp16 tiles) of chunk n+1, issues
//     A|P, reads A and P out of TMEM and inverts I + A.  Everything it does is
//     independent of the state.
//   consumer (warps 8-15): chunk n's state chain: S^ from the master, [Y; O] MMA,
//     beta V, U MMA, master += K-^T U and O += P U, output store.
// The per-chunk tiles are double-buffered; mbarriers hand a buffer over (full) and
// back (empty, committed by the consumer's last MMA that reads it).  Inputs arrive by
// TMA straight into the tiles that consume them and are converted in place: q and k
// of chunk n+2 land in the Q+ / beta K+ slots of their buffer set as soon as the
// consumer's [Y; O] MMA of chunk n has read them, v of chunk n+1 lands in the beta V
// tile once chunk n's U MMA has read it, and g of chunk n+1 in a staging tile once the
// producer has summed chunk n's.
//
// Shared-memory operand tiles use the no-swizzle core-matrix layout: 8 rows x 16 B
// blocks of 128 contiguous bytes.  A thread that owns one key channel writes 8
// consecutive chunk positions as one 16-byte store, so the channel-major tiles serve
// both as MN-major operands (chunk position = M/N) and K-major ones (position = K).
//
// All waits are bounded (kWaitNs).  On expiry the kernel records DEV_TIMEOUT in the
// device status word and stops waiting: both warp groups still run every barrier of
// their loop (so neither can hang on the other), results are undefined, and before
// TMEM is freed each MMA-issuing thread drains its own MMAs.

#include <mutex>
#include <type_traits>
#include <vector>

#include "internal.h"
#include "sm100.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int C = 64;         // chunk length
constexpr int D = 128;        // Dk = Dv
constexpr int NT = 512;       // threads per CTA
constexpr int NG = 256;       // threads per warp group
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s bound on every wait
constexpr float kLog2e = 1.4426950408889634f;
enum { MODE_STATE = 0, MODE_OUTPUT = 1 };

// ---- shared-memory plan (bytes) --------------------------------------------------
// Two buffer sets (one per chunk parity) of channel-major fp16 tiles: 8-position group
// ig at tile + ig*2048, channel c at (c >> 3)*128 + (c & 7)*16 inside it.  Q+ follows
// beta K+ directly, so [beta K+; Q+] is one M = 128 operand.  T (and P) sit in the
// set: 8-column groups of T are T_LBO apart; in MODE_OUTPUT P fills the other 1 KB
// halves, so [T; P] is one M = 128 operand.  The consumer's S^ region holds Y
// (position-major: 8-position group j at j*NS*16, 8 columns per 16 bytes) once the
// [Y; O] MMA has read S^.
template <int MODE> struct Plan;
template <> struct Plan<MODE_OUTPUT> {
    static constexpr int NS = 128;                 // state columns (values only)
    static constexpr int SET = 65536;              // buffer set stride
    static constexpr int KP = 0, QP = 16384, KM = 32768, TF = 49152;   // inside a set
    static constexpr int T_LBO = 2048;
    static constexpr int VB = 131072;              // beta V (consumer)
    static constexpr int AT = 147456;              // A, fp16 (producer)
    static constexpr int U = 155648;               // U (64 x 128)
    static constexpr int S = 172032;               // S^ (128 x 128 fp16), then Y
    static constexpr int GST = 204800;             // g staging ([64][128] bf16, TMA)
    static constexpr int MISC = 221184;
    static constexpr int QK_BYTES = 2 * 16384;     // q and k of one chunk
};
template <> struct Plan<MODE_STATE> {
    static constexpr int NS = 256;                 // [S | Phi]
    static constexpr int SET = 40960;
    static constexpr int KP = 0, QP = -1, KM = 16384, TF = 32768;
    static constexpr int T_LBO = 1024;
    static constexpr int VB = 81920;
    static constexpr int AT = 98304;
    static constexpr int U = 106496;               // U (64 x 256)
    static constexpr int S = 139264;               // [S^ | Phi^] (128 x 256 fp16), then Y
    static constexpr int GST = 204800;
    static constexpr int MISC = 221184;
    static constexpr int QK_BYTES = 16384;         // k of one chunk
};
// MISC sub-layout
constexpr int M_BETAP = 0;       // float[64]  beta of the producer's chunk
constexpr int M_BETAC = 256;     // float[64]  beta of the consumer's chunk
constexpr int M_TOT = 512;       // float[4][128] per-16-row sums of g log2(e)
constexpr int M_RB = 2560;       // float2[2][128] (r, b_C) per channel, per buffer set
constexpr int M_XS = 4608;       // 8 x 512 B per-warp 16x16 fp16 scratch of the inverse
constexpr int M_BAR = 8704;      // mbarriers, see Bar
constexpr int M_TMEM = 8856;     // uint32 TMEM base
constexpr int M_ABORT = 8860;    // int
constexpr int M_GAMMA = 8864;    // float[128] RMSNorm gain of this CTA's head (gated output)
constexpr int MISC_BYTES = 9376;
// PRO: a set's beta K+, Q+, K- tiles and r, b_C are ready; INV: its T (and P) too;
// EMPTY: the consumer's last MMA on the set is done.
enum Bar { B_PRO = 0, B_EMPTY = 2, B_AP = 4, B_Y = 5, B_U = 6, B_S = 7, B_AFREE = 8, B_UREAD = 9,
           B_DRAIN = 10, B_DRAIN2 = 11, B_TQK = 12, B_TG = 14, B_TV = 15, B_INV = 16, B_TGATE = 18,
           NBAR = 19 };

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
__device__ __forceinline__ uint4 pack8_f16(const float* f)
{
    uint4 u;
    __half2* h = reinterpret_cast<__half2*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
    return u;
}

// Two adjacent 2-byte input elements -> fp32
__device__ __forceinline__ float2 in2(uint32_t u, const __nv_bfloat16*)
{
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}
__device__ __forceinline__ float2 in2(uint32_t u, const __half*) { return unpack_f16x2(u); }

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

// Shared abort state.  A wait that runs out records DEV_TIMEOUT and raises the flag;
// once it is up, pollers stop waiting (barriers still run, so no group can hang).
struct Abort {
    int* flag;
    int* status;
};
// One thread polls; the group (bar_id, NG threads) waits at its named barrier.
__device__ __forceinline__ void group_wait(uint64_t* bar, uint32_t parity, const Abort& a, bool poller, int bar_id)
{
    if (poller && !*a.flag && !mbar_wait_bounded(bar, parity, kWaitNs)) {
        *a.flag = 1;
        atomicCAS(a.status, DEV_OK, DEV_TIMEOUT);
    }
    named_sync(bar_id, NG);
    tc_fence_after();
}
// One thread waits alone (before issuing MMAs that depend on the other group).
__device__ __forceinline__ void thread_wait(uint64_t* bar, uint32_t parity, const Abort& a)
{
    if (!*a.flag && !mbar_wait_bounded(bar, parity, kWaitNs)) {
        *a.flag = 1;
        atomicCAS(a.status, DEV_OK, DEV_TIMEOUT);
    }
}

// Output rows of one chunk, TMEM -> global memory.  O is rows 64-127 of the M = 128
// accumulator [Y; O] (output row i in lane 64 + i), so warps of lane quarters 2 and 3
// copy it into a row-major staging tile (rows padded by 16 bytes: the 8 rows of a
// 16-byte store phase hit 8 different bank groups); after the group barrier every warp
// of the group writes whole rows with coalesced 16-byte stores.
__device__ __forceinline__ void stage_o(uint32_t tl, int q4, int hg, int lane, uint8_t* stg, int o_f32)
{
    if (q4 < 2) return;
    const int i = 32 * (q4 - 2) + lane;
    const int es = o_f32 ? 4 : 2, ld = D * es + 16;
    for (int u = 0; u < 2; ++u) {
        float v[32];
        const int cc = 64 * hg + 32 * u;
        tmem_ld32(tl + Tm<MODE_OUTPUT>::Y + cc, v);
        uint8_t* row = stg + i * ld + cc * es;
        if (o_f32) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
                reinterpret_cast<float4*>(row)[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint4 uu;
                __nv_bfloat162* hh = reinterpret_cast<__nv_bfloat162*>(&uu);
#pragma unroll
                for (int e = 0; e < 4; ++e) hh[e] = __floats2bfloat162_rn(v[8 * j + 2 * e], v[8 * j + 2 * e + 1]);
                reinterpret_cast<uint4*>(row)[j] = uu;
            }
        }
    }
}
// bf16 output through TMA: O rows go into two 64-channel x 64-row tiles (128-byte
// rows, 128-byte swizzle: 16-byte chunk j of row i at i*128 + ((j ^ (i & 7)) * 16), so
// the 8 rows of a store phase hit 8 different bank groups); one thread then stores
// both tiles with the TMA (rows past the end of the sequence are clipped).
__device__ __forceinline__ void stage_o_swz(uint32_t tl, int q4, int hg, int lane, uint8_t* tiles)
{
    if (q4 < 2) return;
    const int i = 32 * (q4 - 2) + lane;
    uint8_t* tile = tiles + hg * 8192;
    for (int u = 0; u < 2; ++u) {
        float v[32];
        tmem_ld32(tl + Tm<MODE_OUTPUT>::Y + 64 * hg + 32 * u, v);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint4 uu;
            __nv_bfloat162* hh = reinterpret_cast<__nv_bfloat162*>(&uu);
#pragma unroll
            for (int e = 0; e < 4; ++e) hh[e] = __floats2bfloat162_rn(v[8 * j + 2 * e], v[8 * j + 2 * e + 1]);
            const int chunk = 4 * u + j;
            *reinterpret_cast<uint4*>(tile + i * 128 + ((chunk ^ (i & 7)) * 16)) = uu;
        }
    }
}
// Output side of Eq. 15 for a bf16 output: y = Sigmoid(gate) * gamma_h * RMSNorm(o) per
// output row, written into the same swizzled tiles as stage_o_swz.  The gate arrives by
// TMA as two swizzled 64-channel tiles (the layout of the output tiles).  A row's 128
// channels sit in two warps (column halves), so its sum of squares is exchanged through
// `red` between two group barriers; TMEM is read twice instead of holding 64 values.
__device__ __forceinline__ void stage_o_gated(uint32_t tl, int q4, int hg, int lane, uint8_t* tiles,
                                              const uint8_t* gtiles, float* red, const float* sGamma, float eps)
{
    const int i = 32 * (q4 - 2) + lane;
    if (q4 >= 2) {
        float ss = 0.f;
        for (int u = 0; u < 2; ++u) {
            float v[32];
            tmem_ld32(tl + Tm<MODE_OUTPUT>::Y + 64 * hg + 32 * u, v);
#pragma unroll
            for (int j = 0; j < 32; ++j) ss = fmaf(v[j], v[j], ss);
        }
        red[2 * i + hg] = ss;
    }
    named_sync(2, NG);
    if (q4 < 2) return;
    const float m = (red[2 * i] + red[2 * i + 1]) * (1.f / D) + eps;
    const float inv = m > 0.f ? rsqrtf(m) : 0.f;
    uint8_t* tile = tiles + hg * 8192;
    const uint8_t* gtile = gtiles + hg * 8192;
    for (int u = 0; u < 2; ++u) {
        float v[32];
        tmem_ld32(tl + Tm<MODE_OUTPUT>::Y + 64 * hg + 32 * u, v);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int chunk = 4 * u + j;
            const int off = i * 128 + ((chunk ^ (i & 7)) * 16);
            const uint4 gu = *reinterpret_cast<const uint4*>(gtile + off);
            const __nv_bfloat162* gb = reinterpret_cast<const __nv_bfloat162*>(&gu);
            const int c0 = 64 * hg + 8 * chunk;
            const float4 g0 = *reinterpret_cast<const float4*>(sGamma + c0);
            const float4 g1 = *reinterpret_cast<const float4*>(sGamma + c0 + 4);
            const float gm[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
            uint4 uu;
            __nv_bfloat162* hh = reinterpret_cast<__nv_bfloat162*>(&uu);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 gv = __bfloat1622float2(gb[e]);
                const float y0 = __fdividef(v[8 * j + 2 * e] * inv * gm[2 * e], 1.f + __expf(-gv.x));
                const float y1 = __fdividef(v[8 * j + 2 * e + 1] * inv * gm[2 * e + 1], 1.f + __expf(-gv.y));
                hh[e] = __floats2bfloat162_rn(y0, y1);
            }
            *reinterpret_cast<uint4*>(tile + off) = uu;
        }
    }
}

__device__ __forceinline__ void flush_o(const uint8_t* stg, int tg, void* o, int o_f32, int64_t rowbase, int T, int H,
                                        int h, int t0)
{
    const int es = o_f32 ? 4 : 2, ld = D * es + 16;
    const int per_row = D * es / 16;                 // 16-byte pieces per row
    for (int e = tg; e < C * per_row; e += NG) {
        const int i = e / per_row, pc = e % per_row;
        if (t0 + i < T) {
            const uint4 x = *reinterpret_cast<const uint4*>(stg + i * ld + pc * 16);
            uint8_t* dst = reinterpret_cast<uint8_t*>(o) + ((((size_t)rowbase + t0 + i) * H + h) * D) * es + pc * 16;
            *reinterpret_cast<uint4*>(dst) = x;
        }
    }
}

// 16 rows x 2 channels (one 4-byte word per row) of a [64][128] 2-byte tile in shared
// memory, as TMA lands it: a warp reads 128 contiguous bytes per row.
__device__ __forceinline__ void ld_rows16(uint32_t (&dst)[16], const uint8_t* tile, int r0, int cp)
{
#pragma unroll
    for (int r = 0; r < 16; ++r) dst[r] = *reinterpret_cast<const uint32_t*>(tile + (r0 + r) * 256 + 4 * cp);
}
// beta of token t0 + i of a sequence that starts at packed token `rowbase` and has T tokens
__device__ __forceinline__ uint32_t load_beta(const __nv_bfloat16* beta, int64_t rowbase, int T, int H, int h, int t0,
                                              int i, bool live)
{
    const int tt = t0 + i;
    return (live && tt < T) ? (uint32_t) * reinterpret_cast<const unsigned short*>(beta + ((size_t)rowbase + tt) * H + h)
                            : 0u;
}
// Store two channels' packed fp16 rows (one 16-byte vector per channel) into a
// channel-major tile.  Threads with (cp & 4) store their odd channel first: each
// 8-thread phase of a 16-byte store then covers all 32 banks once.
__device__ __forceinline__ void st_pair(uint8_t* tile, int ig, int cp, const uint32_t (&pp)[2][4])
{
    const bool sw = (cp & 4) != 0;
    const int c_first = 2 * cp + (sw ? 1 : 0), c_second = 2 * cp + (sw ? 0 : 1);
    const uint4 a0 = make_uint4(pp[0][0], pp[0][1], pp[0][2], pp[0][3]);
    const uint4 a1 = make_uint4(pp[1][0], pp[1][1], pp[1][2], pp[1][3]);
    *reinterpret_cast<uint4*>(tile + ig * 2048 + (c_first >> 3) * 128 + (c_first & 7) * 16) = sw ? a1 : a0;
    *reinterpret_cast<uint4*>(tile + ig * 2048 + (c_second >> 3) * 128 + (c_second & 7) * 16) = sw ? a0 : a1;
}

// The kernel ---------------------------------------------------------------------------
template <int MODE, typename TQ>
__global__ void __launch_bounds__(NT, 1)
kda_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
              const __grid_constant__ CUtensorMap tm_o, const __grid_constant__ CUtensorMap tm_gate,
              const __nv_bfloat16* __restrict__ beta, void* __restrict__ o, int o_f32,
              const float* __restrict__ S_in, int s_in_per_segment, float* __restrict__ maps,
              float* __restrict__ S_T, int B, int T, int H, int P, int L, int* status, int dbg_drop,
              const float* __restrict__ gamma, float eps, int gated, const int* __restrict__ items)
{
    using PL = Plan<MODE>;
    constexpr bool OUT = MODE == MODE_OUTPUT;
    constexpr int NS = PL::NS;
    constexpr int YJ = NS * 16;               // Y tile: bytes per 8-position group
    constexpr int T_LBO = PL::T_LBO;          // T's 8-column group stride
    constexpr uint32_t T_Y = Tm<MODE>::Y, T_UU = Tm<MODE>::UU;
    auto cmT = [](int i, int j) -> uint32_t { return (j >> 3) * T_LBO + (i >> 3) * 128 + (i & 7) * 16; };
    extern __shared__ __align__(1024) uint8_t sm[];

    const int t = threadIdx.x, w = t >> 5, lane = t & 31;
    const int q4 = w & 3;                     // TMEM lane quarter of this warp
    const int hg = (w >> 2) & 1;              // column half inside a warp group
    const int tg = t & (NG - 1);              // thread index inside its group
    const int cp = tg & 63, rq = tg >> 6;     // channel pair, 16-row quarter (loads, prologue)
    const int c = t & 127;                    // channel / TMEM row of the state steps
    // This CTA's work: chunks [n0, n1) of head h of one sequence that starts at packed
    // token `rowbase` and has `Tq` tokens.  Uniform batch: sequence b of B rows of T
    // tokens, segment p of P; packed samples: one entry of the host-built item table
    // {rowbase, Tq, n0, n1, h, sequence, slot, last}.  `slot` indexes the maps (state
    // pass) or the start states (output pass); `last` marks the sequence's final segment.
    int64_t rowbase;
    int Tq, n0, n1, h, seq, slot, last;
    if (items) {
        const int* it = items + 8 * blockIdx.x;
        rowbase = it[0]; Tq = it[1]; n0 = it[2]; n1 = it[3]; h = it[4]; seq = it[5]; slot = it[6]; last = it[7];
    } else {
        const int nseg = (MODE == MODE_STATE) ? P - 1 : P;
        const int bh = blockIdx.x / nseg, p = blockIdx.x % nseg;
        seq = bh / H;
        h = bh % H;
        rowbase = (int64_t)seq * T;
        Tq = T;
        const int NC = (T + C - 1) / C;
        n0 = p * L;
        n1 = min(NC, n0 + L);
        slot = (MODE == MODE_STATE) ? bh * (P - 1) + p : (s_in_per_segment ? bh * P + p : bh);
        last = p == P - 1;
    }
    const int nk = max(0, n1 - n0);
    // the bf16 output leaves by TMA store through a [B, T, H, 128] map that clips at the
    // end of a row; packed samples share one row, so a chunk that runs past its sample's
    // end is written with masked stores instead
    const int o_b = items ? 0 : seq;
    const int64_t o_t = items ? rowbase : 0;

    float* sBetaP = reinterpret_cast<float*>(sm + PL::MISC + M_BETAP);
    float* sBetaC = reinterpret_cast<float*>(sm + PL::MISC + M_BETAC);
    float* sTot = reinterpret_cast<float*>(sm + PL::MISC + M_TOT);
    float2* sRB = reinterpret_cast<float2*>(sm + PL::MISC + M_RB);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + PL::MISC + M_BAR);
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(sm + PL::MISC + M_TMEM);
    int* sAbort = reinterpret_cast<int*>(sm + PL::MISC + M_ABORT);
    const uint32_t sbase = smem_addr(sm);
    const Abort ab{sAbort, status};

    if (t == 0) {
        for (int i = 0; i < NBAR; ++i) mbar_init(&bars[i], 1);
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
    // TMA of chunk n's [64][128] tiles (packed rows rowbase + n*C ..; rows past the sequence
    // come from the next batch row or the zero fill and are masked where they are used)
    auto tma_qk = [&](int n) {   // q (MODE_OUTPUT) and k into the Q+ / beta K+ slots of set n&1
        const int bs = (n - n0) & 1, row = (int)(rowbase + n * C);
        mbar_arrive_expect_tx(&bars[B_TQK + bs], PL::QK_BYTES);
        if (OUT) tma_load_3d(sm + bs * PL::SET + PL::QP, &tm_q, &bars[B_TQK + bs], 0, h, row);
        tma_load_3d(sm + bs * PL::SET + PL::KP, &tm_k, &bars[B_TQK + bs], 0, h, row);
    };
    auto tma_g = [&](int n) {
        mbar_arrive_expect_tx(&bars[B_TG], 16384);
        tma_load_3d(sm + PL::GST, &tm_g, &bars[B_TG], 0, h, (int)(rowbase + n * C));
    };
    auto tma_v = [&](int n) {
        mbar_arrive_expect_tx(&bars[B_TV], 16384);
        tma_load_3d(sm + PL::VB, &tm_v, &bars[B_TV], 0, h, (int)(rowbase + n * C));
    };
    // gated bf16 output: chunk n's gate as two swizzled 64-channel tiles in the upper half
    // of the S^ region (free from the end of chunk n's [Y; O] MMA to chunk n+1's S^)
    auto tma_gate = [&](int n) {
        mbar_arrive_expect_tx(&bars[B_TGATE], 16384);
        tma_load_3d(sm + PL::S + 16384, &tm_gate, &bars[B_TGATE], 0, h, (int)(rowbase + n * C));
        tma_load_3d(sm + PL::S + 24576, &tm_gate, &bars[B_TGATE], 64, h, (int)(rowbase + n * C));
    };
    const bool gate_fused = OUT && gated && !o_f32;
    float* sGamma = reinterpret_cast<float*>(sm + PL::MISC + M_GAMMA);

    if (t < NG) {
        // ================= producer: state-independent work of chunk n0 + kc ==============
        const TQ* tq = nullptr;
        uint32_t betaR = 0;
        int g_issued = 0;   // thread 0: g tiles requested so far
        if (tg == 0 && nk > 0) {
            tma_g(n0);
            g_issued = 1;
        }
        if (tg < C) betaR = load_beta(beta, rowbase, Tq, H, h, n0 * C, tg, nk > 0);
        uint32_t gP[16];     // this chunk's g rows, kept from part 1 to part 2 of the prologue
        for (int kc = 0; kc < nk; ++kc) {
            const int n = n0 + kc, t0 = n * C, bs = kc & 1;
            uint8_t* set = sm + bs * PL::SET;
            const uint32_t sset = sbase + bs * PL::SET;
            // ---- prologue, part 1: g of this chunk (staging) -> cumulative log-decay ------
            // (needs only the g tile, so it runs before the wait for the buffer set)
            group_wait(&bars[B_TG], kc & 1, ab, tg == 0, 1);
            {
                uint32_t gR[16];
                ld_rows16(gR, sm + PL::GST, 16 * rq, cp);
                const bool full = t0 + C <= Tq;
                if (!full) {
#pragma unroll
                    for (int r = 0; r < 16; ++r)
                        if (t0 + 16 * rq + r >= Tq) gR[r] = 0u;
                }
                const float2 l2e = make_float2(kLog2e, kLog2e);
                float2 tot = make_float2(0.f, 0.f);
#pragma unroll
                for (int r = 0; r < 16; ++r) tot = __ffma2_rn(in2(gR[r], (const __nv_bfloat16*)nullptr), l2e, tot);
                *reinterpret_cast<float2*>(sTot + rq * D + 2 * cp) = tot;
                if (tg < C) sBetaP[tg] = __uint_as_float(betaR << 16);
#pragma unroll
                for (int r = 0; r < 16; ++r) gP[r] = gR[r];
            }
            named_sync(1, NG);   // the g tile is in registers: the next chunk's may land
            if (tg == 0 && n + 1 < n1 && !*sAbort) {
                tma_g(n + 1);
                g_issued = kc + 2;
            }
            if (tg < C) betaR = load_beta(beta, rowbase, Tq, H, h, (n + 1) * C, tg, n + 1 < n1);
            float2 r2, bC, run;
            {
                float2 tq4[4];
#pragma unroll
                for (int qb = 0; qb < 4; ++qb) tq4[qb] = *reinterpret_cast<const float2*>(sTot + qb * D + 2 * cp);
                r2 = __fadd2_rn(tq4[0], tq4[1]);                     // b at row 31
                bC = __fadd2_rn(r2, __fadd2_rn(tq4[2], tq4[3]));     // b at row 63
                run = make_float2(-r2.x, -r2.y);                     // running b - r
#pragma unroll
                for (int qb = 0; qb < 3; ++qb)
                    if (qb < rq) run = __fadd2_rn(run, tq4[qb]);
            }
            // ---- part 2: buffer set bs is free once the consumer is done with chunk kc - 2
            // (its K- and T tiles, and r, b_C); this chunk's q, k have landed in the set -----
            if (tg == 0 && kc >= 2) thread_wait(&bars[B_EMPTY + bs], ((kc >> 1) - 1) & 1, ab);
            group_wait(&bars[B_TQK + bs], (kc >> 1) & 1, ab, tg == 0, 1);
            {
                uint32_t kR[16], qR[16];
                const uint32_t (&gR)[16] = gP;
                ld_rows16(kR, set + PL::KP, 16 * rq, cp);
                if (OUT) ld_rows16(qR, set + PL::QP, 16 * rq, cp);
                if (t0 + C > Tq) {
#pragma unroll
                    for (int r = 0; r < 16; ++r)
                        if (t0 + 16 * rq + r >= Tq) kR[r] = qR[r] = 0u;
                }
                const float2 l2e = make_float2(kLog2e, kLog2e);
                if (rq == 0) {
                    sRB[bs * D + 2 * cp] = make_float2(r2.x, bC.x);
                    sRB[bs * D + 2 * cp + 1] = make_float2(r2.y, bC.y);
                }
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t pk[2][4], pm[2][4], pq[2][4];
                    float2 lk = make_float2(0.f, 0.f), lm = lk, lq = lk;
#pragma unroll
                    for (int r8 = 0; r8 < 8; ++r8) {
                        const int r = 8 * half + r8, i = 16 * rq + r;
                        run = __ffma2_rn(in2(gR[r], (const __nv_bfloat16*)nullptr), l2e, run);
                        const float2 kk = in2(kR[r], tq);
                        const float bi = sBetaP[i];
                        const float2 ep = make_float2(ex2_approx(run.x), ex2_approx(run.y));
                        const float2 em = make_float2(ex2_approx(-run.x), ex2_approx(-run.y));
                        const float2 kp = __fmul2_rn(__fmul2_rn(kk, make_float2(bi, bi)), ep);   // beta K+
                        const float2 km = __fmul2_rn(kk, em);                                   // K-
                        const float2 qp = OUT ? __fmul2_rn(in2(qR[r], tq), ep) : make_float2(0.f, 0.f);   // Q+
                        if (r8 & 1) {
                            const int m = r8 >> 1;
                            pk[0][m] = pack_f16x2(lk.x, kp.x); pk[1][m] = pack_f16x2(lk.y, kp.y);
                            pm[0][m] = pack_f16x2(lm.x, km.x); pm[1][m] = pack_f16x2(lm.y, km.y);
                            pq[0][m] = pack_f16x2(lq.x, qp.x); pq[1][m] = pack_f16x2(lq.y, qp.y);
                        } else {
                            lk = kp; lm = km; lq = qp;
                        }
                    }
                    const int ig = 2 * rq + half;
                    st_pair(set + PL::KP, ig, cp, pk);
                    st_pair(set + PL::KM, ig, cp, pm);
                    if (OUT) st_pair(set + PL::QP, ig, cp, pq);
                }
            }
            fence_async_smem();
            tc_fence_before();
            named_sync(1, NG);
            // tiles, r and b_C ready (the test hook withholds chunk 0's signal)
            if (tg == 0 && !(dbg_drop && kc == 0)) mbar_arrive(&bars[B_PRO + bs]);
            // ---- A (and P) on the tensor core -------------------------------------------
            if (tg == 0) {
                // MODE_STATE: A's TMEM columns are the consumer's U until it has read U
                if (MODE == MODE_STATE && kc >= 1) thread_wait(&bars[B_UREAD], (kc - 1) & 1, ab);
                tc_fence_after();
                // [beta K+; Q+] (M = 128) x K-^T: rows 0-63 give A, rows 64-127 give P
                const uint32_t id = idesc_f16(OUT ? 128 : 64, 64, true, true);
                for (int kk = 0; kk < 8; ++kk)
                    umma_f16(tmem + T_AP, sdesc(sset + PL::KP + 256 * kk, 128, 2048),
                             sdesc(sset + PL::KM + 256 * kk, 128, 2048), id, kk > 0);
                umma_commit(&bars[B_AP]);
            }
            group_wait(&bars[B_AP], kc & 1, ab, tg == 0, 1);
            // ---- A -> fp16 tile (and P -> the T region's other halves) ------------------
            const uint32_t Ah = sbase + PL::AT;          // A, fp16 K-major core-matrix tile
            const uint32_t Tt = sset + PL::TF;           // T: the consumer's operand
            {
                float v[32];
                tmem_ld32(tl + T_AP + 32 * hg, v);
                int i = -1;
                bool isP = false;
                if (OUT) {
                    // M = 128 layout: row i in lane i; rows 0-63 are A, rows 64-127 are P
                    i = 32 * (q4 & 1) + lane;
                    isP = q4 >= 2;
                } else if (lane < 16) {
                    i = 16 * q4 + lane;                  // M = 64 layout
                }
                if (i >= 0) {
#pragma unroll
                    for (int g8 = 0; g8 < 4; ++g8) {
                        float f[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const int col = 32 * hg + 8 * g8 + j;
                            f[j] = (isP ? (col <= i) : (col < i)) ? v[8 * g8 + j] : 0.f;
                        }
                        uint8_t* dst = isP ? set + PL::TF + 1024 + cmT(i, 32 * hg + 8 * g8)
                                           : sm + PL::AT + cm64(i, 32 * hg + 8 * g8);
                        *reinterpret_cast<uint4*>(dst) = pack8_f16(f);
                    }
                }
                // the six upper 16x16 blocks of T are zero
                if (tg < 192) {
                    const int e = tg >> 5, u = tg & 31;
                    const int I = (e < 3) ? 0 : (e < 5 ? 1 : 2);
                    const int J = (e < 3) ? e + 1 : (e < 5 ? e - 1 : 3);
                    const int row = 16 * I + 8 * (u >> 4) + (u & 7), col = 16 * J + 8 * ((u >> 3) & 1);
                    *reinterpret_cast<uint4*>(set + PL::TF + cmT(row, col)) = make_uint4(0u, 0u, 0u, 0u);
                }
            }
            tc_fence_before();
            named_sync(1, NG);
            if (MODE == MODE_STATE && tg == 0) mbar_arrive(&bars[B_AFREE]);   // Y may overwrite A
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
            // off-diagonal blocks by halves of the matrix (each warp: one 8-column half of one
            // 16x16 block; X products through per-warp fp16 scratch):
            //   level 1: T_10 = -T_11 (A_10 T_00),  T_32 = -T_33 (A_32 T_22)
            //   level 2: X_IJ = sum_{K=J}^{1} A_IK T_KJ  (I = 2, 3; J = 0, 1), then
            //            T_IJ = -sum_{K=2}^{I} T_IK X_KJ
            {
                const int g = lane >> 2, q = lane & 3, half = w & 1;
                const uint32_t scr = sbase + PL::MISC + M_XS + 512 * w;
                auto scr_of = [&](int wx) { return sbase + PL::MISC + M_XS + 512 * wx; };
                auto put_x = [&](uint32_t dst, const float (&x)[4]) {
                    st_shared_b32(dst + cm16(g, 0) + 4 * q, pack_f16x2(x[0], x[1]));
                    st_shared_b32(dst + cm16(g + 8, 0) + 4 * q, pack_f16x2(x[2], x[3]));
                };
                auto put_t = [&](int I, int N0, const float (&tt)[4]) {
                    st_shared_b32(Tt + cmT(16 * I + g, N0) + 4 * q, pack_f16x2(-tt[0], -tt[1]));
                    st_shared_b32(Tt + cmT(16 * I + g + 8, N0) + 4 * q, pack_f16x2(-tt[2], -tt[3]));
                };
                auto a_frag = [&](uint32_t (&fr)[4], uint32_t base, int I, int K, bool isT) {
                    if (isT) ldsm_x4(fr, base + cmT(16 * I + (lane & 15), 16 * K + 8 * (lane >> 4)));
                    else ldsm_x4(fr, base + cm64(16 * I + (lane & 15), 16 * K + 8 * (lane >> 4)));
                };
                if (w < 4) {   // level 1
                    const int I = (w >> 1) ? 3 : 1, J = I - 1, N0 = 16 * J + 8 * half;
                    uint32_t aA[4], bT[2], bX[2], aT[4];
                    float x[4] = {0.f, 0.f, 0.f, 0.f}, tt[4] = {0.f, 0.f, 0.f, 0.f};
                    a_frag(aA, Ah, I, J, false);
                    ldsm_x2_t(bT, Tt + cmT(16 * J + (lane & 7) + 8 * ((lane >> 3) & 1), N0));
                    mma16816(x, aA, bT);
                    put_x(scr, x);
                    __syncwarp();
                    ldsm_x2_t(bX, scr + cm16((lane & 7) + 8 * ((lane >> 3) & 1), 0));
                    a_frag(aT, Tt, I, I, true);
                    mma16816(tt, aT, bX);
                    put_t(I, N0, tt);
                }
                named_sync(1, NG);
                // level 2, X: warp w -> block (I, J) = (2 + (w >> 2), (w >> 1) & 1), half w & 1
                const int I2 = 2 + (w >> 2), J2 = (w >> 1) & 1, N2 = 16 * J2 + 8 * half;
                {
                    float x[4] = {0.f, 0.f, 0.f, 0.f};
                    for (int K = J2; K < 2; ++K) {
                        uint32_t aA[4], bT[2];
                        a_frag(aA, Ah, I2, K, false);
                        ldsm_x2_t(bT, Tt + cmT(16 * K + (lane & 7) + 8 * ((lane >> 3) & 1), N2));
                        mma16816(x, aA, bT);
                    }
                    put_x(scr, x);
                }
                named_sync(1, NG);
                // level 2, T: the same (I, J, half); X_KJ half was written by warp 4(K-2) + 2J + half
                {
                    float tt[4] = {0.f, 0.f, 0.f, 0.f};
                    for (int K = 2; K <= I2; ++K) {
                        uint32_t aT[4], bX[2];
                        a_frag(aT, Tt, I2, K, true);
                        ldsm_x2_t(bX, scr_of(4 * (K - 2) + 2 * J2 + half) + cm16((lane & 7) + 8 * ((lane >> 3) & 1), 0));
                        mma16816(tt, aT, bX);
                    }
                    put_t(I2, N2, tt);
                }
            }
            fence_async_smem();
            named_sync(1, NG);
            if (tg == 0) mbar_arrive(&bars[B_INV + bs]);    // T (and P) ready
        }
        // after a timeout some requested g tile may not have been waited for: let it land
        if (tg == 0 && *sAbort && g_issued > 0) mbar_wait_bounded(&bars[B_TG], (g_issued - 1) & 1, kWaitNs);
    } else {
        // ================= consumer: the state chain of chunk n0 + kc =====================
        const TQ* tq = nullptr;
        // initial state in TMEM: warp (q4, hg) holds lanes 32*q4.. and columns hg*NS/2 ..
        {
            const int col0 = hg * (NS / 2);
            for (int cc = 0; cc < NS / 2; cc += 32) {
                float vv[32];
                if (MODE == MODE_STATE) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) vv[j] = (col0 + cc + j == D + c) ? 1.f : 0.f;
                } else if (S_in) {
                    const size_t idx = s_in_per_segment ? (size_t)slot : (size_t)seq * H + h;
                    const float4* s4 = reinterpret_cast<const float4*>(S_in + (idx * D + c) * D + col0 + cc);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float4 x = s4[j];
                        vv[4 * j] = x.x; vv[4 * j + 1] = x.y; vv[4 * j + 2] = x.z; vv[4 * j + 3] = x.w;
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) vv[j] = 0.f;
                }
                tmem_st32(tl + TM_S + col0 + cc, vv);
            }
        }
        if (gate_fused && tg < D) sGamma[tg] = gamma ? gamma[(size_t)h * D + tg] : 1.f;   // read after later barriers
        uint32_t betaR = 0;
        // thread NG + 32 (not the MMA issuer) requests the consumer-side TMA loads, just
        // before a barrier at which the group waits for an MMA anyway
        const bool loader = tg == 32;
        int v_issued = 0, qk_last[2] = {-1, -1}, gate_issued = 0;   // its TMA requests so far
        bool o_pending = false;                    // poller: a bf16 output store is in flight
        if (loader && nk > 0) {
            tma_v(n0);
            v_issued = 1;
            tma_qk(n0);
            qk_last[0] = 0;
            if (nk > 1) {
                tma_qk(n0 + 1);
                qk_last[1] = 1;
            }
        }
        if (tg < C) betaR = load_beta(beta, rowbase, Tq, H, h, n0 * C, tg, nk > 0);
        // the master holds diag(2^{-carry}) S for channel c (log2 units; 0 before any chunk)
        float carry = 0.f;
        const bool poller = tg == 0;
        for (int kc = 0; kc < nk; ++kc) {
            const int n = n0 + kc, t0 = n * C, bs = kc & 1;
            const uint32_t sset = sbase + bs * PL::SET;
            group_wait(&bars[B_PRO + bs], (kc >> 1) & 1, ab, poller, 2);
            // ---- S^ = 2^{r + carry} master ------------------------------------------------
            {
                const float2 rb = sRB[bs * D + c];
                const float s_scale = ex2_approx(rb.x + carry);
                carry = rb.y - rb.x;
                const int col0 = hg * (NS / 2);
                for (int cc = 0; cc < NS / 2; cc += 32) {
                    float vv[32];
                    tmem_ld32(tl + TM_S + col0 + cc, vv);
#pragma unroll
                    for (int j = 0; j < 32; ++j) vv[j] *= s_scale;
#pragma unroll
                    for (int g8 = 0; g8 < 4; ++g8) {
                        const int col = col0 + cc + g8 * 8;
                        *reinterpret_cast<uint4*>(sm + PL::S + (col >> 3) * 2048 + (c >> 3) * 128 + (c & 7) * 16) =
                            pack8_f16(&vv[8 * g8]);
                    }
                    tmem_st32(tl + TM_S + col0 + cc, vv);
                }
            }
            if (tg < C) sBetaC[tg] = __uint_as_float(betaR << 16);
            fence_async_smem();
            tc_fence_before();
            named_sync(2, NG);
            if (poller) {
                // MODE_STATE: Y's TMEM columns hold A until the producer has read it
                if (MODE == MODE_STATE) thread_wait(&bars[B_AFREE], kc & 1, ab);
                tc_fence_after();
                // OUT:   [Y; O] = [beta K+; Q+] S^   (M = 128, N = 128)
                // STATE: Y = beta K+ [S^ | Phi^]     (M = 64,  N = 256)
                const uint32_t idy = idesc_f16(OUT ? 128 : 64, NS, true, true);
                for (int kk = 0; kk < 8; ++kk)
                    umma_f16(tmem + T_Y, sdesc(sset + PL::KP + 256 * kk, 128, 2048),
                             sdesc(sbase + PL::S + 256 * kk, 128, 2048), idy, kk > 0);
                umma_commit(&bars[B_Y]);
            }
            // ---- beta V while Y runs: v (landed in the beta V tile) converted in place ---------
            group_wait(&bars[B_TV], kc & 1, ab, poller, 2);
            {
                uint32_t vR[16];
                ld_rows16(vR, sm + PL::VB, 16 * rq, cp);
                if (t0 + C > Tq) {
#pragma unroll
                    for (int r = 0; r < 16; ++r)
                        if (t0 + 16 * rq + r >= Tq) vR[r] = 0u;
                }
                named_sync(2, NG);
                uint32_t pv[2][4];
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float2 lv = make_float2(0.f, 0.f);
#pragma unroll
                    for (int r8 = 0; r8 < 8; ++r8) {
                        const int r = 8 * half + r8;
                        const float bi = sBetaC[16 * rq + r];
                        const float2 vb = __fmul2_rn(in2(vR[r], tq), make_float2(bi, bi));
                        if (r8 & 1) {
                            pv[0][r8 >> 1] = pack_f16x2(lv.x, vb.x);
                            pv[1][r8 >> 1] = pack_f16x2(lv.y, vb.y);
                        } else {
                            lv = vb;
                        }
                    }
                    st_pair(sm + PL::VB, 2 * rq + half, cp, pv);
                }
            }
            if (tg < C) betaR = load_beta(beta, rowbase, Tq, H, h, (n + 1) * C, tg, n + 1 < n1);
            if (OUT) {
                // U = T (beta V) - T Y: the first half needs no Y, so it queues behind [Y; O]
                fence_async_smem();
                named_sync(2, NG);
                if (poller) {
                    thread_wait(&bars[B_INV + bs], (kc >> 1) & 1, ab);   // T of this chunk
                    tc_fence_after();
                    const uint32_t idv = idesc_f16(64, 128, false, false);
                    const uint32_t Tb = sset + PL::TF;
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16(tmem + T_UU, sdesc(Tb + 2 * T_LBO * kk, T_LBO, 128),
                                 sdesc(sbase + PL::VB + 4096 * kk, 2048, 128), idv, kk > 0);
                }
            }
            group_wait(&bars[B_Y], kc & 1, ab, poller, 2);
            // ---- Y -> fp16 position-major tile in the S^ region --------------------------
            if (OUT) {
                if (q4 < 2) {
                    const int j = 32 * q4 + lane;    // M = 128 layout: row j in lane j
                    for (int cc = 0; cc < 64; cc += 32) {
                        float vv[32];
                        tmem_ld32(tl + T_Y + 64 * hg + cc, vv);
#pragma unroll
                        for (int g8 = 0; g8 < 4; ++g8) {
                            const int cg = (64 * hg + cc) / 8 + g8;
                            *reinterpret_cast<uint4*>(sm + PL::S + (j >> 3) * YJ + cg * 128 + (j & 7) * 16) =
                                pack8_f16(&vv[8 * g8]);
                        }
                    }
                }
            } else {
                const int j = 16 * q4 + lane;        // M = 64 layout: lanes 0-15 of each quarter
                for (int cc = 0; cc < 128; cc += 32) {
                    float vv[32];
                    tmem_ld32(tl + T_Y + 128 * hg + cc, vv);
                    if (lane < 16) {
#pragma unroll
                        for (int g8 = 0; g8 < 4; ++g8) {
                            const int cg = (128 * hg + cc) / 8 + g8;
                            *reinterpret_cast<uint4*>(sm + PL::S + (j >> 3) * YJ + cg * 128 + (j & 7) * 16) =
                                pack8_f16(&vv[8 * g8]);
                        }
                    }
                }
            }
            fence_async_smem();
            tc_fence_before();
            named_sync(2, NG);
            // ---- U = T (beta V) - T Y  (value columns; identity columns: -T Y) -------------
            if (poller) {
                if (!OUT) thread_wait(&bars[B_INV + bs], (kc >> 1) & 1, ab);   // T of this chunk
                tc_fence_after();
                const uint32_t idv = idesc_f16(64, 128, false, false);
                const uint32_t idy = idesc_f16(64, NS, false, true, true);
                const uint32_t Tb = sset + PL::TF;
                if (OUT) {
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16(tmem + T_UU, sdesc(Tb + 2 * T_LBO * kk, T_LBO, 128),
                                 sdesc(sbase + PL::S + 2 * YJ * kk, YJ, 128), idy, 1);
                } else {
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16(tmem + T_UU, sdesc(Tb + 2 * T_LBO * kk, T_LBO, 128),
                                 sdesc(sbase + PL::S + 2 * YJ * kk, YJ, 128), idy, kk > 0);
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16(tmem + T_UU, sdesc(Tb + 2 * T_LBO * kk, T_LBO, 128),
                                 sdesc(sbase + PL::VB + 4096 * kk, 2048, 128), idv, 1);
                }
                umma_commit(&bars[B_U]);
            }
            // [Y; O] of this chunk is done: chunk n+2's q, k may land in this set's
            // Q+ / beta K+ slots (and this chunk's gate in the upper half of S^)
            if (loader && n + 2 < n1 && !*sAbort) {
                tma_qk(n + 2);
                qk_last[bs] = kc + 2;
            }
            if (gate_fused && loader && !*sAbort) {
                tma_gate(n);
                gate_issued = kc + 1;
            }
            // the output store must have read the U region before U is written there
            if (poller && o_pending) {
                bulk_wait_read0();
                o_pending = false;
            }
            group_wait(&bars[B_U], kc & 1, ab, poller, 2);
            // U -> fp16 MN-major tile [i][col] at U (M = 64 layout: row 16*q4 + l in lane 32*q4 + l)
            for (int cc = 0; cc < NS / 2; cc += 32) {
                const int col = hg * (NS / 2) + cc;
                float vv[32];
                tmem_ld32(tl + T_UU + col, vv);
                if (lane < 16) {
                    const int i = 16 * q4 + lane;
#pragma unroll
                    for (int g8 = 0; g8 < 4; ++g8) {
                        const int cg = col / 8 + g8;
                        *reinterpret_cast<uint4*>(sm + PL::U + cg * 1024 + (i >> 3) * 128 + (i & 7) * 16) =
                            pack8_f16(&vv[8 * g8]);
                    }
                }
            }
            fence_async_smem();
            tc_fence_before();
            named_sync(2, NG);
            // ---- master += K-^T U  (and O += P U) ------------------------------------------
            if (poller) {
                if (MODE == MODE_STATE) mbar_arrive(&bars[B_UREAD]);   // A may take U's columns
                tc_fence_after();
                const uint32_t ids = idesc_f16(128, NS, false, true);
                for (int kk = 0; kk < 4; ++kk)
                    umma_f16(tmem + TM_S, sdesc(sset + PL::KM + 4096 * kk, 2048, 128),
                             sdesc(sbase + PL::U + 256 * kk, 128, 1024), ids, 1);
                if (OUT) {
                    // O += P U as rows 64-127 of an M = 128 MMA whose rows 0-63 read T (their
                    // result lands on Y's rows, already consumed)
                    const uint32_t ido = idesc_f16(128, 128, false, true);
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16(tmem + T_Y, sdesc(sset + PL::TF + 4096 * kk, 2048, 128),
                                 sdesc(sbase + PL::U + 256 * kk, 128, 1024), ido, 1);
                }
                umma_commit(&bars[B_S]);
                umma_commit(&bars[B_EMPTY + bs]);   // buffer set bs may be refilled
            }
            // the U MMA has read beta V: chunk n+1's v may land in its tile
            if (loader && n + 1 < n1 && !*sAbort) {
                tma_v(n + 1);
                v_issued = kc + 2;
            }
            group_wait(&bars[B_S], kc & 1, ab, poller, 2);
            // ---- this chunk's output, staged in the free U (and Y) regions; done here, at
            // the end of the chunk, it overlaps the wait for the producer's next tiles -----
            if (OUT) {
                if (o_f32 || (items && t0 + C > Tq)) {
                    stage_o(tl, q4, hg, lane, sm + PL::U, o_f32);
                    named_sync(2, NG);
                    flush_o(sm + PL::U, tg, o, o_f32, rowbase, Tq, H, h, t0);
                    named_sync(2, NG);
                } else {
                    if (gate_fused) {
                        group_wait(&bars[B_TGATE], kc & 1, ab, poller, 2);
                        stage_o_gated(tl, q4, hg, lane, sm + PL::U, sm + PL::S + 16384,
                                      reinterpret_cast<float*>(sm + PL::S), sGamma, eps);
                    } else {
                        stage_o_swz(tl, q4, hg, lane, sm + PL::U);
                    }
                    fence_async_smem();
                    named_sync(2, NG);
                    if (poller) {
                        tma_store_4d(&tm_o, sm + PL::U, 0, h, (int)(o_t + t0), o_b);
                        tma_store_4d(&tm_o, sm + PL::U + 8192, 64, h, (int)(o_t + t0), o_b);
                        bulk_commit();
                        o_pending = true;
                    }
                }
            }
        }
        if (poller) bulk_wait0();   // every output store has landed before the CTA exits
        // after a timeout some requested tiles may not have been waited for: let them land
        if (loader && *sAbort) {
            if (gate_issued > 0) mbar_wait_bounded(&bars[B_TGATE], (gate_issued - 1) & 1, kWaitNs);
            if (v_issued > 0) mbar_wait_bounded(&bars[B_TV], (v_issued - 1) & 1, kWaitNs);
            for (int s2 = 0; s2 < 2; ++s2)
                if (qk_last[s2] >= 0) mbar_wait_bounded(&bars[B_TQK + s2], (qk_last[s2] >> 1) & 1, kWaitNs);
        }
        // ---- end of segment: write the state S = diag(2^{carry}) master -----------------
        float* dst = nullptr;
        if (MODE == MODE_STATE) dst = maps + (size_t)slot * 2 * D * D;  // [N | M]
        else if (S_T && last) dst = S_T + ((size_t)seq * H + h) * D * D;
        if (dst && !*sAbort) {
            const float sc = ex2_approx(carry);
            const int col0 = hg * (NS / 2);
            for (int cc = 0; cc < NS / 2; cc += 32) {
                float vv[32];
                tmem_ld32(tl + TM_S + col0 + cc, vv);
                // maps: N block (value columns) then M block (identity columns); a 32-column
                // run never straddles the two
                const int col = col0 + cc;
                const size_t idx = (col < D) ? ((size_t)c * D + col) : ((size_t)D * D + (size_t)c * D + (col - D));
                float4* d4 = reinterpret_cast<float4*>(dst + idx);
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    d4[j] = make_float4(vv[4 * j] * sc, vv[4 * j + 1] * sc, vv[4 * j + 2] * sc, vv[4 * j + 3] * sc);
            }
        }
    }
    // ---- teardown: after a timeout, each MMA issuer drains its own MMAs; free TMEM --------
    if (*sAbort && (t == 0 || t == NG)) {
        uint64_t* dr = &bars[t == 0 ? B_DRAIN : B_DRAIN2];
        umma_commit(dr);
        mbar_wait_bounded(dr, 0, kWaitNs);
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

// Uniform batch (seqinfo == nullptr): sequence z = blockIdx.z has P segments, its maps at
// (z*H + h)*(P-1) and start states at (z*H + h)*P.  Packed samples: seqinfo[3z..3z+2] =
// {P_z, map base, start base}, head h's maps at map base + h*(P_z-1) and starts at start
// base + h*P_z (P_z = 0: empty sample, nothing to do).
__global__ void __launch_bounds__(CB_THREADS)
kda_combine_kernel(const float* __restrict__ maps, const float* __restrict__ S0,
                   float* __restrict__ starts, int H, int P, const int* __restrict__ seqinfo)
{
    extern __shared__ __align__(16) float csm[];
    float* sS = csm + 2 * D * CB_LD;     // [128][16]
    const int t = threadIdx.x, col0 = blockIdx.x * 16;
    const int bh = blockIdx.z * H + blockIdx.y;
    const int r = t >> 1, c8 = (t & 1) * 8;
    size_t map0 = (size_t)bh * (P - 1), start0 = (size_t)bh * P;
    if (seqinfo) {
        P = seqinfo[3 * blockIdx.z];
        map0 = (size_t)seqinfo[3 * blockIdx.z + 1] + (size_t)blockIdx.y * (P > 0 ? P - 1 : 0);
        start0 = (size_t)seqinfo[3 * blockIdx.z + 2] + (size_t)blockIdx.y * P;
        if (P == 0) return;
    }
    const float* mp = maps + map0 * 2 * D * D;   // [P-1][N | M]
    if (P > 1) cb_stage(csm, mp + D * D, t);
    float s[8], nxt[8];   // nxt: this thread's 8 values of N_p, loaded one step ahead
#pragma unroll
    for (int j = 0; j < 8; ++j) s[j] = S0 ? S0[((size_t)bh * D + r) * D + col0 + c8 + j] : 0.f;
    auto load_n = [&](int p) {
        const float4* n4 = reinterpret_cast<const float4*>(mp + (size_t)p * 2 * D * D + (size_t)r * D + col0 + c8);
        const float4 a = n4[0], b = n4[1];
        nxt[0] = a.x; nxt[1] = a.y; nxt[2] = a.z; nxt[3] = a.w; nxt[4] = b.x; nxt[5] = b.y; nxt[6] = b.z; nxt[7] = b.w;
    };
    if (P > 1) load_n(0);
    for (int p = 0; p < P; ++p) {
        float4* out = reinterpret_cast<float4*>(starts + (start0 + p) * D * D + (size_t)r * D + col0 + c8);
        out[0] = make_float4(s[0], s[1], s[2], s[3]);
        out[1] = make_float4(s[4], s[5], s[6], s[7]);
        if (p == P - 1) break;
        float acc[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] = nxt[j];
        if (p + 1 < P - 1) load_n(p + 1);        // in flight during this step
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

// The work items of the two-wave split of a uniform batch, built on the device (so a call
// makes no host-to-device copy and can be captured in a CUDA graph).  One thread per
// (b, h, segment p): p = 0 -> it0 (segment 0's output pass; slot = b*H + h, last = 1);
// p >= 1 -> ito (output pass, slot (b*H + h)*(P-1) + p-1) and, for p <= P-2, its (state
// pass, slot (b*H + h)*(P-2) + p-1).  Items are {row, length, n0, n1, head, sequence,
// slot, last}.
__global__ void wave_items_kernel(int* __restrict__ it0, int* __restrict__ its, int* __restrict__ ito, int B, int T,
                                  int H, int P, int L)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= B * H * P) return;
    const int p = i % P, bh = i / P, b = bh / H, h = bh % H;
    const int NC = (T + C - 1) / C, n0 = p * L, n1 = min(NC, n0 + L);
    auto put = [&](int* dst, int slot, int last) {
        dst[0] = b * T; dst[1] = T; dst[2] = n0; dst[3] = n1;
        dst[4] = h; dst[5] = b; dst[6] = slot; dst[7] = last;
    };
    if (p == 0) {
        put(it0 + 8 * bh, bh, 1);
        return;
    }
    put(ito + 8 * (bh * (P - 1) + p - 1), bh * (P - 1) + p - 1, p == P - 1);
    if (p <= P - 2) put(its + 8 * (bh * (P - 2) + p - 1), bh * (P - 2) + p - 1, 0);
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

// bf16 output o [B, T, H, 128] as a 4-D tensor (channels, heads, tokens, batch), box =
// 64 channels x 1 head x 64 tokens, 128-byte swizzle.  Tokens past T are clipped by the
// T dimension, so a ragged last chunk never writes into the next batch row.
bool make_map_o(CUtensorMap* m, void* base, int B, int T, int H)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)T * H * D * 2};
    const cuuint32_t box[4] = {64u, 1u, (cuuint32_t)C, 1u};
    const cuuint32_t es[4] = {1u, 1u, 1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Gate [B*T, H, 128] bf16 as two 64-channel halves per chunk (box 64 x 1 x 64), 128-byte
// swizzle: lands in the layout of the swizzled output tiles.
bool make_map_gate(CUtensorMap* m, const void* base, int B, int T, int H)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)B * (cuuint64_t)T};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
    const cuuint32_t box[3] = {64u, 1u, (cuuint32_t)C};
    const cuuint32_t es[3] = {1u, 1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct Maps {
    CUtensorMap q, k, v, g, o;   // o: only for a bf16 output (else a copy of q, unused)
    CUtensorMap gate;            // only for the fused gated epilogue (else a copy of q)
};

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
cudaError_t launch_pass(const Maps& mp, const KdaArgs& a, const float* S_in, int per_seg, float* maps, int P, int L,
                        int* status, cudaStream_t s, const int* items = nullptr, int nitems = 0,
                        const char* prof_name = nullptr)
{
    auto kern = kda_tc_kernel<MODE, TQ>;
    const int smem = smem_bytes<MODE>();
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int nseg = MODE == MODE_STATE ? P - 1 : P;
    const unsigned grid = items ? (unsigned)nitems : (unsigned)(a.B * a.H * nseg);
    if (grid == 0) return cudaSuccess;
    ProfileScope prof(prof_name ? prof_name : (MODE == MODE_STATE ? "kda_tc_state" : "kda_tc_output"), s);
    count_launch();
    kern<<<grid, NT, smem, s>>>(mp.q, mp.k, mp.v, mp.g, mp.o, mp.gate, (const __nv_bfloat16*)a.beta, a.o, a.out_t == ET_F32 ? 1 : 0,
                                S_in, per_seg, maps, a.ST, a.B, a.T, a.H, P, L, status, debug_drop_handoff(),
                                a.gamma, a.eps, a.gate != nullptr ? 1 : 0, items);
    return cudaGetLastError();
}

template <typename TQ>
bool build_maps(const KdaArgs& a, Maps& mp)
{
    const CUtensorMapDataType dq =
        std::is_same<TQ, __half>::value ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    if (!make_map(&mp.q, a.q, dq, a.B, a.T, a.H) || !make_map(&mp.k, a.k, dq, a.B, a.T, a.H) ||
        !make_map(&mp.v, a.v, dq, a.B, a.T, a.H) ||
        !make_map(&mp.g, a.g, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.B, a.T, a.H))
        return false;
    if (a.out_t == ET_F32 || !a.o) mp.o = mp.q;
    else if (!make_map_o(&mp.o, a.o, a.B, a.T, a.H)) return false;
    if (a.gate && a.out_t == ET_BF16) return make_map_gate(&mp.gate, a.gate, a.B, a.T, a.H);
    mp.gate = mp.q;
    return true;
}

int sm_count()
{
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

// Start states of every segment from a.S0 and the maps of segments 0..P-2 (uniform
// layout, head bh's at bh*(P-1)), then the output pass.
template <typename TQ>
cudaError_t combine_output(const Maps& mp, const KdaArgs& a, const Split& sp, float* maps, float* starts,
                           int* status, cudaStream_t s)
{
    if (sp.P == 1) return launch_pass<MODE_OUTPUT, TQ>(mp, a, a.S0, 0, nullptr, 1, sp.L, status, s);
    {
        cudaError_t e = cudaFuncSetAttribute(kda_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             cb_smem_bytes());
        if (e != cudaSuccess) return e;
        ProfileScope prof("kda_tc_combine", s);
        count_launch();
        kda_combine_kernel<<<dim3(D / 16, a.H, a.B), CB_THREADS, cb_smem_bytes(), s>>>(maps, a.S0, starts, a.H, sp.P,
                                                                                        nullptr);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return launch_pass<MODE_OUTPUT, TQ>(mp, a, starts, 1, maps, sp.P, sp.L, status, s);
}

// ---- uniform batch: two waves ------------------------------------------------------------
// With W = floor(#SM / (B*H)) >= 2 CTAs per head and wave, a head's chunks are cut into
// P = W + 1 segments of L chunks:
//   wave 1: the output pass of segment 0 (from S0; it also yields S_start(1) exactly) on an
//           auxiliary stream, beside the state pass of segments 1..P-2,
//   combine: S_start(p+1) = M_p S_start(p) + N_p from S_start(1), p = 1..P-2,
//   wave 2: the output pass of segments 1..P-1.
// Both waves hold W CTAs per head, so L = ceil(NC / (W+1)) instead of ceil(NC / W).
// Workspace: maps [B*H][P-2][N | M], starts [B*H][P-1][D][D], S_start(1) [B*H][D][D],
// three item tables.
struct Waves {
    int P, L;
    size_t maps_b, starts_b, s1_b, it0_b, its_b, ito_b;
    size_t total() const { return maps_b + starts_b + s1_b + it0_b + its_b + ito_b; }
};

size_t a256(size_t x) { return (x + 255) & ~size_t(255); }

Waves waves_for(int B, int T, int H, int sms)
{
    Waves w{};
    const int NC = (T + C - 1) / C, BH = max(1, B * H);
    const int W = sms / BH;
    if (W < 2 || NC < 2) {   // one wave: every head one segment, or the plain split
        w.P = 1;
        w.L = NC;
        return w;
    }
    int P = min(W + 1, NC);
    w.L = (NC + P - 1) / P;
    w.P = P = (NC + w.L - 1) / w.L;   // no empty segment
    const size_t bh = (size_t)B * H;
    w.maps_b = a256(bh * (size_t)max(0, P - 2) * 2 * D * D * sizeof(float));
    w.starts_b = a256(bh * (size_t)(P - 1) * D * D * sizeof(float));
    w.s1_b = a256(bh * D * D * sizeof(float));
    w.it0_b = a256(bh * 8 * sizeof(int));
    w.its_b = a256(bh * (size_t)max(0, P - 2) * 8 * sizeof(int));
    w.ito_b = a256(bh * (size_t)(P - 1) * 8 * sizeof(int));
    return w;
}

// The auxiliary stream of this device for wave 1's segment-0 pass, and the two events of
// its fork and join.  One enqueue sequence at a time uses them (the mutex), so the events
// always refer to the call that recorded them.
struct Aux {
    cudaStream_t s = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};
std::mutex g_aux_mu;
Aux g_aux[64];

template <typename TQ>
cudaError_t launch_all(const KdaArgs& a, void* ws, int* status, cudaStream_t s)
{
    const Waves wv = waves_for(a.B, a.T, a.H, sm_count());
    const Split sp = split_for(a.B, a.T, a.H, sm_count());
    Maps mp;
    if (!build_maps<TQ>(a, mp)) return cudaErrorInvalidValue;
    // the gated epilogue needs whole-chunk TMA stores, which the item tables' ragged
    // sequence ends do not give: it keeps the one-table split
    if (wv.P == 1 || a.gate) {
        float* maps = reinterpret_cast<float*>(ws);
        float* starts = maps + (size_t)a.B * a.H * (sp.P - 1) * 2 * D * D;
        if (sp.P > 1) {
            const cudaError_t e = launch_pass<MODE_STATE, TQ>(mp, a, nullptr, 0, maps, sp.P, sp.L, status, s);
            if (e != cudaSuccess) return e;
        }
        return combine_output<TQ>(mp, a, sp, maps, starts, status, s);
    }
    const int P = wv.P, L = wv.L, BH = a.B * a.H;
    // item tables address packed rows: the bf16 output map spans all B*T rows as one
    if (a.out_t == ET_BF16 && !make_map_o(&mp.o, a.o, 1, a.B * a.T, a.H)) return cudaErrorInvalidValue;
    char* base = reinterpret_cast<char*>(ws);
    float* maps = reinterpret_cast<float*>(base);
    float* starts = reinterpret_cast<float*>(base + wv.maps_b);
    float* s1 = reinterpret_cast<float*>(base + wv.maps_b + wv.starts_b);
    int* it0 = reinterpret_cast<int*>(base + wv.maps_b + wv.starts_b + wv.s1_b);
    int* its = reinterpret_cast<int*>(base + wv.maps_b + wv.starts_b + wv.s1_b + wv.it0_b);
    int* ito = reinterpret_cast<int*>(base + wv.maps_b + wv.starts_b + wv.s1_b + wv.it0_b + wv.its_b);
    cudaError_t e;
    {
        const int n = BH * P;
        count_launch();
        wave_items_kernel<<<(n + 255) / 256, 256, 0, s>>>(it0, its, ito, a.B, a.T, a.H, P, L);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    {
        std::lock_guard<std::mutex> lk(g_aux_mu);
        Aux& ax = g_aux[dev];
        if (!ax.s) {
            e = cudaStreamCreateWithFlags(&ax.s, cudaStreamNonBlocking);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ax.fork, cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ax.join, cudaEventDisableTiming);
            if (e != cudaSuccess) return e;
        }
        // wave 1: segment 0's output pass (end state -> s1) beside the state pass
        e = cudaEventRecord(ax.fork, s);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(ax.s, ax.fork, 0);
        if (e != cudaSuccess) return e;
        KdaArgs a0 = a;
        a0.ST = s1;
        e = launch_pass<MODE_OUTPUT, TQ>(mp, a0, a.S0, 0, nullptr, P, L, status, ax.s, it0, BH, "kda_tc_output_first");
        if (e == cudaSuccess) e = cudaEventRecord(ax.join, ax.s);
        if (e != cudaSuccess) return e;
        if (P > 2) {
            e = launch_pass<MODE_STATE, TQ>(mp, a, nullptr, 0, maps, P, L, status, s, its, BH * (P - 2));
            if (e != cudaSuccess) return e;
        }
        e = cudaStreamWaitEvent(s, ax.join, 0);
        if (e != cudaSuccess) return e;
    }
    if (P == 2)   // segment 1 starts from segment 0's end state
        return launch_pass<MODE_OUTPUT, TQ>(mp, a, s1, 0, nullptr, P, L, status, s, ito, BH);
    e = cudaFuncSetAttribute(kda_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, cb_smem_bytes());
    if (e != cudaSuccess) return e;
    {
        ProfileScope prof("kda_tc_combine", s);
        count_launch();
        kda_combine_kernel<<<dim3(D / 16, a.H, a.B), CB_THREADS, cb_smem_bytes(), s>>>(maps, s1, starts, a.H, P - 1,
                                                                                        nullptr);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return launch_pass<MODE_OUTPUT, TQ>(mp, a, starts, 1, maps, P, L, status, s, ito, BH * (P - 1));
}

// ---- one shard of a sequence cut across devices -----------------------------------------
// The state pass runs every segment of the shard, the last one included: segments
// 0..P-2 write their maps in the uniform layout (the output pass reads them), the last
// one into a tail slot per head after them.  Workspace: maps [B*H*P][N | M], start
// states [B*H*P][D][D], the item table.
struct SpLayout {
    Split sp;
    size_t maps_bytes, starts_bytes, items_bytes;
    size_t total() const { return maps_bytes + starts_bytes + items_bytes; }
};

SpLayout sp_layout(int B, int T, int H, int sms)
{
    SpLayout l;
    l.sp = split_for(B, T, H, sms);
    const size_t bhp = (size_t)B * H * l.sp.P;
    l.maps_bytes = a256(bhp * 2 * D * D * sizeof(float));
    l.starts_bytes = a256(bhp * D * D * sizeof(float));
    l.items_bytes = a256(bhp * 8 * sizeof(int));
    return l;
}

template <typename TQ>
cudaError_t launch_sp_state(const KdaArgs& a, void* ws, int* status, cudaStream_t s, TcShardMaps* out)
{
    const SpLayout l = sp_layout(a.B, a.T, a.H, sm_count());
    const int P = l.sp.P, L = l.sp.L, NC = (a.T + C - 1) / C, BH = a.B * a.H;
    Maps mp;
    if (!build_maps<TQ>(a, mp)) return cudaErrorInvalidValue;
    float* maps = reinterpret_cast<float*>(ws);
    int* items = reinterpret_cast<int*>(reinterpret_cast<char*>(ws) + l.maps_bytes + l.starts_bytes);
    std::vector<int> it;
    it.reserve((size_t)BH * P * 8);
    for (int b = 0; b < a.B; ++b)
        for (int h = 0; h < a.H; ++h)
            for (int p = 0; p < P; ++p) {
                const int bh = b * a.H + h;
                const int slot = p < P - 1 ? bh * (P - 1) + p : BH * (P - 1) + bh;
                const int e[8] = {b * a.T, a.T, p * L, min(NC, (p + 1) * L), h, b, slot, p == P - 1};
                it.insert(it.end(), e, e + 8);
            }
    // pageable source: the copy is staged before the call returns
    cudaError_t e = cudaMemcpyAsync(items, it.data(), it.size() * sizeof(int), cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return e;
    e = launch_pass<MODE_STATE, TQ>(mp, a, nullptr, 0, maps, P, L, status, s, items, BH * P);
    out->P = P;
    out->maps = maps;
    out->tail = maps + (size_t)BH * (P - 1) * 2 * D * D;
    return e;
}

template <typename TQ>
cudaError_t launch_sp_output(const KdaArgs& a, void* ws, int* status, cudaStream_t s)
{
    const SpLayout l = sp_layout(a.B, a.T, a.H, sm_count());
    Maps mp;
    if (!build_maps<TQ>(a, mp)) return cudaErrorInvalidValue;
    float* maps = reinterpret_cast<float*>(ws);
    float* starts = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + l.maps_bytes);
    return combine_output<TQ>(mp, a, l.sp, maps, starts, status, s);
}

// ---- packed samples (cu_seqlens) ------------------------------------------------------
// Every sample gets P_i = ceil(NC_i / L) segments of L chunks, with one L for the call,
// the smallest that keeps sum_i H * P_i within one wave of CTAs (or L = the longest
// sample).  Items are 8 ints {rowbase, length, n0, n1, head, sample, slot, last}.
struct VarlenPlan {
    int L = 1;
    std::vector<int> st_items, out_items, seqinfo;   // state pass, output pass, per sample
    size_t n_maps = 0, n_starts = 0;
};

VarlenPlan plan_varlen(const int* cu, int n, int H, int sms)
{
    VarlenPlan pl;
    int64_t work = 0;
    int max_nc = 0;
    for (int i = 0; i < n; ++i) {
        const int nc = (cu[i + 1] - cu[i] + C - 1) / C;
        work += (int64_t)nc * H;
        max_nc = max(max_nc, nc);
    }
    if (max_nc > 0) {
        int64_t L0 = (work + sms - 1) / sms;
        int L = (int)(L0 < 1 ? 1 : L0);
        auto ctas = [&](int Lc) {
            int64_t m = 0;
            for (int i = 0; i < n; ++i) m += (int64_t)H * (((cu[i + 1] - cu[i] + C - 1) / C + Lc - 1) / Lc);
            return m;
        };
        while (L < max_nc && ctas(L) > sms) ++L;
        pl.L = min(L, max_nc);
    }
    pl.seqinfo.resize(3 * (size_t)n);
    for (int i = 0; i < n; ++i) {
        const int len = cu[i + 1] - cu[i], nc = (len + C - 1) / C;
        const int Pi = nc ? (nc + pl.L - 1) / pl.L : 0;
        const size_t map_base = pl.n_maps, start_base = pl.n_starts;
        pl.seqinfo[3 * i] = Pi;
        pl.seqinfo[3 * i + 1] = (int)map_base;
        pl.seqinfo[3 * i + 2] = (int)start_base;
        for (int h = 0; h < H; ++h)
            for (int p = 0; p < Pi; ++p) {
                const int n0 = p * pl.L, n1 = min(nc, n0 + pl.L);
                if (p < Pi - 1) {
                    const int st[8] = {cu[i], len, n0, n1, h, i, (int)(map_base + (size_t)h * (Pi - 1) + p), 0};
                    pl.st_items.insert(pl.st_items.end(), st, st + 8);
                }
                const int ot[8] = {cu[i], len, n0, n1, h, i, (int)(start_base + (size_t)h * Pi + p), p == Pi - 1};
                pl.out_items.insert(pl.out_items.end(), ot, ot + 8);
            }
        pl.n_maps += (size_t)H * (Pi > 0 ? Pi - 1 : 0);
        pl.n_starts += (size_t)H * Pi;
    }
    return pl;
}

size_t varlen_ws_bytes(const VarlenPlan& pl, int n)
{
    return a256(pl.n_maps * 2 * D * D * sizeof(float)) + a256(pl.n_starts * D * D * sizeof(float)) +
           a256(pl.st_items.size() * sizeof(int)) + a256(pl.out_items.size() * sizeof(int)) +
           a256(3 * (size_t)n * sizeof(int));
}

template <typename TQ>
cudaError_t launch_varlen(const KdaArgs& a, const int* cu, int n, void* ws, int* status, cudaStream_t s)
{
    const VarlenPlan pl = plan_varlen(cu, n, a.H, sm_count());
    const CUtensorMapDataType dq =
        std::is_same<TQ, __half>::value ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    Maps mp;
    if (!make_map(&mp.q, a.q, dq, 1, a.T, a.H) || !make_map(&mp.k, a.k, dq, 1, a.T, a.H) ||
        !make_map(&mp.v, a.v, dq, 1, a.T, a.H) || !make_map(&mp.g, a.g, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 1, a.T, a.H))
        return cudaErrorInvalidValue;
    if (a.out_t == ET_F32) mp.o = mp.q;
    else if (!make_map_o(&mp.o, a.o, 1, a.T, a.H)) return cudaErrorInvalidValue;
    mp.gate = mp.q;
    char* base = reinterpret_cast<char*>(ws);
    float* maps = reinterpret_cast<float*>(base);
    base += a256(pl.n_maps * 2 * D * D * sizeof(float));
    float* starts = reinterpret_cast<float*>(base);
    base += a256(pl.n_starts * D * D * sizeof(float));
    int* st_items = reinterpret_cast<int*>(base);
    base += a256(pl.st_items.size() * sizeof(int));
    int* out_items = reinterpret_cast<int*>(base);
    base += a256(pl.out_items.size() * sizeof(int));
    int* seqinfo = reinterpret_cast<int*>(base);
    // pageable sources: the copies are staged before the calls return
    cudaError_t e = cudaSuccess;
    if (!pl.st_items.empty())
        e = cudaMemcpyAsync(st_items, pl.st_items.data(), pl.st_items.size() * sizeof(int), cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess && !pl.out_items.empty())
        e = cudaMemcpyAsync(out_items, pl.out_items.data(), pl.out_items.size() * sizeof(int), cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(seqinfo, pl.seqinfo.data(), pl.seqinfo.size() * sizeof(int), cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return e;
    KdaArgs b1 = a;
    b1.B = 1;
    const int n_st = (int)(pl.st_items.size() / 8), n_out = (int)(pl.out_items.size() / 8);
    if (n_st > 0) {
        e = launch_pass<MODE_STATE, TQ>(mp, b1, nullptr, 0, maps, 0, pl.L, status, s, st_items, n_st);
        if (e != cudaSuccess) return e;
    }
    if (n_out == 0) return cudaSuccess;
    {
        e = cudaFuncSetAttribute(kda_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, cb_smem_bytes());
        if (e != cudaSuccess) return e;
        ProfileScope prof("kda_tc_combine", s);
        count_launch();
        kda_combine_kernel<<<dim3(D / 16, a.H, n), CB_THREADS, cb_smem_bytes(), s>>>(maps, a.S0, starts, a.H, 0,
                                                                                    seqinfo);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return launch_pass<MODE_OUTPUT, TQ>(mp, b1, starts, 1, maps, 0, pl.L, status, s, out_items, n_out);
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
    if (a.gate && (a.in_t != ET_BF16 || !aligned16(a.gate) || (a.gamma && !aligned16(a.gamma)))) return false;
    return encode_fn() != nullptr;
}

size_t kda_tc_workspace_bytes(int B, int T, int H, int chunk, int num_sms)
{
    if (chunk != C || T < 1) return 0;
    // the larger of the two-wave layout and the one-table split (the gated epilogue)
    const Split sp = split_for(B, T, H, num_sms);
    const size_t one = sp.P == 1 ? 0 : (size_t)B * H * ((size_t)(sp.P - 1) * 2 + sp.P) * D * D * sizeof(float);
    const Waves wv = waves_for(B, T, H, num_sms);
    return std::max<size_t>(one, wv.P == 1 ? (size_t)0 : wv.total());
}

size_t kda_tc_varlen_workspace_bytes(const int* cu, int n, int H, int num_sms)
{
    const VarlenPlan pl = plan_varlen(cu, n, H, num_sms);
    return varlen_ws_bytes(pl, n);
}

cudaError_t launch_kda_tc_varlen(const KdaArgs& a, const int* cu, int n, void* ws, int* status, cudaStream_t s)
{
    if (a.in_t == ET_F16) return launch_varlen<__half>(a, cu, n, ws, status, s);
    return launch_varlen<__nv_bfloat16>(a, cu, n, ws, status, s);
}

size_t kda_tc_sp_workspace_bytes(int B, int T, int H, int num_sms)
{
    if (B < 1 || T < 1) return 0;
    return sp_layout(B, T, H, num_sms).total();
}

void kda_tc_plan(int B, int T, int H, int num_sms, int* P, int* L)
{
    const Waves wv = waves_for(B, T, H, num_sms);
    *P = wv.P;
    *L = wv.L;
}

cudaError_t launch_kda_tc_sp_state(const KdaArgs& a, void* ws, int* status, cudaStream_t s, TcShardMaps* out)
{
    if (a.in_t == ET_F16) return launch_sp_state<__half>(a, ws, status, s, out);
    return launch_sp_state<__nv_bfloat16>(a, ws, status, s, out);
}

cudaError_t launch_kda_tc_sp_output(const KdaArgs& a, void* ws, int* status, cudaStream_t s)
{
    if (a.in_t == ET_F16) return launch_sp_output<__half>(a, ws, status, s);
    return launch_sp_output<__nv_bfloat16>(a, ws, status, s);
}

cudaError_t launch_kda_tc(const KdaArgs& a, void* ws, size_t ws_bytes, int* status, cudaStream_t s)
{
    (void)ws_bytes;
    // the gated epilogue is fused into the output stage for a bf16 output; an fp32 output
    // gets the plain scan followed by the separate epilogue kernel
    KdaArgs scan = a;
    if (a.gate && a.out_t == ET_F32) scan.gate = nullptr;
    const cudaError_t e = a.in_t == ET_F16 ? launch_all<__half>(scan, ws, status, s)
                                           : launch_all<__nv_bfloat16>(scan, ws, status, s);
    if (e != cudaSuccess || !a.gate || a.out_t != ET_F32) return e;
    return launch_gate_rmsnorm(a, s);
}

}  // namespace kda
