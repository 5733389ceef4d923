// Tensor-core (tcgen05 / TMEM) chunkwise KDA forward for Dk = Dv = 128, chunk 64.
//
// What it computes is Eq. 14 of the Chimera paper (section 3.3) with the readout
// o_t = S_t^T q_t (Eq. 15, inner term).  Section 5.1 of the paper names a "chunked" KDA
// kernel without giving its algebra; the chunk algebra here is derived from Eq. 14.
// Inside a chunk of C = 64 tokens with entry state S0, b_i = sum_{r<=i} g_r (per key
// channel, base 2, fp32) and two per-channel references rp, rm:
//   K+ = k 2^{b - rp},  Q+ = q 2^{b - rp},  K- = k 2^{rm - b}
//   A  = strict_lower((diag(beta) K+) K-^T),   P = lower(Q+ K-^T)  (incl. diagonal)
//   T  = (I + A)^{-1}                     (16x16 blocks on warp MMAs, fp16 operands)
//   W  = T (diag(beta) K+),   U~ = T (diag(beta) V)            (state-independent)
//   S^ = diag(2^{rp}) S0:     U  = U~ - W S^,     O = Q+ S^ + P U
//   S_C = diag(2^{b_C - rm}) (diag(2^{rm}) S0 + K-^T U)
// With rp = rm = r (the chunk's middle row) A and P are products of K+ and K- whose
// factors stay within 2^{+-|b_C|/2}; a chunk whose decay is too strong for that keeps
// rp = 0 and rm = b_C (every factor <= 1) and forms A and P with pairwise exponentials
// on CUDA cores instead (chunk_ap_direct).  Every MMA operand is fp16 except the U~
// product, which takes V as it arrives (bf16 or fp16); accumulation is fp32 in TMEM.
//
// Transposed state.  The state lives in TMEM as S^T: lane j holds value column j, TMEM
// column c key channel c (fp32 master).  Every product on the state's serial chain then
// takes S^T (or U^T) as the A operand straight from TMEM, with no shared-memory round trip:
//   [U | -O]^T = [U~^T | 0] - S^T [W^T | Q+^T]      (M = 128 values, N = 128, K = 128)
//   master    += U^T K-                              (N = 128 channels, K = 64)
//   -O^T      -= U^T P^T                             (N = 64, K = 64)
// (the instruction descriptor's A negation gives the minus signs; O is negated back when
// it is written out).  The fp32 master holds diag(2^{-carry}) S: the row scales of one
// chunk and the next are applied together, once, when the next chunk reads it (S^ =
// 2^{rp + carry} master in fp16 for the A operand, and the master itself rescaled by
// 2^{rm + carry}).
//
// Parallelism.  A head's scan is sequential over chunks, and one B200 workload has
// only B*H = 16 heads for 148 SMs, so each head's chunk sequence is cut into P
// segments of L chunks.  Eq. 14 is affine in the state, so a segment maps its entry
// state S to M S + N.
//   state pass (MODE_STATE): two state chains over the segment, S from 0 with the
//          segment's values (-> N) and Phi from I without values (-> M).
//   combine: S_start(p+1) = M_p S_start(p) + N_p in fp32 (CUDA cores).
//   output pass (MODE_OUTPUT): the recurrence from S_start(p), writing o (and S_T from
//          the last segment).
//
// Inside a CTA (one per (b, h, segment), 512 threads) four roles of four warps each
// work on three chunks at once (see the kernel's comment): the prologue of chunk n+2,
// the inverse of chunk n+1 and the state chain of chunk n, with an auxiliary role for
// the output rows and the V side.  Three buffer sets of per-chunk tiles rotate; mbarriers
// hand a set from role to role and back to the loads (EMPTY, committed by the chain's
// last MMA on it).  Inputs arrive by TMA straight into the tiles that consume them.
//
// Shared-memory operand tiles use the no-swizzle core-matrix layout (8 rows x 16 B
// blocks of 128 contiguous bytes); a descriptor takes the byte stride between core
// matrices along K and along M or N.  A "channel-major" tile holds element (position i,
// channel c) at (i >> 3) * 2048 + (c >> 3) * 128 + (c & 7) * 16 + (i & 7) * 2, so it
// serves as an MN-major operand when positions are M or N and as a K-major one when
// positions are K.
//
// All waits are bounded (kWaitNs).  On expiry the kernel records DEV_TIMEOUT in the
// device status word and stops waiting: every role still runs every barrier of its loop
// (so none can hang on another), results are undefined, and before TMEM is freed each
// MMA-issuing thread drains its own MMAs.

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
constexpr int NR = 128;       // threads per role (4 warps)
// named barriers: one per role, plus the per-row-half barriers of the in-place conversions
enum { BAR_P = 1, BAR_I = 2, BAR_X = 3, BAR_Y = 4, BAR_P2 = 5 /* 5, 6 */, BAR_Y2 = 7 /* 7, 8 */ };
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s bound on every wait
constexpr float kLog2e = 1.4426950408889634f;
// Largest log2 decay factor a middle-row reference may produce in an operand tile: with
// 2^11 = 2048 an fp16 tile holds k or q components up to 32 in magnitude, and the small
// factors stay above 2^-11 (normal fp16 for components >= 1/32).
constexpr float kRangeMax = 11.f;
enum { MODE_STATE = 0, MODE_OUTPUT = 1 };

// ---- shared-memory plan (bytes) --------------------------------------------------
// NSET buffer sets of per-chunk tiles; chunk x uses set x % NSET.  Per set: KP (k -> beta
// K+ -> -W^T) and QP (q -> Q+) as channel-major tiles, QP directly after KP so [beta K+;
// Q+] and [-W^T | Q+^T] are single 128-row operands; KM (g as TMA lands it -> K-); PF (P
// as the K-major B operand of O^T += U^T P^T); TF (T as the K-major B operand T^T of W^T
// and, scaled by beta per column, of U~^T = V^T (T diag(beta))^T).  Three sets keep three
// chunks in flight (prologue, inverse, state chain), so the loads of a chunk have a whole
// chunk period to land.  One v tile (core matrices [value group][position][8]).
constexpr int NSET = 3;
template <int MODE> struct Plan;
template <> struct Plan<MODE_OUTPUT> {
    static constexpr int SET = 65536;
    static constexpr int KP = 0, QP = 16384, KM = 32768, PF = 49152, TF = 57344;
    static constexpr int T_LBO = 1024, T_BYTES = 8192;
    static constexpr int VB = NSET * SET;
    static constexpr int SCR = -1;                 // (chunk_ap_direct's table: the set's PF and TF)
    static constexpr int MISC = VB + 16384;
    static constexpr int LOAD_BYTES = 3 * 16384;   // q, k and g of one chunk
};
template <> struct Plan<MODE_STATE> {
    static constexpr int SET = 40960;
    static constexpr int KP = 0, QP = -1, KM = 16384, PF = 0, TF = 32768;   // no q, no P
    static constexpr int T_LBO = 1024, T_BYTES = 8192;
    static constexpr int VB = NSET * SET;
    static constexpr int SCR = VB + 16384;         // 16 KB table of chunk_ap_direct
    static constexpr int MISC = SCR + 16384;
    static constexpr int LOAD_BYTES = 2 * 16384;   // k and g of one chunk
};
// MISC sub-layout
constexpr int NBETA = 8;         // beta slots (written two chunks ahead, read up to two behind)
constexpr int M_BETA = 0;        // bf16[NBETA][64]  beta of chunk x in slot x % NBETA
constexpr int M_BRAW = 1024;     // uint32[64]    the head pair's beta words as cp.async lands them
constexpr int M_TOT = 1280;      // float[2][128] per-32-row sums of g log2(e)
constexpr int M_SC = 2304;       // float[NSET][3][128] per set: S^ scale, master scale, carry after
constexpr int M_XS = 6912;       // 8 x 512 B per-item 16x16 fp16 scratch of the inverse
constexpr int M_BAR = 11008;     // mbarriers, see Bar
constexpr int M_TMEM = 11264;    // uint32 TMEM base
constexpr int M_ABORT = 11268;   // int
constexpr int M_DIRECT = 11272;  // int[NSET] per set: its chunk's A and P came from chunk_ap_direct
constexpr int M_RED = 11296;     // float[4][64] per-row sums of squares (gated output)
constexpr int MISC_BYTES = 12320;
enum Bar {
    B_LD = 0,       // [3] set s: q, k, g of its chunk landed
    B_TV = 3,       // the v tile landed
    B_VE = 4,       // [2] chunk parity x: the U~ MMA of chunk x (which read the v tile) is done.
                    // Two of them: U~ of chunk kc+1 may be done before the chain role has
                    // polled chunk kc's, and a waiter must never be two phases behind
    B_SC = 6,       // [3] set s: prologue done (scales, direct flag, K+ / Q+ / K- tiles, beta)
    B_INV = 9,      // [3] set s: T ready
    B_PRO = 12,     // [3] set s: every tile ready (W^T written)
    B_EMPTY = 15,   // [3] set s: the chain's last MMA on it is done
    B_O = 18,       // [2] [U | O] buffer x: the chunk's O is complete
    B_AP = 20, B_W = 21, B_U = 22, B_U2 = 23, B_S = 24,
    B_APWF = 25,    // the output role has read W^T out of A|P's TMEM columns
    B_C1Y = 26,     // MODE_STATE: the output role has rescaled the Phi half of the master
    B_DRAIN = 27,   // [4] one per MMA-issuing role, after a timeout
    NBAR = 31
};
// set of chunk x (counted from the segment start) and the phase parity of its set barriers
__device__ __forceinline__ int set_of(int x) { return x % NSET; }
__device__ __forceinline__ uint32_t set_par(int x) { return (uint32_t)(x / NSET) & 1u; }
static_assert(M_BAR + NBAR * 8 <= M_TMEM, "barrier block");
static_assert(M_DIRECT + 4 * NSET <= M_RED && M_SC + NSET * 3 * 128 * 4 <= M_XS, "misc block");
static_assert(M_RED % 16 == 0 && M_RED + 1024 <= MISC_BYTES, "misc block");

template <int MODE> constexpr int smem_bytes() { return Plan<MODE>::MISC + MISC_BYTES; }
static_assert(smem_bytes<MODE_OUTPUT>() <= 232448 && smem_bytes<MODE_STATE>() <= 232448, "shared memory");

// TMEM columns.
//   MODE_OUTPUT: master S^T [0,128) | S^ fp16 [128,192) | [U|O] x2 [192,448) | A|P, W^T [448,512)
//   MODE_STATE:  S^T [0,128), Phi^T [128,256) | S^, Phi^ fp16 [256,320), [320,384) |
//                U [384,448) | A, W^T [448,512)
constexpr uint32_t TM_APW = 448;
template <int MODE> struct Tm;
// (UO / UACC name the same region for the mode that has no such buffer; never used there)
template <> struct Tm<MODE_OUTPUT> { static constexpr uint32_t MASTER = 0, S16 = 128, UO = 192, UACC = 192; };
template <> struct Tm<MODE_STATE> { static constexpr uint32_t MASTER = 0, S16 = 256, UACC = 384, UO = 384; };

// ---- helpers ------------------------------------------------------------------------
__device__ __forceinline__ uint4 pack8_f16(const float* f)
{
    uint4 u;
    __half2* h = reinterpret_cast<__half2*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
    return u;
}

// Two fp32 values -> a packed pair of the input type (bf16 or fp16)
template <typename TQ> __device__ __forceinline__ uint32_t pack2_in(float lo, float hi);
template <> __device__ __forceinline__ uint32_t pack2_in<__half>(float lo, float hi) { return pack_f16x2(lo, hi); }
template <> __device__ __forceinline__ uint32_t pack2_in<__nv_bfloat16>(float lo, float hi)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

// Two adjacent 2-byte input elements -> fp32
__device__ __forceinline__ float2 in2(uint32_t u, const __nv_bfloat16*)
{
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}
__device__ __forceinline__ float2 in2(uint32_t u, const __half*) { return unpack_f16x2(u); }

// Byte offset of (row i, column j), j % 8 == 0, in a 64 x 64 fp16 tile in the
// K-major core-matrix layout (8-column groups 1 KB apart).
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
// The slow part of a wait, out of line (one copy per kernel instead of one per wait):
// sleep-poll the barrier for at most kWaitNs; on expiry raise the abort flag and record
// DEV_TIMEOUT.
__device__ __noinline__ void wait_slow(uint64_t* bar, uint32_t parity, int* flag, int* status)
{
    if (!mbar_wait_bounded(bar, parity, kWaitNs)) {
        *flag = 1;
        atomicCAS(status, DEV_OK, DEV_TIMEOUT);
    }
}
// One thread waits alone (before issuing MMAs that depend on another role).
__device__ __forceinline__ void thread_wait(uint64_t* bar, uint32_t parity, const Abort& a)
{
    if (!*a.flag && !mbar_try_wait(bar, parity)) wait_slow(bar, parity, a.flag, a.status);
}
// One thread polls; the role (bar_id, NR threads) waits at its named barrier.
__device__ __forceinline__ void group_wait(uint64_t* bar, uint32_t parity, const Abort& a, bool poller, int bar_id)
{
    if (poller) thread_wait(bar, parity, a);
    named_sync(bar_id, NR);
    tc_fence_after();
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
// 4 bytes global -> shared by cp.async (valid = false: zero-filled, nothing is read)
__device__ __forceinline__ void cp_async4_zfill(void* smem, const void* gmem, bool valid)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_addr(smem)), "l"(gmem), "r"(valid ? 4 : 0)
                 : "memory");
}
// beta of token t0 + i as raw bf16 bits (0 past the sequence end)
__device__ __forceinline__ uint16_t beta_bits(const __nv_bfloat16* beta, int64_t rowbase, int T, int H, int h, int t0,
                                              int i, bool live)
{
    return (uint16_t)load_beta(beta, rowbase, T, H, h, t0, i, live);
}
__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

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

// A (and P) of one chunk on CUDA cores, for a chunk whose decay range is too wide for a
// single reference: A_ij = beta_i sum_c k_ic k_jc 2^{b_ic - b_jc} (j < i) and P_ij =
// sum_c q_ic k_jc 2^{b_ic - b_jc} (j <= i), every exponential <= 1 formed directly.  In
// the buffer set `set` the raw k (and q) tiles are still in KP (QP) and g in KM; `tot`
// holds each channel's sum of g log2(e) over rows 0-31; nv rows are inside the sequence.
// The fp32 table b[64][64] of one 64-channel half (base 2, from the chunk start) is built
// in `scr` (16 KB) for each half in turn.  Writes A (fp16) to TF and P to PF in the cm64
// layout (both zero above the diagonal); `scr` may overlap them.  Called by the 128
// threads of the prologue role (thread: row i, two 16-column blocks); barriers on BAR_P.
template <int MODE, typename TQ>
__device__ __noinline__ void chunk_ap_direct(uint8_t* set, uint8_t* scr, const float* tot, const uint16_t* sBeta,
                                             int rt, int nv)
{
    using PL = Plan<MODE>;
    constexpr bool OUT = MODE == MODE_OUTPUT;
    constexpr int bar_id = BAR_P;
    const uint8_t* gst = set + PL::KM;
    const uint8_t* ktile = set + PL::KP;
    const uint8_t* qtile = OUT ? set + PL::QP : set + PL::KP;
    uint8_t* at = set + PL::TF;
    uint8_t* pf = set + PL::PF;
    float* bT = reinterpret_cast<float*>(scr);
    const int i = rt & 63, jh = rt >> 6;
    const float bi = bf16_bits_to_f32(sBeta[i]);
    uint4 resA[2][2], resP[2][2];            // fp16 results of the two blocks (written last)
    const TQ* tq = nullptr;
    for (int pass = 0; pass < 2; ++pass) {
        const int cq = 2 * jh + pass;        // 16-column block of this pass
        float accA[16], accP[16];
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) accA[jj] = accP[jj] = 0.f;
        for (int hc = 0; hc < 2; ++hc) {
            // the table of channels 64 hc .. 64 hc + 63: thread (channel cc, 32-row half)
            named_sync(bar_id, 128);         // the previous table is no longer read
            {
                const int cc = rt & 63, rh2 = rt >> 6, c = 64 * hc + cc;
                float run = rh2 ? tot[c] : 0.f;
#pragma unroll 4
                for (int r = 0; r < 32; ++r) {
                    const int ii = 32 * rh2 + r;
                    const float gv = ii < nv ? bf16_bits_to_f32(*reinterpret_cast<const uint16_t*>(gst + ii * 256 + 2 * c)) : 0.f;
                    run = fmaf(gv, kLog2e, run);
                    bT[ii * 64 + cc] = run;
                }
            }
            named_sync(bar_id, 128);
            if (16 * cq <= i && i < nv) {
                for (int c8h = 0; c8h < 8; ++c8h) {
                    const int c8 = 8 * hc + c8h;
                    const uint4 ku = *reinterpret_cast<const uint4*>(ktile + i * 256 + c8 * 16);
                    const uint4 qu = OUT ? *reinterpret_cast<const uint4*>(qtile + i * 256 + c8 * 16) : make_uint4(0, 0, 0, 0);
                    const float4 b0 = *reinterpret_cast<const float4*>(bT + i * 64 + 8 * c8h);
                    const float4 b1 = *reinterpret_cast<const float4*>(bT + i * 64 + 8 * c8h + 4);
                    float ki[8], qi[8];
                    const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
                    {
                        const uint32_t kw[4] = {ku.x, ku.y, ku.z, ku.w}, qw[4] = {qu.x, qu.y, qu.z, qu.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 x = in2(kw[e], tq), y = in2(qw[e], tq);
                            ki[2 * e] = x.x; ki[2 * e + 1] = x.y;
                            qi[2 * e] = y.x; qi[2 * e + 1] = y.y;
                        }
                    }
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj) {
                        const int j = 16 * cq + jj;
                        if (j <= i) {
                            const uint4 kj = *reinterpret_cast<const uint4*>(ktile + j * 256 + c8 * 16);
                            const float4 c0 = *reinterpret_cast<const float4*>(bT + j * 64 + 8 * c8h);
                            const float4 c1 = *reinterpret_cast<const float4*>(bT + j * 64 + 8 * c8h + 4);
                            const float bj[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                            const uint32_t kw[4] = {kj.x, kj.y, kj.z, kj.w};
                            float sa = 0.f, sp = 0.f;
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 kk = in2(kw[e], tq);
                                const float d0 = ex2_approx(bv[2 * e] - bj[2 * e]) * kk.x;
                                const float d1 = ex2_approx(bv[2 * e + 1] - bj[2 * e + 1]) * kk.y;
                                sa = fmaf(ki[2 * e], d0, fmaf(ki[2 * e + 1], d1, sa));
                                if (OUT) sp = fmaf(qi[2 * e], d0, fmaf(qi[2 * e + 1], d1, sp));
                            }
                            accA[jj] += sa;
                            accP[jj] += sp;
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            float fa[8], fp[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int jj = 8 * half + e, j = 16 * cq + jj;
                fa[e] = j < i ? bi * accA[jj] : 0.f;
                fp[e] = j <= i ? accP[jj] : 0.f;
            }
            resA[pass][half] = pack8_f16(fa);
            resP[pass][half] = pack8_f16(fp);
        }
    }
    named_sync(bar_id, 128);   // the table may be overwritten (in MODE_OUTPUT it covers PF and TF)
#pragma unroll
    for (int pass = 0; pass < 2; ++pass)
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int j0 = 16 * (2 * jh + pass) + 8 * half;
            *reinterpret_cast<uint4*>(at + cm64(i, j0)) = resA[pass][half];
            if (OUT) *reinterpret_cast<uint4*>(pf + cm64(i, j0)) = resP[pass][half];
        }
}

// Inverse T = (I + A)^{-1} of the strictly lower 64 x 64 A, in place: A (fp16, zero above
// the diagonal) is in the T tile, whose cmT layout equals cm64 for T_LBO = 1024, and each
// block of A is read before the block of T at its place is written.
// Diagonal 16x16 blocks (warp w4 owns block w4): with N = A_ww (strictly lower, N^16 = 0),
// (I + N)^{-1} = (I - N)(I + N^2)(I + N^4)(I + N^8) on warp MMAs.  Then the off-diagonal
// blocks by halves of the matrix (a work item: one 8-column half of one 16x16 block; X
// products through per-item fp16 scratch):
//   level 1: T_10 = -T_11 (A_10 T_00),  T_32 = -T_33 (A_32 T_22)
//   level 2: X_IJ = sum_{K=J}^{1} A_IK T_KJ  (I = 2, 3; J = 0, 1), then T_IJ = -sum_{K=2}^{I} T_IK X_KJ
// Called by the 4 warps (128 threads) of the inverse role; barriers on bar_id.
template <int T_LBO>
__device__ __forceinline__ void invert_unit_lower(uint32_t Tt, uint32_t xs, int w4, int lane, int bar_id)
{
    static_assert(T_LBO == 1024, "A and T share the tile layout");
    const uint32_t Ah = Tt;
    auto cmT = [](int i, int j) -> uint32_t { return (j >> 3) * T_LBO + (i >> 3) * 128 + (i & 7) * 16; };
    const int g = lane >> 2, q = lane & 3;
    {
        const int b0 = 16 * w4;
        const uint32_t scr = xs + 512 * w4;
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
        // Z = I - N + N^2 - N^3, in the C layout (rows g, g+8; columns 2q, 2q+1 of each
        // 8-column half); N's values come from its A fragment
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
    named_sync(bar_id, 128);
    auto scr_of = [&](int it) { return xs + 512 * it; };
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
    {   // level 1: warp w4 -> block (I, I-1), half w4 & 1
        const int half = w4 & 1;
        const int I = (w4 >> 1) ? 3 : 1, J = I - 1, N0 = 16 * J + 8 * half;
        uint32_t aA[4], bT[2], bX[2], aT[4];
        float x[4] = {0.f, 0.f, 0.f, 0.f}, tt[4] = {0.f, 0.f, 0.f, 0.f};
        a_frag(aA, Ah, I, J, false);
        named_sync(bar_id, 128);   // both halves of A_IJ are read before T_IJ's halves are written
        ldsm_x2_t(bT, Tt + cmT(16 * J + (lane & 7) + 8 * ((lane >> 3) & 1), N0));
        mma16816(x, aA, bT);
        put_x(scr_of(w4), x);
        __syncwarp();
        ldsm_x2_t(bX, scr_of(w4) + cm16((lane & 7) + 8 * ((lane >> 3) & 1), 0));
        a_frag(aT, Tt, I, I, true);
        mma16816(tt, aT, bX);
        put_t(I, N0, tt);
    }
    named_sync(bar_id, 128);
    // level 2, X: item it -> block (I, J) = (2 + (it >> 2), (it >> 1) & 1), half it & 1
#pragma unroll
    for (int r2 = 0; r2 < 2; ++r2) {
        const int it = w4 + 4 * r2;
        const int I2 = 2 + (it >> 2), J2 = (it >> 1) & 1, N2 = 16 * J2 + 8 * (it & 1);
        float x[4] = {0.f, 0.f, 0.f, 0.f};
        for (int K = J2; K < 2; ++K) {
            uint32_t aA[4], bT[2];
            a_frag(aA, Ah, I2, K, false);
            ldsm_x2_t(bT, Tt + cmT(16 * K + (lane & 7) + 8 * ((lane >> 3) & 1), N2));
            mma16816(x, aA, bT);
        }
        put_x(scr_of(it), x);
    }
    named_sync(bar_id, 128);
    // level 2, T: the same items; X_KJ half was written by item 4(K-2) + 2J + half
#pragma unroll
    for (int r2 = 0; r2 < 2; ++r2) {
        const int it = w4 + 4 * r2;
        const int I2 = 2 + (it >> 2), J2 = (it >> 1) & 1, half = it & 1, N2 = 16 * J2 + 8 * half;
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

// 8 x 8 transpose of 16-bit values inside each group of 8 lanes.  Lane l (of the group)
// holds row l as w[m] = (column 2m, column 2m + 1) (low half first); on return z[m] =
// (row 2m, row 2m + 1) of column l.  Three exchange rounds (lane distance 4, 2, 1), each
// moving half of the data: 6 shuffles.
__device__ __forceinline__ void transpose8x8_b16(const uint32_t* w, uint32_t (&z)[4], int lane)
{
    const bool b = (lane & 4) != 0, c = (lane & 2) != 0, d = (lane & 1) != 0;
    // distance 4: keep columns 4b .. 4b+3; A[0..1] = row l & ~4, A[2..3] = row l | 4
    const uint32_t r0 = __shfl_xor_sync(0xffffffffu, b ? w[0] : w[2], 4);
    const uint32_t r1 = __shfl_xor_sync(0xffffffffu, b ? w[1] : w[3], 4);
    const uint32_t A0 = b ? r0 : w[0], A1 = b ? r1 : w[1], A2 = b ? w[2] : r0, A3 = b ? w[3] : r1;
    // distance 2: keep column pair 2b + c; B[k] = row (l & 1) + 2k
    const uint32_t q0 = __shfl_xor_sync(0xffffffffu, c ? A0 : A1, 2);
    const uint32_t q1 = __shfl_xor_sync(0xffffffffu, c ? A2 : A3, 2);
    const uint32_t B0 = c ? q0 : A0, B1 = c ? A1 : q0, B2 = c ? q1 : A2, B3 = c ? A3 : q1;
    // distance 1: keep column l (the low halves if d = 0, the high halves if d = 1)
    const uint32_t t0 = __shfl_xor_sync(0xffffffffu, d ? __byte_perm(B0, B1, 0x5410) : __byte_perm(B0, B1, 0x7632), 1);
    const uint32_t t1 = __shfl_xor_sync(0xffffffffu, d ? __byte_perm(B2, B3, 0x5410) : __byte_perm(B2, B3, 0x7632), 1);
    if (d) {
        z[0] = __byte_perm(t0, B0, 0x7610);
        z[1] = __byte_perm(t0, B1, 0x7632);
        z[2] = __byte_perm(t1, B2, 0x7610);
        z[3] = __byte_perm(t1, B3, 0x7632);
    } else {
        z[0] = __byte_perm(B0, t0, 0x5410);
        z[1] = __byte_perm(B1, t0, 0x7610);
        z[2] = __byte_perm(B2, t1, 0x5410);
        z[3] = __byte_perm(B3, t1, 0x7610);
    }
}

// One 128-column half of the transposed state at the start of a chunk: S^ = fp16(2^{rp +
// carry} master) into the 64 fp16x2 columns at hcol, master <- 2^{rm + carry} master in
// place (columns mcol ..).  sY, sMs: the chunk's per-channel scales.  One thread per TMEM
// lane (tl: this warp's lane quarter); the stores are waited for by the caller.
__device__ __forceinline__ void rescale_master(uint32_t tl, uint32_t mcol, uint32_t hcol, const float* sY,
                                               const float* sMs)
{
#pragma unroll 1
    for (int c0 = 0; c0 < D; c0 += 32) {
        float vv[32];
        uint32_t hv[16], mv[32];
        tmem_ld32(tl + mcol + c0, vv);
#pragma unroll
        for (int e = 0; e < 32; e += 4) {   // packed fp32 multiplies, two channels each
            const float4 y4 = *reinterpret_cast<const float4*>(sY + c0 + e);
            const float4 m4 = *reinterpret_cast<const float4*>(sMs + c0 + e);
            const float2 v0 = make_float2(vv[e], vv[e + 1]), v1 = make_float2(vv[e + 2], vv[e + 3]);
            const float2 h0 = __fmul2_rn(v0, make_float2(y4.x, y4.y)), h1 = __fmul2_rn(v1, make_float2(y4.z, y4.w));
            hv[e / 2] = pack_f16x2(h0.x, h0.y);
            hv[e / 2 + 1] = pack_f16x2(h1.x, h1.y);
            const float2 m0 = __fmul2_rn(v0, make_float2(m4.x, m4.y)), m1 = __fmul2_rn(v1, make_float2(m4.z, m4.w));
            mv[e] = __float_as_uint(m0.x); mv[e + 1] = __float_as_uint(m0.y);
            mv[e + 2] = __float_as_uint(m1.x); mv[e + 3] = __float_as_uint(m1.y);
        }
        tmem_st16u_nowait(tl + hcol + c0 / 2, hv);
        tmem_st32u_nowait(tl + mcol + c0, mv);
    }
}

// 32 positions (32 hp0 ..) of this warp's 32 value columns, as -O, -> bf16 o rows by
// 16-byte stores (sign restored): after an 8 x 8 transpose inside each group of 8 lanes, lane l of group g8 holds
// values 8 g8 .. 8 g8 + 7 at position 8 blk + l.  row0: packed token of position 0.
__device__ __forceinline__ void store_rows_bf16(const float (&v)[32], __nv_bfloat16* o, int64_t row0, int hp0, int nvx,
                                                int H, int h, int q4, int lane)
{
    uint32_t wv[16];   // -v: the O columns hold -O
#pragma unroll
    for (int m = 0; m < 16; ++m) wv[m] = pack2_in<__nv_bfloat16>(v[2 * m], v[2 * m + 1]) ^ 0x80008000u;
    const int i0 = hp0 + (lane & 7);
    uint4* dst = reinterpret_cast<uint4*>(o + ((size_t)row0 + i0) * ((size_t)H * D) + h * D + 32 * q4 + 8 * (lane >> 3));
    const size_t step = (size_t)H * D;   // 8 positions, in 16-byte units
#pragma unroll
    for (int blk = 0; blk < 4; ++blk) {
        uint32_t z[4];
        transpose8x8_b16(wv + 4 * blk, z, lane);
        if (i0 + 8 * blk < nvx) dst[blk * step] = make_uint4(z[0], z[1], z[2], z[3]);
    }
}

__device__ __forceinline__ float tanh_approx(float x)
{
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Parameters of the output rows that only the gated or fp32 output needs.
struct OutParams {
    const __nv_bfloat16* gate;
    void* o;
    float* red;        // float[4][64] shared scratch
    float gam, eps;
    int o_f32, H, h, q4, lane;
    int64_t row_end;   // packed token just past the sequence
};
// Output rows of one chunk with the Eq. 15 output gate, or to an fp32 o; the plain bf16
// case stays inline in the kernel.  ocol: this warp's TMEM address of the chunk's -O^T
// (lane = value column, 64 position columns).  Called by the 128 threads of the output
// role; the gated case syncs them once (BAR_Y).
__device__ __forceinline__ void out_rows_general(const OutParams* op, uint32_t ocol, int64_t row0, int nvx)
{
    const __nv_bfloat16* gate = op->gate;
    void* o = op->o;
    float* red = op->red;
    const float gam = op->gam, eps = op->eps;
    const int o_f32 = op->o_f32, H = op->H, h = op->h, q4 = op->q4, lane = op->lane;
    const int j = 32 * q4 + lane;
    float inv_lo = 0.f, inv_hi = 0.f;   // per-position inverse RMS (gated output)
    if (gate) {
        // the next chunk's gate rows toward L2 (one 128-byte line per thread)
        const int t128 = 32 * q4 + lane;
        const int64_t rn = row0 + C + (t128 >> 1);
        if (rn < op->row_end)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(gate + ((size_t)rn * H + h) * D + 64 * (t128 & 1)));
        // y = Sigmoid(gate) * gamma * RMSNorm over the head's values (Eq. 15, output side).
        // Per position, the sum of squares over this warp's 32 values by a transposing
        // butterfly (lane l ends with position 32*hp + l), then over the 4 lane quarters.
        for (int hp = 0; hp < 2; ++hp) {
            float sq[32];
            tmem_ld32(ocol + 32 * hp, sq);
#pragma unroll
            for (int u = 0; u < 32; ++u) sq[u] = sq[u] * sq[u];
#pragma unroll
            for (int sft = 16; sft >= 1; sft >>= 1) {
                const bool up = (lane & sft) != 0;
#pragma unroll
                for (int k = 0; k < sft; ++k) {
                    const float send = up ? sq[k] : sq[k + sft];
                    const float recv = __shfl_xor_sync(0xffffffffu, send, sft);
                    sq[k] = (up ? sq[k + sft] : sq[k]) + recv;
                }
            }
            red[q4 * C + 32 * hp + lane] = sq[0];
        }
        named_sync(BAR_Y, NR);
        const float m0 = (red[lane] + red[C + lane] + red[2 * C + lane] + red[3 * C + lane]) * (1.f / D) + eps;
        const float m1 =
            (red[32 + lane] + red[C + 32 + lane] + red[2 * C + 32 + lane] + red[3 * C + 32 + lane]) * (1.f / D) + eps;
        inv_lo = m0 > 0.f ? rsqrtf(m0) : 0.f;
        inv_hi = m1 > 0.f ? rsqrtf(m1) : 0.f;
    }
    for (int hp = 0; hp < 2; ++hp) {
        float v[32];
        uint16_t gb[32];   // the gate of this column at the 32 positions: all loads in flight at once
        if (gate) {
            const unsigned short* gp = reinterpret_cast<const unsigned short*>(gate) + ((size_t)row0 * H + h) * D + j;
#pragma unroll
            for (int u = 0; u < 32; ++u) gb[u] = 32 * hp + u < nvx ? __ldg(gp + (size_t)(32 * hp + u) * H * D) : 0;
        }
        tmem_ld32(ocol + 32 * hp, v);
        if (gate) {
#pragma unroll
            for (int u = 0; u < 32; ++u) {
                const float iu = __shfl_sync(0xffffffffu, hp ? inv_hi : inv_lo, u);
                const float gv = __uint_as_float((uint32_t)gb[u] << 16);
                // Sigmoid(g) = (1 + tanh(g / 2)) / 2: one MUFU operation
                v[u] = -v[u] * iu * gam * fmaf(0.5f, tanh_approx(0.5f * gv), 0.5f);
            }
        }
        if (!o_f32) {
            if (gate) {   // store_rows_bf16 negates
#pragma unroll
                for (int u = 0; u < 32; ++u) v[u] = -v[u];
            }
            store_rows_bf16(v, reinterpret_cast<__nv_bfloat16*>(o), row0, 32 * hp, nvx, H, h, q4, lane);
        } else {
            // fp32: a warp writes 32 consecutive values of a position
#pragma unroll
            for (int u = 0; u < 32; ++u) {
                const int i = 32 * hp + u;
                if (i < nvx) reinterpret_cast<float*>(o)[((size_t)row0 + i) * ((size_t)H * D) + (size_t)h * D + j] = gate ? v[u] : -v[u];
            }
        }
    }
}

// The kernel ---------------------------------------------------------------------------
// Four roles of 4 warps each (role = warp / 4; warp w4 = warp % 4 also names the TMEM lane
// quarter it may access):
//   P (role 0)  prologue: log-decay prefix and references of chunk n, the K+ / Q+ / K- tiles
//               (or A and P on CUDA cores for a wide chunk), the A|P MMA.
//   I (role 1)  inverse: A and P out of TMEM, T = (I + A)^{-1}, W^T MMA, T diag(beta) into
//               the set.
//   X (role 2)  state chain: S^ from the master, the [U | O] MMA, U -> fp16, the master and O
//               MMAs; one thread per TMEM lane (value column).  Its MMA thread also issues
//               the TMA loads of q, k, g as soon as a set is free.
//   Y (role 3)  auxiliary: W^T out of TMEM into the set, U~ MMA, zeroing the O
//               accumulator, the output rows (16-byte stores after an in-register
//               transpose), and the TMA loads of v.
// GOUT (MODE_OUTPUT only): the gated or fp32 output path is compiled in; without it the
// kernel writes plain bf16 rows.
template <int MODE, typename TQ, bool GOUT>
__global__ void __launch_bounds__(NT, 1)
kda_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
              const __nv_bfloat16* __restrict__ beta, void* __restrict__ o, int o_f32,
              const float* __restrict__ S_in, int s_in_per_segment, float* __restrict__ maps,
              float* __restrict__ S_T, int B, int T, int H, int P, int L, int* status, int dbg_drop,
              const __nv_bfloat16* __restrict__ gate, const float* __restrict__ gamma, float eps,
              const int* __restrict__ items)
{
    using PL = Plan<MODE>;
    using TM = Tm<MODE>;
    constexpr bool OUT = MODE == MODE_OUTPUT;
    constexpr int T_LBO = PL::T_LBO;
    extern __shared__ __align__(1024) uint8_t sm[];

    const int t = threadIdx.x, w = t >> 5, lane = t & 31;
    const int q4 = w & 3;                     // TMEM lane quarter of this warp
    const int role = w >> 2;                  // P, I, X, Y
    const int rt = t & (NR - 1);              // thread index inside its role
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

    uint16_t* sBeta = reinterpret_cast<uint16_t*>(sm + PL::MISC + M_BETA);
    uint32_t* sBRaw = reinterpret_cast<uint32_t*>(sm + PL::MISC + M_BRAW);
    float* sTot = reinterpret_cast<float*>(sm + PL::MISC + M_TOT);
    float* sSC = reinterpret_cast<float*>(sm + PL::MISC + M_SC);
    int* sDirect = reinterpret_cast<int*>(sm + PL::MISC + M_DIRECT);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + PL::MISC + M_BAR);
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(sm + PL::MISC + M_TMEM);
    int* sAbort = reinterpret_cast<int*>(sm + PL::MISC + M_ABORT);
    const uint32_t sbase = smem_addr(sm);
    const Abort ab{sAbort, status};
    // beta arrives by 4-byte cp.async (the head pair's words) when that is aligned
    const bool beta_async = (H % 2 == 0) && ((reinterpret_cast<uintptr_t>(beta) & 3u) == 0);

    if (t == 0) {
        for (int i = 0; i < NBAR; ++i) mbar_init(&bars[i], 1);
        *sAbort = 0;
        fence_mbar_init();
    }
    if (w == 0) {
        tmem_alloc(sTmem, 512);
        tmem_relinquish();
    }
    // T tiles start zero (their upper blocks stay zero)
    for (int e = t; e < NSET * (PL::T_BYTES / 16); e += NT) {
        const int s = e / (PL::T_BYTES / 16), off = (e % (PL::T_BYTES / 16)) * 16;
        *reinterpret_cast<uint4*>(sm + s * PL::SET + PL::TF + off) = make_uint4(0u, 0u, 0u, 0u);
    }
    // beta of the first two chunks into their slots (later chunks: the prologue, two ahead)
    if (t < 2 * C) {
        const int x = t / C, i = t % C;
        sBeta[x * C + i] = beta_bits(beta, rowbase, Tq, H, h, (n0 + x) * C, i, x < nk);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *sTmem;
    const uint32_t tl = tmem + ((uint32_t)(32 * q4) << 16);   // this warp's lane quarter
    // TMA of chunk n's [64][128] tiles (packed rows rowbase + n*C ..; rows past the sequence
    // come from the next batch row or the zero fill and are masked where they are used)
    // q (MODE_OUTPUT), k and g of chunk n into the Q+ / beta K+ / K- tiles of its set
    auto tma_set = [&](int n) {
        const int s = set_of(n - n0), row = (int)(rowbase + n * C);
        uint8_t* set = sm + s * PL::SET;
        mbar_arrive_expect_tx(&bars[B_LD + s], PL::LOAD_BYTES);
        tma_load_3d(set + PL::KM, &tm_g, &bars[B_LD + s], 0, h, row);
        tma_load_3d(set + PL::KP, &tm_k, &bars[B_LD + s], 0, h, row);
        if (OUT) tma_load_3d(set + PL::QP, &tm_q, &bars[B_LD + s], 0, h, row);
    };
    auto tma_v = [&](int n) {   // v in core matrices: [value group][position][8 values]
        mbar_arrive_expect_tx(&bars[B_TV], 16384);
        tma_load_4d(sm + PL::VB, &tm_v, &bars[B_TV], 0, (int)(rowbase + n * C), 0, h);
    };
    const TQ* tq = nullptr;

    // ---- the first NSET chunks' q, k, g (the chain role's MMA thread issues every load of
    // them), and the initial state in TMEM, split over the four roles: 32 columns each of
    // the master (MODE_STATE: of N from 0 and of Phi from I), lane j = value column j -----
    if (t == 2 * NR)
        for (int x = 0; x < min(NSET, nk); ++x) tma_set(n0 + x);
    {
        const int j = 32 * q4 + lane, c0 = 32 * role;
        float vv[32];
        if (MODE == MODE_STATE) {
#pragma unroll
            for (int e = 0; e < 32; ++e) vv[e] = 0.f;
            tmem_st32(tl + TM::MASTER + c0, vv);
#pragma unroll
            for (int e = 0; e < 32; ++e) vv[e] = (c0 + e == j) ? 1.f : 0.f;
            tmem_st32(tl + TM::MASTER + D + c0, vv);
        } else {
            if (S_in) {
                const size_t idx = s_in_per_segment ? (size_t)slot : (size_t)seq * H + h;
                const float* src = S_in + idx * D * D + j;
#pragma unroll
                for (int e = 0; e < 32; ++e) vv[e] = src[(size_t)(c0 + e) * D];
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) vv[e] = 0.f;
            }
            tmem_st32(tl + TM::MASTER + c0, vv);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (role == 0) {
        // ================= P: prologue of chunk n0 + kc =====================================
        const int cp = rt & 63, rh = rt >> 6;   // channel pair, 32-row half
        float2 carry = make_float2(0.f, 0.f);   // rh == 0: carry of channels 2cp, 2cp+1
        for (int kc = 0; kc < nk; ++kc) {
            const int n = n0 + kc, t0 = n * C, s = set_of(kc);
            uint8_t* set = sm + s * PL::SET;
            const uint8_t* gst = set + PL::KM;                     // g as TMA landed it
            const uint16_t* sBk = sBeta + (kc % NBETA) * C;
            // beta of chunk kc+2 starts its way into shared memory (stored into its slot below)
            if (rt < C && beta_async) {
                const int tt = (n + 2) * C + rt;
                const bool live = n + 2 < n1 && tt < Tq;
                cp_async4_zfill(sBRaw + rt, beta + (((size_t)rowbase + (live ? tt : 0)) * H + (h & ~1)), live);
                cp_async_commit();
            }
            // ---- g of this chunk -> cumulative log-decay (base 2), references, range -----
            group_wait(&bars[B_LD + s], set_par(kc), ab, rt == 0, BAR_P);   // q, k, g landed
            const int nv = min(C, Tq - t0);   // rows of this chunk inside the sequence
            {
                const float2 l2e = make_float2(kLog2e, kLog2e);
                float2 tot = make_float2(0.f, 0.f);
#pragma unroll 8
                for (int r = 0; r < 32; ++r) {
                    const uint32_t gw = 32 * rh + r < nv ? *reinterpret_cast<const uint32_t*>(gst + (32 * rh + r) * 256 + 4 * cp) : 0u;
                    tot = __ffma2_rn(in2(gw, (const __nv_bfloat16*)nullptr), l2e, tot);
                }
                *reinterpret_cast<float2*>(sTot + rh * D + 2 * cp) = tot;
            }
            named_sync(BAR_P, NR);   // sTot published
            const float2 r2 = *reinterpret_cast<const float2*>(sTot + 2 * cp);            // b at row 31
            const float2 bC = __fadd2_rn(r2, *reinterpret_cast<const float2*>(sTot + D + 2 * cp));   // b at row 63
            const float2 pre = rh ? r2 : make_float2(0.f, 0.f);                          // b before my rows
            // the middle-row reference keeps a factor within 2^{max(b_0 - r, r - b_63)}
            bool wide = false;
            if (rh == 0) {
                const uint32_t g0 = nv > 0 ? *reinterpret_cast<const uint32_t*>(gst + 4 * cp) : 0u;
                const float2 b0 = __fmul2_rn(in2(g0, (const __nv_bfloat16*)nullptr), make_float2(kLog2e, kLog2e));
                wide = fmaxf(b0.x - r2.x, r2.x - bC.x) > kRangeMax || fmaxf(b0.y - r2.y, r2.y - bC.y) > kRangeMax;
            }
            const bool direct = bar_red_or(BAR_P, NR, wide);
            const float2 rp = direct ? make_float2(0.f, 0.f) : r2;   // reference of K+ and Q+
            const float2 rm = direct ? bC : r2;                      // reference of K-
            if (rh == 0) {
                // the chain's scales: S^ = 2^{rp + carry} master, master <- 2^{rm + carry} master
                float* sc = sSC + s * 3 * D;
                *reinterpret_cast<float2*>(sc + 2 * cp) = make_float2(ex2_approx(rp.x + carry.x), ex2_approx(rp.y + carry.y));
                *reinterpret_cast<float2*>(sc + D + 2 * cp) =
                    make_float2(ex2_approx(rm.x + carry.x), ex2_approx(rm.y + carry.y));
                carry = make_float2(bC.x - rm.x, bC.y - rm.y);
                *reinterpret_cast<float2*>(sc + 2 * D + 2 * cp) = carry;
            }
            if (rt == 0) sDirect[s] = direct ? 1 : 0;
            if (direct) {
                // A and P from pairwise exponentials; the log-decay table, one 64-channel half
                // at a time, goes over PF and TF in MODE_OUTPUT (free until the inverse role
                // fills them), else into the scratch region
                uint8_t* scr = OUT ? set + PL::PF : sm + Plan<MODE_STATE>::SCR;
                chunk_ap_direct<MODE, TQ>(set, scr, sTot, sBk, rt, nv);
            }
            // ---- beta K+, Q+ in place, K-; per 8-row block, the 64 threads of a row half read
            // their raw rows before any of them rewrites the block they share -----------------
            {
                const float2 l2e = make_float2(kLog2e, kLog2e);
                const float2 dlt = make_float2(rm.x - rp.x, rm.y - rp.y);
                float2 run = make_float2(pre.x - rp.x, pre.y - rp.y);   // b - rp
#pragma unroll 1
                for (int blk = 0; blk < 4; ++blk) {
                    const int rb = 32 * rh + 8 * blk;                     // first row of this block
                    uint32_t gR[8], kR[8], qR[8];
#pragma unroll
                    for (int r = 0; r < 8; ++r) {
                        const bool live = rb + r < nv;
                        gR[r] = live ? *reinterpret_cast<const uint32_t*>(gst + (rb + r) * 256 + 4 * cp) : 0u;
                        kR[r] = live ? *reinterpret_cast<const uint32_t*>(set + PL::KP + (rb + r) * 256 + 4 * cp) : 0u;
                        qR[r] = (OUT && live) ? *reinterpret_cast<const uint32_t*>(set + PL::QP + (rb + r) * 256 + 4 * cp) : 0u;
                    }
                    named_sync(BAR_P2 + rh, 64);
                    uint32_t pk[2][4], pm[2][4], pq[2][4];
                    float2 lk = make_float2(0.f, 0.f), lm = lk, lq = lk;
#pragma unroll
                    for (int r8 = 0; r8 < 8; ++r8) {
                        run = __ffma2_rn(in2(gR[r8], (const __nv_bfloat16*)nullptr), l2e, run);
                        const float2 kk = in2(kR[r8], tq);
                        const float bi = bf16_bits_to_f32(sBk[rb + r8]);
                        const float2 ep = make_float2(ex2_approx(run.x), ex2_approx(run.y));
                        const float2 em = make_float2(ex2_approx(dlt.x - run.x), ex2_approx(dlt.y - run.y));
                        const float2 kp = __fmul2_rn(__fmul2_rn(kk, make_float2(bi, bi)), ep);   // beta K+
                        const float2 km = __fmul2_rn(kk, em);                                   // K-
                        const float2 qp = OUT ? __fmul2_rn(in2(qR[r8], tq), ep) : make_float2(0.f, 0.f);
                        if (r8 & 1) {
                            const int m = r8 >> 1;
                            pk[0][m] = pack_f16x2(lk.x, kp.x); pk[1][m] = pack_f16x2(lk.y, kp.y);
                            pm[0][m] = pack_f16x2(lm.x, km.x); pm[1][m] = pack_f16x2(lm.y, km.y);
                            pq[0][m] = pack_f16x2(lq.x, qp.x); pq[1][m] = pack_f16x2(lq.y, qp.y);
                        } else {
                            lk = kp; lm = km; lq = qp;
                        }
                    }
                    const int ig = 4 * rh + blk;
                    st_pair(set + PL::KP, ig, cp, pk);
                    st_pair(set + PL::KM, ig, cp, pm);
                    if (OUT) st_pair(set + PL::QP, ig, cp, pq);
                }
            }
            // beta of chunk kc+2 into its slot (read by this role's prologue and by the inverse
            // role's T diag(beta); the slot's previous chunk is long done with)
            if (rt < C) {
                uint16_t bb;
                if (beta_async) {
                    cp_async_wait_all();
                    bb = (uint16_t)(sBRaw[rt] >> (16 * (h & 1)));
                } else {
                    bb = beta_bits(beta, rowbase, Tq, H, h, (n + 2) * C, rt, n + 2 < n1);
                }
                sBeta[((kc + 2) % NBETA) * C + rt] = bb;
            }
            fence_async_smem();
            tc_fence_before();
            named_sync(BAR_P, NR);
            if (rt == 0) {
                mbar_arrive(&bars[B_SC + s]);   // scales, direct flag, tiles (and beta) in place
                if (!direct) {
                    // A|P's TMEM columns are free once the output role has read chunk kc-1's W^T
                    if (kc > 0) thread_wait(&bars[B_APWF], (kc - 1) & 1, ab);
                    tc_fence_after();
                    // [beta K+; Q+] (M = 128) x K-^T: rows 0-63 give A, rows 64-127 give P (the
                    // state pass reads K- as rows 64-127 and ignores them)
                    const uint32_t id = idesc_f16(128, 64, true, true);
                    const uint32_t sset = sbase + s * PL::SET;
#pragma unroll 1
                    for (int kk = 0; kk < 8; ++kk)
                        umma_f16(tmem + TM_APW, sdesc(sset + PL::KP + 256 * kk, 128, 2048),
                                 sdesc(sset + PL::KM + 256 * kk, 128, 2048), id, kk > 0);
                    umma_commit(&bars[B_AP]);
                }
            }
        }
        if (beta_async) cp_async_wait_all();
    } else if (role == 1) {
        // ================= I: T and -W^T of chunk n0 + kc ===================================
        int n_ap = 0;
        for (int kc = 0; kc < nk; ++kc) {
            const int s = set_of(kc);
            uint8_t* set = sm + s * PL::SET;
            const uint32_t sset = sbase + s * PL::SET;
            group_wait(&bars[B_SC + s], set_par(kc), ab, rt == 0, BAR_I);   // the prologue is done
            if (!sDirect[s]) {
                // the prologue role issued the A|P MMA (once W^T of chunk kc-1 was read)
                group_wait(&bars[B_AP], n_ap & 1, ab, rt == 0, BAR_I);
                ++n_ap;
                // A (lanes 0-63) -> fp16 tile, P (lanes 64-127) -> the set's P tile
                if (OUT || q4 < 2) {
                    float v[64];
                    tmem_ld64(tl + TM_APW, v);
                    const bool isP = q4 >= 2;
                    const int i = 32 * (q4 & 1) + lane;
                    const int lim = i + (isP ? 1 : 0);        // A: columns < i; P: columns <= i
                    uint8_t* dst = set + (isP ? PL::PF : PL::TF) + cm64(i, 0);
#pragma unroll
                    for (int g8 = 0; g8 < 8; ++g8) {
                        float f[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j) f[j] = 8 * g8 + j < lim ? v[8 * g8 + j] : 0.f;
                        *reinterpret_cast<uint4*>(dst + g8 * 1024) = pack8_f16(f);
                    }
                }
                tc_fence_before();
                named_sync(BAR_I, NR);
            }
            invert_unit_lower<T_LBO>(sset + PL::TF, sbase + PL::MISC + M_XS, q4, lane, BAR_I);
            fence_async_smem();
            tc_fence_before();
            named_sync(BAR_I, NR);
            if (rt == 0) {
                tc_fence_after();
                // W^T = (beta K+)^T T^T: M = 128 channels, N = 64 positions, K = 64 positions
                const uint32_t id = idesc_f16(128, 64, false, false);
#pragma unroll 1
                for (int kk = 0; kk < 4; ++kk)
                    umma_f16(tmem + TM_APW, sdesc(sset + PL::KP + 4096 * kk, 2048, 128),
                             sdesc(sset + PL::TF + 2 * T_LBO * kk, T_LBO, 128), id, kk > 0);
                umma_commit(&bars[B_W]);
            }
            // W^T goes to the set's KP tile by the output role (which then signals PRO)
            group_wait(&bars[B_W], kc & 1, ab, rt == 0, BAR_I);
            {   // T -> T diag(beta) in the input type, in place (the W^T MMA has read T): the B
                // operand of U~^T = V^T (T diag(beta))^T, with V as it landed
                const uint16_t* sBk = sBeta + (kc % NBETA) * C;
#pragma unroll
                for (int e4 = 0; e4 < 4; ++e4) {
                    const int e = 4 * rt + e4;                       // 16-byte piece: 8 consecutive columns
                    const int j0 = 8 * (e >> 6);
                    uint4* pc = reinterpret_cast<uint4*>(set + PL::TF + 16 * e);
                    const uint4 u = *pc;
                    const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
                    uint32_t ow[4];
                    const uint4 bq = *reinterpret_cast<const uint4*>(sBk + j0);   // beta of columns j0 .. j0+7
                    const uint32_t bw[4] = {bq.x, bq.y, bq.z, bq.w};
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const float2 tb = __fmul2_rn(unpack_f16x2(uw[m]),
                                                     make_float2(__uint_as_float(bw[m] << 16), __uint_as_float(bw[m] & 0xffff0000u)));
                        ow[m] = pack2_in<TQ>(tb.x, tb.y);
                    }
                    *pc = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                }
            }
            fence_async_smem();
            tc_fence_before();
            named_sync(BAR_I, NR);
            if (rt == 0) mbar_arrive(&bars[B_INV + s]);   // T diag(beta) ready
        }
    } else if (role == 2) {
        // ================= X: the state chain of chunk n0 + kc ==============================
        const int j = 32 * q4 + lane;              // value column of this thread (TMEM lane)
        const bool mma = rt == 0;
        // rt 0 also issues the loads of q, k, g: chunk kc+2 into the set of chunk kc-1 once
        // the chain is done with it (the first NSET chunks' went out before the roles split)
        int ld_issued = mma ? min(NSET, nk) : 0;
        for (int kc = 0; kc < nk; ++kc) {
            const int s = set_of(kc), ub = kc & 1;   // buffer set; [U | O] buffer
            const uint32_t sset = sbase + s * PL::SET;
            // ---- S^ = fp16(2^{rp + carry} master), master <- 2^{rm + carry} master --------
            if (rt == 0) {
                thread_wait(&bars[B_SC + s], set_par(kc), ab);
                if (kc > 0) thread_wait(&bars[B_S], (kc - 1) & 1, ab);
            }
            named_sync(BAR_X, NR);
            tc_fence_after();
            // (MODE_STATE: the Phi half is rescaled by the output role beside this one)
            rescale_master(tl, TM::MASTER, TM::S16, sSC + s * 3 * D, sSC + s * 3 * D + D);
            tmem_wait_st();
            tc_fence_before();
            named_sync(BAR_X, NR);
            if (mma && kc >= 1 && kc + 2 < nk && !*sAbort) {
                // every MMA on chunk kc-1's set is done (its last commit follows the master update
                // that this role waited for above): chunk kc+2's q, k, g may land there
                thread_wait(&bars[B_EMPTY + set_of(kc - 1)], set_par(kc - 1), ab);
                if (!*sAbort) {
                    tma_set(n0 + kc + 2);
                    ld_issued = kc + 3;
                }
            }
            if (mma) {
                // U~ (Y) initialised the U columns; -W^T and Q+ are in the set (I)
                thread_wait(&bars[B_VE + (kc & 1)], (kc >> 1) & 1, ab);
                thread_wait(&bars[B_PRO + s], set_par(kc), ab);
                tc_fence_after();
                if (OUT) {
                    // [U | -O]^T += -S^T [W^T | Q+^T]   (N = 128: positions of W, then of Q+); the
                    // O columns accumulate -O, negated back when written out
                    const uint32_t id = idesc_f16(128, 128, false, true, true);
#pragma unroll 1
                    for (int kk = 0; kk < 8; ++kk)
                        umma_f16_ts(tmem + TM::UO + 128 * ub, tmem + TM::S16 + 8 * kk,
                                    sdesc(sset + PL::KP + 256 * kk, 128, 2048), id, 1);
                } else {
                    const uint32_t id = idesc_f16(128, 64, false, true, true);   // U^T += -S^T W^T
#pragma unroll 1
                    for (int kk = 0; kk < 8; ++kk)
                        umma_f16_ts(tmem + TM::UACC, tmem + TM::S16 + 8 * kk,
                                    sdesc(sset + PL::KP + 256 * kk, 128, 2048), id, 1);
                }
                umma_commit(&bars[B_U]);
            }
            group_wait(&bars[B_U], kc & 1, ab, rt == 0, BAR_X);
            // ---- U -> fp16 (A operand of the master and O updates); one thread owns its lane,
            // so it may overwrite the columns it has just read ------------------------------------
            {
                const uint32_t usrc = OUT ? TM::UO + 128 * ub : TM::UACC;
                const uint32_t udst = OUT ? TM::UO + 128 * ub : TM::S16;   // MODE_STATE: into S^'s columns
                float vv[64];
                uint32_t hv[32];
                tmem_ld64(tl + usrc, vv);
#pragma unroll
                for (int e = 0; e < 32; ++e) hv[e] = pack_f16x2(vv[2 * e], vv[2 * e + 1]);
                tmem_st32u_nowait(tl + udst, hv);
                tmem_wait_st();
            }
            tc_fence_before();
            named_sync(BAR_X, NR);
            if (mma) {
                tc_fence_after();
                const uint32_t idm = idesc_f16(128, 128, false, false);
                if (OUT) {
                    // master += U^T K-   and   -O^T += -U^T P^T
                    const uint32_t ua = tmem + TM::UO + 128 * ub;
#pragma unroll 1
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16_ts(tmem + TM::MASTER, ua + 8 * kk, sdesc(sset + PL::KM + 4096 * kk, 2048, 128), idm, 1);
                    umma_commit(&bars[B_S]);
                    const uint32_t ido = idesc_f16(128, 64, false, false, true);
#pragma unroll 1
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16_ts(ua + 64, ua + 8 * kk, sdesc(sset + PL::PF + 2048 * kk, 1024, 128), ido, 1);
                    umma_commit(&bars[B_O + ub]);
                } else {
                    // S chain: master_N += U_N^T K-; Phi chain: U_Phi^T = -Phi^T W^T (fresh), once
                    // the output role has rescaled the Phi half
#pragma unroll 1
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16_ts(tmem + TM::MASTER, tmem + TM::S16 + 8 * kk,
                                    sdesc(sset + PL::KM + 4096 * kk, 2048, 128), idm, 1);
                    thread_wait(&bars[B_C1Y], kc & 1, ab);
                    tc_fence_after();
                    const uint32_t id = idesc_f16(128, 64, false, true, true);
#pragma unroll 1
                    for (int kk = 0; kk < 8; ++kk)
                        umma_f16_ts(tmem + TM::UACC, tmem + TM::S16 + 64 + 8 * kk,
                                    sdesc(sset + PL::KP + 256 * kk, 128, 2048), id, kk > 0);
                    umma_commit(&bars[B_U2]);
                }
            }
            if (!OUT) {
                group_wait(&bars[B_U2], kc & 1, ab, rt == 0, BAR_X);
                {
                    float vv[64];
                    uint32_t hv[32];
                    tmem_ld64(tl + TM::UACC, vv);
#pragma unroll
                    for (int e = 0; e < 32; ++e) hv[e] = pack_f16x2(vv[2 * e], vv[2 * e + 1]);
                    tmem_st32u_nowait(tl + TM::S16 + 64, hv);
                    tmem_wait_st();
                }
                tc_fence_before();
                named_sync(BAR_X, NR);
                if (mma) {
                    tc_fence_after();
                    const uint32_t idm = idesc_f16(128, 128, false, false);
#pragma unroll 1
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16_ts(tmem + TM::MASTER + D, tmem + TM::S16 + 64 + 8 * kk,
                                    sdesc(sset + PL::KM + 4096 * kk, 2048, 128), idm, 1);
                    umma_commit(&bars[B_S]);
                }
            }
            if (mma) umma_commit(&bars[B_EMPTY + s]);   // set s may be refilled
        }
        // ---- end of segment: the state S = diag(2^{carry}) master (columns = channels) -----
        if (nk > 0) group_wait(&bars[B_S], (nk - 1) & 1, ab, rt == 0, BAR_X);
        // after a timeout some requested tiles may not have been waited for: let them land
        if (mma && *sAbort)
            for (int x = max(0, ld_issued - NSET); x < ld_issued; ++x)
                mbar_wait_bounded(&bars[B_LD + set_of(x)], set_par(x), kWaitNs);
        float* dst = nullptr;
        if (MODE == MODE_STATE) dst = maps + (size_t)slot * 2 * D * D;  // [N | M]
        else if (S_T && last) dst = S_T + ((size_t)seq * H + h) * D * D;
        if (dst && !*sAbort) {
            const float* cn = nk > 0 ? sSC + set_of(nk - 1) * 3 * D + 2 * D : nullptr;
            for (int mi = 0; mi < (OUT ? 1 : 2); ++mi) {
                for (int c0 = 0; c0 < D; c0 += 32) {
                    float vv[32];
                    tmem_ld32(tl + TM::MASTER + D * mi + c0, vv);
                    float* d = dst + (size_t)mi * D * D + j;
#pragma unroll
                    for (int e = 0; e < 32; ++e) d[(size_t)(c0 + e) * D] = vv[e] * (cn ? ex2_approx(cn[c0 + e]) : 1.f);
                }
            }
        }
    } else {
        // ================= Y: U~, the output rows, the loads =================================
        const int j = 32 * q4 + lane;              // value column of this thread (TMEM lane)
        const bool mma = rt == 0, loader = rt == 32;
        int v_issued = 0;                          // loader: chunks whose v was requested
        if (loader && nk > 0) {
            tma_v(n0);
            v_issued = 1;
        }
        float gam = 1.f;
        if (OUT && gate && gamma) gam = gamma[(size_t)h * D + j];
        // zero the O columns of [U | O] buffer x (U~ writes only the U columns)
        auto zero_o = [&](int x) {
            if (!OUT) return;
            float z[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) z[e] = 0.f;
            tmem_st32(tl + TM::UO + 128 * (x & 1) + 64, z);
            tmem_st32(tl + TM::UO + 128 * (x & 1) + 96, z);
        };
        // U~^T = V^T (T diag(beta))^T into the chunk's U columns: V^T straight from the v tile
        // (M = values, MN-major core matrices), operands in the input type
        auto issue_u = [&](int x) {
            const uint32_t sset = sbase + set_of(x) * PL::SET, vbt = sbase + PL::VB;
            const uint32_t id = idesc_f16(128, 64, true, false, false, std::is_same<TQ, __nv_bfloat16>::value);
            const uint32_t d = tmem + (OUT ? TM::UO + 128 * (x & 1) : TM::UACC);
#pragma unroll 1
            for (int kk = 0; kk < 4; ++kk)
                umma_f16(d, sdesc(vbt + 256 * kk, 128, 1024), sdesc(sset + PL::TF + 2 * T_LBO * kk, T_LBO, 128), id,
                         kk > 0);
            umma_commit(&bars[B_VE + (x & 1)]);   // U~ done: the v tile may be refilled
        };
        // chunk x's output rows: O^T (lane j, columns 64 + i of its [U | O] buffer) -> o
        auto out_rows = [&](int x) {
            const int b = x & 1, t0x = (n0 + x) * C;
            group_wait(&bars[B_O + b], (x >> 1) & 1, ab, rt == 0, BAR_Y);
            const int nvx = min(C, Tq - t0x);
            const uint32_t ocol = tl + TM::UO + 128 * b + 64;
            if constexpr (GOUT) {
                const OutParams op{gate, o, reinterpret_cast<float*>(sm + PL::MISC + M_RED), gam, eps, o_f32, H, h, q4, lane,
                                   rowbase + Tq};
                out_rows_general(&op, ocol, rowbase + t0x, nvx);
                return;
            }
#pragma unroll 1
            for (int hp = 0; hp < 2; ++hp) {
                float v[32];
                tmem_ld32(ocol + 32 * hp, v);
                store_rows_bf16(v, reinterpret_cast<__nv_bfloat16*>(o), rowbase + t0x, 32 * hp, nvx, H, h, q4, lane);
            }
        };
        zero_o(0);
        if (nk > 1) zero_o(1);
        tc_fence_before();
        named_sync(BAR_Y, NR);   // the zeroed O columns are in place
        tc_fence_after();
        bool u_done = false;     // rt 0: U~ of chunk kc already issued
        for (int kc = 0; kc < nk; ++kc) {
            const int n = n0 + kc, s = set_of(kc);
            // ---- W^T of chunk kc (TMEM, channel c in lane c) -> the set's KP tile ----------------
            group_wait(&bars[B_W], kc & 1, ab, rt == 0, BAR_Y);
            {
                uint8_t* kp = sm + s * PL::SET + PL::KP + (j >> 3) * 128 + (j & 7) * 16;
#pragma unroll 1
                for (int hw = 0; hw < 2; ++hw) {
                    float v[32];
                    tmem_ld32(tl + TM_APW + 32 * hw, v);
#pragma unroll
                    for (int g8 = 0; g8 < 4; ++g8)
                        *reinterpret_cast<uint4*>(kp + (4 * hw + g8) * 2048) = pack8_f16(v + 8 * g8);
                }
            }
            fence_async_smem();
            tc_fence_before();
            named_sync(BAR_Y, NR);
            if (rt == 0) {
                mbar_arrive(&bars[B_APWF]);   // A|P's TMEM columns may be reused
                // every tile of the set is ready (the test hook withholds chunk 0's signal)
                if (!(dbg_drop && kc == 0)) mbar_arrive(&bars[B_PRO + s]);
            }
            if constexpr (!OUT) {
                // ---- the Phi half of the master at the start of chunk kc (beside the chain role's
                // S half): after the chain's last master update of chunk kc-1 --------------------
                if (rt == 0) {
                    thread_wait(&bars[B_SC + s], set_par(kc), ab);
                    if (kc > 0) thread_wait(&bars[B_S], (kc - 1) & 1, ab);
                }
                named_sync(BAR_Y, NR);
                tc_fence_after();
                rescale_master(tl, TM::MASTER + D, TM::S16 + 64, sSC + s * 3 * D, sSC + s * 3 * D + D);
                tmem_wait_st();
                tc_fence_before();
                named_sync(BAR_Y, NR);
                if (rt == 0) mbar_arrive(&bars[B_C1Y]);
            }
            if (mma && !u_done) {
                thread_wait(&bars[B_INV + s], set_par(kc), ab);
                thread_wait(&bars[B_TV], kc & 1, ab);   // this chunk's v has landed
                // MODE_STATE: one U accumulator; the chain of chunk kc-1 has read it once its
                // last master update is done
                if (!OUT && kc > 0) thread_wait(&bars[B_S], (kc - 1) & 1, ab);
                tc_fence_after();
                issue_u(kc);
            }
            // the v tile is free once U~ of chunk kc is done: chunk kc+1's may land
            if (loader && kc + 1 < nk && !*sAbort) {
                thread_wait(&bars[B_VE + (kc & 1)], (kc >> 1) & 1, ab);
                if (!*sAbort) {
                    tma_v(n + 1);
                    v_issued = kc + 2;
                }
            }
            // ---- chunk kc-1's output rows, then its O columns are zeroed for chunk kc+1 -------
            if (OUT && kc > 0) {
                out_rows(kc - 1);
                if (kc + 1 < nk) zero_o(kc + 1);
            }
            tc_fence_before();
            named_sync(BAR_Y, NR);
            // U~ of the next chunk now, if its T and v are ready (else at the top of the next step)
            if (mma) {
                u_done = false;
                if (OUT && kc + 1 < nk && !*sAbort && mbar_try_wait(&bars[B_INV + set_of(kc + 1)], set_par(kc + 1)) &&
                    mbar_try_wait(&bars[B_TV], (kc + 1) & 1)) {
                    tc_fence_after();
                    issue_u(kc + 1);
                    u_done = true;
                }
            }
        }
        if (OUT && nk > 0) out_rows(nk - 1);
        // after a timeout some requested tiles may not have been waited for: let them land
        if (loader && *sAbort && v_issued > 0) mbar_wait_bounded(&bars[B_TV], (v_issued - 1) & 1, kWaitNs);
    }
    // ---- teardown: after a timeout, each MMA issuer drains its own MMAs; free TMEM --------
    if (*sAbort && (t == 0 || t == NR || t == 2 * NR || t == 3 * NR)) {
        uint64_t* dr = &bars[B_DRAIN + role];
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
// threads in two halves that split each product's k sum (k < 64 and k >= 64), so every
// SM partition runs one warp of each.  Thread t of a half owns column quad t%4 of the
// CTA's 16 state columns on rows t/4 + 32i (i = 0..3): one 16-byte read of M (four k of a
// row) and one of S (four columns of a k) feed 8 packed multiply-adds.  The second half
// hands its partial sums to the first through shared memory.  Three shared buffers hold
// M_p, M_{p+1}, M_{p+2}: the cp.async of M_{p+2} is issued as step p starts.
constexpr int CB_THREADS = 256;
constexpr int CB_LD = 132;      // row stride in floats (16-byte rows for cp.async)
constexpr int CB_NBUF = 3;
constexpr int cb_smem_bytes() { return (CB_NBUF * D * CB_LD + D * 16 + 4 * 128 * 4) * (int)sizeof(float); }

// One commit group per map, empty past the last one, so group p always holds M_p.
__device__ __forceinline__ void cb_stage(float* dst, const float* M, int t, bool any)
{
    if (any) {
#pragma unroll
        for (int u = 0; u < D * D / 4 / CB_THREADS; ++u) {
            const int i = t + u * CB_THREADS, row = i >> 5, col = (i & 31) * 4;
            cp_async16(dst + row * CB_LD + col, M + (size_t)row * D + col);
        }
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
    float* sS = csm + CB_NBUF * D * CB_LD;   // [128][16] the state columns S_start(p)
    float4* sR = reinterpret_cast<float4*>(sS + D * 16);   // [4][128] the second half's sums
    const int t = threadIdx.x;
    const int half = t >> 7, tt = t & 127;
    const int rg = tt >> 2, c4 = (tt & 3) * 4;        // rows rg + 32 i, columns c4 .. c4+3
    const int col = blockIdx.x * 16 + c4;
    const int bh = blockIdx.z * H + blockIdx.y;
    size_t map0 = (size_t)bh * (P - 1), start0 = (size_t)bh * P;
    if (seqinfo) {
        P = seqinfo[3 * blockIdx.z];
        map0 = (size_t)seqinfo[3 * blockIdx.z + 1] + (size_t)blockIdx.y * (P > 0 ? P - 1 : 0);
        start0 = (size_t)seqinfo[3 * blockIdx.z + 2] + (size_t)blockIdx.y * P;
        if (P == 0) return;
    }
    const float* mp = maps + map0 * 2 * D * D;   // [P-1][N | M]
    auto map_m = [&](int p) { return mp + (size_t)p * 2 * D * D + D * D; };
    cb_stage(csm, mp + D * D, t, P > 1);
    cb_stage(csm + D * CB_LD, P > 2 ? map_m(1) : mp, t, P > 2);
    // the first half holds the state (s) and N_p one step ahead (nxt)
    float4 s[4], nxt[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {   // the caller's S0 need not be 16-byte aligned
        const float* s0 = S0 + ((size_t)bh * D + rg + 32 * i) * D + col;
        s[i] = S0 && half == 0 ? make_float4(s0[0], s0[1], s0[2], s0[3]) : make_float4(0.f, 0.f, 0.f, 0.f);
        nxt[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    auto load_n = [&](int p) {
        if (half != 0) return;
#pragma unroll
        for (int i = 0; i < 4; ++i)
            nxt[i] = *reinterpret_cast<const float4*>(mp + (size_t)p * 2 * D * D + (size_t)(rg + 32 * i) * D + col);
    };
    if (P > 1) load_n(0);
    for (int p = 0; p < P; ++p) {
        if (half == 0) {
            float* out = starts + (start0 + p) * D * D + col;
#pragma unroll
            for (int i = 0; i < 4; ++i) *reinterpret_cast<float4*>(out + (size_t)(rg + 32 * i) * D) = s[i];
        }
        if (p == P - 1) break;
        float2 a2[4][2];   // packed fp32 FMAs: row i, column pairs (c4, c4+1) and (c4+2, c4+3)
#pragma unroll
        for (int i = 0; i < 4; ++i) {   // zero in the second half
            a2[i][0] = make_float2(nxt[i].x, nxt[i].y);
            a2[i][1] = make_float2(nxt[i].z, nxt[i].w);
        }
        if (p + 1 < P - 1) load_n(p + 1);        // in flight during this step
        __syncthreads();                         // sS, sR and the buffer of M_{p-1} are free
        if (half == 0) {
#pragma unroll
            for (int i = 0; i < 4; ++i) *reinterpret_cast<float4*>(sS + (rg + 32 * i) * 16 + c4) = s[i];
        }
        cb_stage(csm + ((p + 2) % CB_NBUF) * D * CB_LD, p + 2 < P - 1 ? map_m(p + 2) : mp, t, p + 2 < P - 1);
        asm volatile("cp.async.wait_group 2;" ::: "memory");   // groups 0..p done: M_p landed
        __syncthreads();                         // M_p staged, sS written
        const float* sM = csm + (p % CB_NBUF) * D * CB_LD;
        const int kq0 = half * (D / 8);
#pragma unroll 2
        for (int k4 = kq0; k4 < kq0 + D / 8; ++k4) {
            float4 m[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) m[i] = *reinterpret_cast<const float4*>(sM + (rg + 32 * i) * CB_LD + 4 * k4);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float4 sv = *reinterpret_cast<const float4*>(sS + (4 * k4 + u) * 16 + c4);
                const float2 lo = make_float2(sv.x, sv.y), hi = make_float2(sv.z, sv.w);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float mk = u == 0 ? m[i].x : u == 1 ? m[i].y : u == 2 ? m[i].z : m[i].w;
                    const float2 mm = make_float2(mk, mk);
                    a2[i][0] = __ffma2_rn(mm, lo, a2[i][0]);
                    a2[i][1] = __ffma2_rn(mm, hi, a2[i][1]);
                }
            }
        }
        if (half == 1) {
#pragma unroll
            for (int i = 0; i < 4; ++i) sR[i * 128 + tt] = make_float4(a2[i][0].x, a2[i][0].y, a2[i][1].x, a2[i][1].y);
        }
        __syncthreads();                         // the second half's sums are in sR
        if (half == 0) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float4 r = sR[i * 128 + tt];
                s[i] = make_float4(a2[i][0].x + r.x, a2[i][0].y + r.y, a2[i][1].x + r.z, a2[i][1].y + r.w);
            }
        }
    }
}

// The work items of the two-wave split of a uniform batch, built on the device (so a call
// makes no host-to-device copy and can be captured in a CUDA graph).  One thread per
// (b, h, segment p): p = 0 -> it0 (segment 0's output pass; slot = b*H + h, last = 1);
// p >= 1 -> ito (output pass, slot (b*H + h)*(P-1) + p-1) and, for p <= P-2, its (state
// pass, slot (b*H + h)*(P-2) + p-1).  Items are {row, length, n0, n1, head, sequence,
// slot, last}.
__global__ void wave_items_kernel(int* __restrict__ it0, int* __restrict__ its, int* __restrict__ ito, int B, int T,
                                  int H, int P, int L0, int L)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= B * H * P) return;
    const int p = i % P, bh = i / P, b = bh / H, h = bh % H;
    // segment 0: chunks [0, L0); segment p >= 1: L chunks from L0 + (p-1) L (the last may be shorter)
    const int NC = (T + C - 1) / C, n0 = p == 0 ? 0 : L0 + (p - 1) * L, n1 = min(NC, p == 0 ? L0 : n0 + L);
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

// v [B*T, H, 128] as 4-D (8 values, tokens, 16 value groups, heads), box 8 x 64 x 16 x 1:
// a chunk lands as [value group][position][8 values], the MN-major core-matrix layout of
// the A operand V^T (values = M, positions = K) of the U~ MMA.
bool make_map_v(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int B, int T, int H)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[4] = {8u, (cuuint64_t)B * (cuuint64_t)T, (cuuint64_t)(D / 8), (cuuint64_t)H};
    const cuuint64_t strides[3] = {(cuuint64_t)H * D * 2, 16u, (cuuint64_t)D * 2};
    const cuuint32_t box[4] = {8u, (cuuint32_t)C, (cuuint32_t)(D / 8), 1u};
    const cuuint32_t es[4] = {1u, 1u, 1u, 1u};
    return fn(m, dt, 4, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct Maps {
    CUtensorMap q, k, v, g;
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
    const bool gout = MODE == MODE_OUTPUT && (a.gate != nullptr || a.out_t == ET_F32);
    auto kern = gout ? kda_tc_kernel<MODE, TQ, MODE == MODE_OUTPUT> : kda_tc_kernel<MODE, TQ, false>;
    const int smem = smem_bytes<MODE>();
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int nseg = MODE == MODE_STATE ? P - 1 : P;
    const unsigned grid = items ? (unsigned)nitems : (unsigned)(a.B * a.H * nseg);
    if (grid == 0) return cudaSuccess;
    ProfileScope prof(prof_name ? prof_name : (MODE == MODE_STATE ? "kda_tc_state" : "kda_tc_output"), s);
    count_launch();
    kern<<<grid, NT, smem, s>>>(mp.q, mp.k, mp.v, mp.g, (const __nv_bfloat16*)a.beta, a.o, a.out_t == ET_F32 ? 1 : 0,
                                S_in, per_seg, maps, a.ST, a.B, a.T, a.H, P, L, status, debug_drop_handoff(),
                                (const __nv_bfloat16*)a.gate, a.gamma, a.eps, items);
    return cudaGetLastError();
}

template <typename TQ>
bool build_maps(const KdaArgs& a, Maps& mp)
{
    const CUtensorMapDataType dq =
        std::is_same<TQ, __half>::value ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    if (!make_map(&mp.q, a.q, dq, a.B, a.T, a.H) || !make_map(&mp.k, a.k, dq, a.B, a.T, a.H) ||
        !make_map_v(&mp.v, a.v, dq, a.B, a.T, a.H) ||
        !make_map(&mp.g, a.g, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.B, a.T, a.H))
        return false;
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
    int P, L0, L;   // segments; chunks of segment 0; chunks of each later one (the last may be shorter)
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
        w.L0 = w.L = NC;
        return w;
    }
    int P = min(W + 1, NC);
    w.L = (NC + P - 1) / P;
    w.P = P = (NC + w.L - 1) / w.L;   // no empty segment
    w.L0 = w.L;
    if (P >= 3) {
        // Wave 1 runs segment 0's output pass beside the state pass of segments 1..P-2,
        // whose chunks cost ~4% more (measured: 4.39-4.64 against 4.23-4.40 us), so when
        // that shortens the later segments, they take L = ceil(NC / (P - 1 + 1.04)) chunks
        // each and segment 0 the rest (between L and 1.04 L).
        const int L = (25 * NC + 25 * (P - 1) + 25) / (25 * (P - 1) + 26);
        if (L < w.L) {
            w.L0 = NC - (P - 1) * L;
            w.L = L;
        }
    }
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
    if (wv.P == 1) {
        float* maps = reinterpret_cast<float*>(ws);
        float* starts = maps + (size_t)a.B * a.H * (sp.P - 1) * 2 * D * D;
        if (sp.P > 1) {
            const cudaError_t e = launch_pass<MODE_STATE, TQ>(mp, a, nullptr, 0, maps, sp.P, sp.L, status, s);
            if (e != cudaSuccess) return e;
        }
        return combine_output<TQ>(mp, a, sp, maps, starts, status, s);
    }
    const int P = wv.P, L = wv.L, BH = a.B * a.H;
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
        wave_items_kernel<<<(n + 255) / 256, 256, 0, s>>>(it0, its, ito, a.B, a.T, a.H, P, wv.L0, L);
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
        !make_map_v(&mp.v, a.v, dq, 1, a.T, a.H) || !make_map(&mp.g, a.g, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 1, a.T, a.H))
        return cudaErrorInvalidValue;
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
    if (a.gate && a.in_t != ET_BF16) return false;
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
    // the output side of Eq. 15 (a.gate) is applied in the output pass's store stage
    return a.in_t == ET_F16 ? launch_all<__half>(a, ws, status, s) : launch_all<__nv_bfloat16>(a, ws, status, s);
}

}  // namespace kda
