// Sequence-parallel forward scan: each row of the stream is cut along time into R
// consecutive shards, one per device.
//
// Eq. 14 of the Chimera paper (section 3.3) is affine in the state.  Over any run of
// tokens S_out = M S_in + N, where M = prod_t (I - beta_t k_t k_t^T) Diag(alpha_t)
// (latest token leftmost) and N is the state the run reaches from S_in = 0.  A row cut
// into shards is scanned in four steps:
//   1. every rank: (M_r, N_r) of its own shard                          kda_sp_transition
//   2. all ranks:  exchange the maps (one all-gather, in the Python layer)
//   3. rank r:     S_in(r) = the maps of shards 0..r-1 folded over S0    kda_sp_prefix
//   4. rank r:     the scan of its shard from S_in(r): o and S_T         kda_sp_output
// On the tensor-core path step 1 is the scan's own state pass over every segment of
// the shard plus a fold of the segment maps, and step 4 reuses those segment maps from
// the workspace.  A shard then costs one state pass, one output pass and two small folds.
// The CUDA-core path gets N_r from a scan from zero and M_r from a scan of v = 0 from
// S0 = I, and step 4 is a plain scan from S_in(r).

#include "internal.h"
#include "sm100.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int FOLD_THREADS = 256;
constexpr int FOLD_COLS = 32;   // state / M columns per CTA: 16 per thread, two threads per row

// X <- M_j X + [N_j | 0] for j = 0..J-1, from X = [S0 (or 0) | I], per head (blockIdx.y),
// in fp32.  Each CTA owns 32 columns (blockIdx.x): blocks below DK/32 hold state columns,
// the others (when the grid has 2*DK/32 of them) columns of the accumulated M.  The map
// of step j of head bh sits at maps + (j*sj + bh*sbh) * 2*DK*DK floats as [N | M]; with
// `tail` set, the last step's map is at tail + bh*2*DK*DK instead.  The final X goes to
// out + bh*out_stride (state columns) and out + bh*out_stride + DK*DK (M columns).
// M_{j+1} streams into the second shared buffer (cp.async) while step j computes, and a
// thread's 16 values of N_{j+1} are loaded one step ahead.
template <int DK>
__global__ void __launch_bounds__(FOLD_THREADS)
sp_fold_kernel(const float* __restrict__ maps, int64_t sj, int64_t sbh, const float* __restrict__ tail, int J,
               const float* __restrict__ S0, float* __restrict__ out, int64_t out_stride)
{
    constexpr int LD = DK + 4;          // 16-byte rows, conflict-free float4 reads across rows
    constexpr int64_t DD = (int64_t)DK * DK;
    constexpr int CB = DK / FOLD_COLS;  // column blocks of one D x D matrix
    extern __shared__ __align__(16) float fsm[];
    float* sX = fsm + 2 * DK * LD;      // this CTA's columns of X, [DK][32]
    const int t = threadIdx.x, r = t >> 1, c16 = (t & 1) * 16;
    const bool live = r < DK;
    const int64_t bh = blockIdx.y;
    const bool mcol = (int)blockIdx.x >= CB;
    const int col0 = ((int)blockIdx.x - (mcol ? CB : 0)) * FOLD_COLS + c16;
    auto map_of = [&](int s) -> const float* {
        return (tail && s == J - 1) ? tail + bh * 2 * DD : maps + (s * sj + bh * sbh) * 2 * DD;
    };
    auto stage = [&](float* dst, const float* M) {
        for (int i = t; i < DK * DK / 4; i += FOLD_THREADS) {
            const int row = i / (DK / 4), c4 = (i % (DK / 4)) * 4;
            cp_async16(dst + row * LD + c4, M + (int64_t)row * DK + c4);
        }
        cp_async_commit();
    };
    float x[16], nxt[16];
    auto load_n = [&](int s) {
        if (mcol || !live) {
#pragma unroll
            for (int j = 0; j < 16; ++j) nxt[j] = 0.f;
            return;
        }
        const float4* n4 = reinterpret_cast<const float4*>(map_of(s) + (int64_t)r * DK + col0);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 v = n4[q];
            nxt[4 * q] = v.x; nxt[4 * q + 1] = v.y; nxt[4 * q + 2] = v.z; nxt[4 * q + 3] = v.w;
        }
    };
#pragma unroll
    for (int j = 0; j < 16; ++j)
        x[j] = !live ? 0.f
             : mcol  ? (r == col0 + j ? 1.f : 0.f)
                     : (S0 ? S0[bh * DD + (int64_t)r * DK + col0 + j] : 0.f);
    if (J > 0) {
        stage(fsm, map_of(0) + DD);
        load_n(0);
    }
    for (int s = 0; s < J; ++s) {
        float acc[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) acc[j] = nxt[j];
        if (s + 1 < J) load_n(s + 1);   // in flight during this step
        __syncthreads();                // sX and the other M buffer are free
        if (live) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
                *reinterpret_cast<float4*>(sX + r * FOLD_COLS + c16 + 4 * q) =
                    make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
        }
        if (s + 1 < J) {
            stage(fsm + ((s + 1) & 1) * DK * LD, map_of(s + 1) + DD);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            cp_async_wait_all();
        }
        __syncthreads();                // M_s staged, sX written
        if (live) {
            const float* sM = fsm + (s & 1) * DK * LD + r * LD;
#pragma unroll 2
            for (int k4 = 0; k4 < DK / 4; ++k4) {
                const float4 m = *reinterpret_cast<const float4*>(sM + 4 * k4);
                const float mk[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float* xr = sX + (4 * k4 + u) * FOLD_COLS + c16;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float4 xv = *reinterpret_cast<const float4*>(xr + 4 * q);
                        acc[4 * q] = fmaf(mk[u], xv.x, acc[4 * q]);
                        acc[4 * q + 1] = fmaf(mk[u], xv.y, acc[4 * q + 1]);
                        acc[4 * q + 2] = fmaf(mk[u], xv.z, acc[4 * q + 2]);
                        acc[4 * q + 3] = fmaf(mk[u], xv.w, acc[4 * q + 3]);
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) x[j] = acc[j];
        }
    }
    if (live) {
        float4* o = reinterpret_cast<float4*>(out + bh * out_stride + (mcol ? DD : 0) + (int64_t)r * DK + col0);
#pragma unroll
        for (int q = 0; q < 4; ++q) o[q] = make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
    }
}

template <int DK>
cudaError_t fold_t(const float* maps, int64_t sj, int64_t sbh, const float* tail, int J, const float* S0,
                   float* out, int64_t out_stride, int BH, bool with_m, cudaStream_t s)
{
    const int smem = (2 * DK * (DK + 4) + DK * FOLD_COLS) * (int)sizeof(float);
    auto kern = sp_fold_kernel<DK>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    ProfileScope prof("kda_sp_fold", s);
    count_launch();
    kern<<<dim3((with_m ? 2 : 1) * DK / FOLD_COLS, BH), FOLD_THREADS, smem, s>>>(maps, sj, sbh, tail, J, S0, out,
                                                                          out_stride);
    return cudaGetLastError();
}

cudaError_t fold(int D, const float* maps, int64_t sj, int64_t sbh, const float* tail, int J, const float* S0,
                 float* out, int64_t out_stride, int BH, bool with_m, cudaStream_t s)
{
    switch (D) {
        case 32: return fold_t<32>(maps, sj, sbh, tail, J, S0, out, out_stride, BH, with_m, s);
        case 64: return fold_t<64>(maps, sj, sbh, tail, J, S0, out, out_stride, BH, with_m, s);
        case 128: return fold_t<128>(maps, sj, sbh, tail, J, S0, out, out_stride, BH, with_m, s);
    }
    return cudaErrorInvalidValue;
}

__global__ void eye_kernel(float* S, int D, int64_t n)
{
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t e = i % ((int64_t)D * D);
        S[i] = (e / D == e % D) ? 1.f : 0.f;
    }
}

bool dim_ok(int d) { return d == 32 || d == 64 || d == 128; }
int num_sms()
{
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}
size_t al256(size_t x) { return (x + 255) & ~size_t(255); }
ElemType et_of(kda_dtype d) { return d == KDA_F32 ? ET_F32 : ET_BF16; }

// The shard's scan arguments, no output attached.  Both the transition and the output
// call take the tensor-core route exactly when this does, so the segment maps that the
// first leaves in the workspace are the ones the second reads.
KdaArgs shard_args(const void* q, const void* k, const void* v, const void* g, const void* beta, int B, int T,
                   int H, int D, kda_dtype dtype, int chunk)
{
    return KdaArgs{q, k, v, g, beta, nullptr, nullptr, nullptr, B, T, H, D, D,
                   chunk ? chunk : (dtype == KDA_F32 ? 16 : 64), et_of(dtype), et_of(dtype), et_of(dtype)};
}

// Generic route: o scratch (fp32), v = 0, S0 = I, S_T scratch.
struct GenericWs {
    size_t o, vz, eye, st, total;
};
GenericWs generic_ws(int B, int T, int H, int D, kda_dtype dtype)
{
    const size_t tok = (size_t)B * T * H * D, st = (size_t)B * H * D * D * sizeof(float);
    GenericWs w;
    w.o = 0;
    w.vz = al256(tok * sizeof(float));
    w.eye = w.vz + al256(tok * (dtype == KDA_F32 ? 4 : 2));
    w.st = w.eye + al256(st);
    w.total = w.st + al256(st);
    return w;
}

bool shard_ok(int B, int T, int H, int D, kda_dtype dtype, int chunk)
{
    if (B < 0 || T < 0 || H <= 0 || !dim_ok(D)) return false;
    if (dtype != KDA_F32 && dtype != KDA_BF16) return false;
    if (chunk != 0 && chunk != 16 && chunk != 32 && chunk != 64 && chunk != 128) return false;
    return (int64_t)B * H <= 65535;
}

kda_status to_status(cudaError_t e) { return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA; }

}  // namespace
}  // namespace kda

using namespace kda;

extern "C" {

size_t kda_sp_workspace_size(int B, int T, int H, int D, kda_dtype dtype, int chunk)
{
    if (!shard_ok(B, T, H, D, dtype, chunk) || B == 0 || T == 0) return 0;
    const KdaArgs a = shard_args(nullptr, nullptr, nullptr, nullptr, nullptr, B, T, H, D, dtype, chunk);
    if (kda_tc_supported(a)) return kda_tc_sp_workspace_bytes(B, T, H, num_sms());
    return generic_ws(B, T, H, D, dtype).total;
}

kda_status kda_sp_transition(const void* q, const void* k, const void* v, const void* g, const void* beta,
                             float* MN, int B, int T, int H, int D, kda_dtype dtype, int chunk, void* workspace,
                             size_t workspace_bytes, kda_stream_t stream)
{
    if (B < 0 || T < 0 || H <= 0 || (dtype != KDA_F32 && dtype != KDA_BF16)) return KDA_ERR_INVALID_ARG;
    if (!shard_ok(B, T, H, D, dtype, chunk)) return KDA_ERR_UNSUPPORTED;
    if (B == 0) return KDA_OK;
    if (!MN || (T > 0 && (!q || !k || !v || !g || !beta))) return KDA_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    const int BH = B * H;
    const int64_t DD = (int64_t)D * D;
    if (T == 0)   // an empty shard maps S to S: [N | M] = [0 | I]
        return to_status(fold(D, nullptr, 0, 0, nullptr, 0, nullptr, MN, 2 * DD, BH, true, s));
    const size_t need = kda_sp_workspace_size(B, T, H, D, dtype, chunk);
    if (!workspace || workspace_bytes < need) return KDA_ERR_WORKSPACE;
    if (((uintptr_t)workspace & 255) != 0) return KDA_ERR_INVALID_ARG;
    KdaArgs a = shard_args(q, k, v, g, beta, B, T, H, D, dtype, chunk);
    if (kda_tc_supported(a)) {
        int* st = device_status_ptr();
        if (!st) return KDA_ERR_CUDA;
        TcShardMaps sm{};
        cudaError_t e = launch_kda_tc_sp_state(a, workspace, st, s, &sm);
        if (e != cudaSuccess) return KDA_ERR_CUDA;
        // fold the P segment maps of each head: [0 | I] -> [N_r | M_r]
        return to_status(fold(D, sm.maps, 1, sm.P - 1, sm.tail, sm.P, nullptr, MN, 2 * DD, BH, true, s));
    }
    // CUDA-core route: N from a scan from zero, M from a scan of v = 0 from S0 = I
    const GenericWs w = generic_ws(B, T, H, D, dtype);
    char* base = reinterpret_cast<char*>(workspace);
    float* st = reinterpret_cast<float*>(base + w.st);
    float* eye = reinterpret_cast<float*>(base + w.eye);
    a.o = base + w.o;
    a.out_t = ET_F32;
    a.ST = st;
    cudaError_t e = launch_kda_generic(a, s);
    const size_t row = (size_t)DD * sizeof(float);
    if (e == cudaSuccess) e = cudaMemcpy2DAsync(MN, 2 * row, st, row, row, BH, cudaMemcpyDeviceToDevice, s);
    if (e == cudaSuccess)
        e = cudaMemsetAsync(base + w.vz, 0, (size_t)B * T * H * D * (dtype == KDA_F32 ? 4 : 2), s);
    if (e == cudaSuccess) {
        eye_kernel<<<256, 256, 0, s>>>(eye, D, (int64_t)BH * DD);
        count_launch();
        e = cudaGetLastError();
    }
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    a.v = base + w.vz;
    a.S0 = eye;
    e = launch_kda_generic(a, s);
    if (e == cudaSuccess) e = cudaMemcpy2DAsync(MN + DD, 2 * row, st, row, row, BH, cudaMemcpyDeviceToDevice, s);
    return to_status(e);
}

kda_status kda_sp_prefix(const float* MN_all, int R, int r, const float* S0, float* S_in, int B, int H, int D,
                         kda_stream_t stream)
{
    if (B < 0 || H <= 0 || R < 1 || r < 0 || r >= R) return KDA_ERR_INVALID_ARG;
    if (!dim_ok(D) || (int64_t)B * H > 65535) return KDA_ERR_UNSUPPORTED;
    if (B == 0) return KDA_OK;
    if (!S_in || (r > 0 && !MN_all)) return KDA_ERR_INVALID_ARG;
    const int BH = B * H;
    return to_status(fold(D, MN_all, BH, 1, nullptr, r, S0, S_in, (int64_t)D * D, BH, false, (cudaStream_t)stream));
}

kda_status kda_sp_output(const void* q, const void* k, const void* v, const void* g, const void* beta,
                         const float* S_in, void* o, float* S_T, int B, int T, int H, int D, kda_dtype dtype,
                         kda_dtype o_dtype, int chunk, void* workspace, size_t workspace_bytes,
                         kda_stream_t stream)
{
    if (B < 0 || T < 0 || H <= 0 || (dtype != KDA_F32 && dtype != KDA_BF16)) return KDA_ERR_INVALID_ARG;
    if (o_dtype != KDA_F32 && o_dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (!shard_ok(B, T, H, D, dtype, chunk)) return KDA_ERR_UNSUPPORTED;
    if (B == 0) return KDA_OK;
    const KdaArgs probe = shard_args(q, k, v, g, beta, B, T, H, D, dtype, chunk);
    KdaArgs a = probe;
    a.S0 = S_in;
    a.o = o;
    a.ST = S_T;
    a.out_t = et_of(o_dtype);
    if (T > 0 && kda_tc_supported(probe) && kda_tc_supported(a)) {
        if (!q || !k || !v || !g || !beta || !o) return KDA_ERR_INVALID_ARG;
        const size_t need = kda_tc_sp_workspace_bytes(B, T, H, num_sms());
        if (!workspace || workspace_bytes < need) return KDA_ERR_WORKSPACE;
        if (((uintptr_t)workspace & 255) != 0) return KDA_ERR_INVALID_ARG;
        int* st = device_status_ptr();
        if (!st) return KDA_ERR_CUDA;
        return to_status(launch_kda_tc_sp_output(a, workspace, st, (cudaStream_t)stream));
    }
    // no segment maps to reuse: the whole scan from S_in
    return kda_forward(q, k, v, g, beta, S_in, o, S_T, B, T, H, D, D, dtype, o_dtype, chunk, nullptr, 0, stream);
}

}  // extern "C"
