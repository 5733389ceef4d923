// C ABI of libkda: argument validation, workspace handling and dispatch.
// The operations and their conventions are documented in include/kda.h.

#include <mutex>
#include <vector>

#include "internal.h"

namespace kda {

namespace {
__device__ int g_status;  // device-side failure word (DEV_*), first writer wins

constexpr int kMaxDevices = 64;
int* g_status_ptr[kMaxDevices];
std::mutex g_status_mu;

bool dim_ok(int d) { return d == 32 || d == 64 || d == 128; }

int default_chunk(kda_dtype dt, int Dk) {
    (void)Dk;
    return dt == KDA_F32 ? 16 : 64;
}

int num_sms() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
}  // namespace

int* device_status_ptr()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_status_mu);
    if (!g_status_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return nullptr;
        g_status_ptr[dev] = (int*)p;
    }
    return g_status_ptr[dev];
}

}  // namespace kda

using namespace kda;

namespace {

kda_status check_kda_args(const void* q, const void* k, const void* v, const void* g,
                          const void* beta, const void* o, int B, int T, int H, int Dk,
                          int Dv, kda_dtype dtype, kda_dtype o_dtype, int chunk)
{
    if (B < 0 || T < 0 || H <= 0) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (o_dtype != KDA_F32 && o_dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (!dim_ok(Dk) || !dim_ok(Dv)) return KDA_ERR_UNSUPPORTED;
    if (chunk != 0 && chunk != 16 && chunk != 32 && chunk != 64 && chunk != 128) return KDA_ERR_UNSUPPORTED;
    if ((int64_t)B * T > 0 && (!q || !k || !v || !g || !beta || !o)) return KDA_ERR_INVALID_ARG;
    return KDA_OK;
}

kda_status from_cuda(cudaError_t e) { return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA; }

// Runs the scan given a resolved chunk and a workspace of the required size.
kda_status run_kda(const KdaArgs& a, void* ws, size_t ws_bytes, cudaStream_t s)
{
    if (kda_tc_supported(a)) {
        int* st = device_status_ptr();
        if (!st) return KDA_ERR_CUDA;
        return from_cuda(launch_kda_tc(a, ws, ws_bytes, st, s));
    }
    cudaError_t e = launch_kda_generic(a, s);
    if (e == cudaSuccess && a.gate) e = launch_gate_rmsnorm(a, s);
    return from_cuda(e);
}

size_t kda_ws_bytes(const KdaArgs& a)
{
    if (!kda_tc_supported(a)) return 0;
    return kda_tc_workspace_bytes(a.B, a.T, a.H, a.chunk, num_sms());
}

// Takes the caller's workspace or a stream-ordered allocation of `need` bytes.
struct Workspace {
    void* ptr = nullptr;
    bool owned = false;
    cudaStream_t stream = nullptr;
    kda_status acquire(void* user, size_t user_bytes, size_t need, cudaStream_t s) {
        stream = s;
        if (need == 0) { ptr = user; return KDA_OK; }
        if (user) {
            if (user_bytes < need) return KDA_ERR_WORKSPACE;
            if (((uintptr_t)user & 255) != 0) return KDA_ERR_INVALID_ARG;
            ptr = user;
            return KDA_OK;
        }
        if (cudaMallocAsync(&ptr, need, s) != cudaSuccess) return KDA_ERR_CUDA;
        owned = true;
        return KDA_OK;
    }
    ~Workspace() { if (owned) cudaFreeAsync(ptr, stream); }
};

}  // namespace

extern "C" {

const char* kda_status_string(kda_status s)
{
    switch (s) {
        case KDA_OK: return "KDA_OK";
        case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG";
        case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED";
        case KDA_ERR_CUDA: return "KDA_ERR_CUDA";
        case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT";
        case KDA_ERR_WORKSPACE: return "KDA_ERR_WORKSPACE";
    }
    return "KDA_ERR_UNKNOWN";
}

kda_status kda_last_device_error(void)
{
    int* p = device_status_ptr();
    if (!p) return KDA_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return KDA_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, p, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return KDA_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpy(p, &zero, sizeof zero, cudaMemcpyHostToDevice) != cudaSuccess) return KDA_ERR_CUDA;
    return v == DEV_OK ? KDA_OK
         : v == DEV_TIMEOUT ? KDA_ERR_TIMEOUT
         : v == DEV_RANGE ? KDA_ERR_UNSUPPORTED
                          : KDA_ERR_CUDA;
}

static ElemType et_of(kda_dtype d) { return d == KDA_F32 ? ET_F32 : ET_BF16; }

size_t kda_forward_workspace_size(int B, int T, int H, int Dk, int Dv, kda_dtype dtype,
                                  kda_dtype o_dtype, int chunk)
{
    if (B < 0 || T < 0 || H <= 0 || !dim_ok(Dk) || !dim_ok(Dv)) return 0;
    KdaArgs a{};
    a.B = B; a.T = T; a.H = H; a.Dk = Dk; a.Dv = Dv;
    a.in_t = a.gb_t = et_of(dtype);
    a.out_t = et_of(o_dtype);
    a.chunk = chunk ? chunk : default_chunk(dtype, Dk);
    return kda_ws_bytes(a);
}

kda_status kda_forward_plan(int B, int T, int H, int Dk, int Dv, kda_dtype dtype, kda_dtype o_dtype, int chunk,
                            int* segments, int* chunks_per_segment)
{
    if (!segments || !chunks_per_segment) return KDA_ERR_INVALID_ARG;
    *segments = *chunks_per_segment = 0;
    if (B < 0 || T < 0 || H <= 0 || !dim_ok(Dk) || !dim_ok(Dv)) return KDA_ERR_INVALID_ARG;
    KdaArgs a{};
    a.B = B; a.T = T; a.H = H; a.Dk = Dk; a.Dv = Dv;
    a.in_t = a.gb_t = et_of(dtype);
    a.out_t = et_of(o_dtype);
    a.chunk = chunk ? chunk : default_chunk(dtype, Dk);
    if (T < 1 || !kda_tc_supported(a)) return KDA_OK;
    kda_tc_plan(B, T, H, num_sms(), segments, chunks_per_segment);
    return KDA_OK;
}

kda_status kda_forward(const void* q, const void* k, const void* v, const void* g,
                       const void* beta, const float* S0, void* o, float* S_T,
                       int B, int T, int H, int Dk, int Dv, kda_dtype dtype,
                       kda_dtype o_dtype, int chunk, void* workspace, size_t workspace_bytes,
                       kda_stream_t stream)
{
    kda_status st = check_kda_args(q, k, v, g, beta, o, B, T, H, Dk, Dv, dtype, o_dtype, chunk);
    if (st != KDA_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    if (B == 0) return KDA_OK;
    if (T == 0) {
        if (!S_T) return KDA_OK;
        const size_t bytes = (size_t)B * H * Dk * Dv * sizeof(float);
        return from_cuda(S0 ? cudaMemcpyAsync(S_T, S0, bytes, cudaMemcpyDeviceToDevice, s)
                            : cudaMemsetAsync(S_T, 0, bytes, s));
    }
    KdaArgs a{q, k, v, g, beta, S0, o, S_T, B, T, H, Dk, Dv,
              chunk ? chunk : default_chunk(dtype, Dk), et_of(dtype), et_of(o_dtype), et_of(dtype)};
    Workspace ws;
    st = ws.acquire(workspace, workspace_bytes, kda_ws_bytes(a), s);
    if (st != KDA_OK) return st;
    return run_kda(a, ws.ptr, kda_ws_bytes(a), s);
}

kda_status kda_forward_gated(const void* q, const void* k, const void* v, const void* g,
                             const void* beta, const float* S0, const void* gate, const float* gamma,
                             float eps, void* o, float* S_T, int B, int T, int H, int Dk, int Dv,
                             kda_dtype dtype, kda_dtype o_dtype, int chunk, void* workspace,
                             size_t workspace_bytes, kda_stream_t stream)
{
    kda_status st = check_kda_args(q, k, v, g, beta, o, B, T, H, Dk, Dv, dtype, o_dtype, chunk);
    if (st != KDA_OK) return st;
    if ((int64_t)B * T > 0 && !gate) return KDA_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || eps > 1e30f) return KDA_ERR_INVALID_ARG;   // also rejects NaN
    cudaStream_t s = (cudaStream_t)stream;
    if (B == 0) return KDA_OK;
    if (T == 0)
        return kda_forward(q, k, v, g, beta, S0, o, S_T, B, T, H, Dk, Dv, dtype, o_dtype, chunk, workspace,
                           workspace_bytes, stream);
    KdaArgs a{q, k, v, g, beta, S0, o, S_T, B, T, H, Dk, Dv,
              chunk ? chunk : default_chunk(dtype, Dk), et_of(dtype), et_of(o_dtype), et_of(dtype)};
    a.gate = gate;
    a.gamma = gamma;
    a.eps = eps;
    Workspace ws;
    st = ws.acquire(workspace, workspace_bytes, kda_ws_bytes(a), s);
    if (st != KDA_OK) return st;
    return run_kda(a, ws.ptr, kda_ws_bytes(a), s);
}

// ---- packed samples -------------------------------------------------------------------
static kda_status check_cu(const int32_t* cu, int n_seqs)
{
    if (n_seqs < 0 || !cu) return KDA_ERR_INVALID_ARG;
    if (cu[0] != 0) return KDA_ERR_INVALID_ARG;
    for (int i = 0; i < n_seqs; ++i)
        if (cu[i + 1] < cu[i]) return KDA_ERR_INVALID_ARG;
    return KDA_OK;
}

static KdaArgs varlen_args(const void* q, const void* k, const void* v, const void* g, const void* beta,
                           const float* S0, void* o, float* S_T, int T_total, int H, int Dk, int Dv,
                           kda_dtype dtype, kda_dtype o_dtype, int chunk)
{
    return KdaArgs{q, k, v, g, beta, S0, o, S_T, 1, T_total, H, Dk, Dv,
                   chunk ? chunk : default_chunk(dtype, Dk), et_of(dtype), et_of(o_dtype), et_of(dtype)};
}

size_t kda_forward_varlen_workspace_size(const int32_t* cu_seqlens, int n_seqs, int H, int Dk, int Dv,
                                         kda_dtype dtype, kda_dtype o_dtype, int chunk)
{
    if (check_cu(cu_seqlens, n_seqs) != KDA_OK || H <= 0 || !dim_ok(Dk) || !dim_ok(Dv)) return 0;
    if (n_seqs == 0 || cu_seqlens[n_seqs] == 0) return 0;
    const KdaArgs a = varlen_args(nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                                  cu_seqlens[n_seqs], H, Dk, Dv, dtype, o_dtype, chunk);
    if (!kda_tc_supported(a)) return 0;
    return kda_tc_varlen_workspace_bytes(cu_seqlens, n_seqs, H, num_sms());
}

kda_status kda_forward_varlen(const void* q, const void* k, const void* v, const void* g, const void* beta,
                              const float* S0, void* o, float* S_T, const int32_t* cu_seqlens, int n_seqs,
                              int H, int Dk, int Dv, kda_dtype dtype, kda_dtype o_dtype, int chunk,
                              void* workspace, size_t workspace_bytes, kda_stream_t stream)
{
    kda_status st = check_cu(cu_seqlens, n_seqs);
    if (st != KDA_OK) return st;
    const int T = n_seqs ? cu_seqlens[n_seqs] : 0;
    st = check_kda_args(q, k, v, g, beta, o, 1, T, H, Dk, Dv, dtype, o_dtype, chunk);
    if (st != KDA_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    if (n_seqs == 0) return KDA_OK;
    // empty samples: S_T = S0 (or zero)
    const size_t sbytes = (size_t)H * Dk * Dv * sizeof(float);
    for (int i = 0; i < n_seqs; ++i) {
        if (cu_seqlens[i + 1] != cu_seqlens[i] || !S_T) continue;
        float* dst = S_T + (size_t)i * H * Dk * Dv;
        const cudaError_t e = S0 ? cudaMemcpyAsync(dst, S0 + (size_t)i * H * Dk * Dv, sbytes, cudaMemcpyDeviceToDevice, s)
                                 : cudaMemsetAsync(dst, 0, sbytes, s);
        if (e != cudaSuccess) return KDA_ERR_CUDA;
    }
    if (T == 0) return KDA_OK;
    const KdaArgs a = varlen_args(q, k, v, g, beta, S0, o, S_T, T, H, Dk, Dv, dtype, o_dtype, chunk);
    if (kda_tc_supported(a)) {
        const size_t need = kda_tc_varlen_workspace_bytes(cu_seqlens, n_seqs, H, num_sms());
        Workspace ws;
        st = ws.acquire(workspace, workspace_bytes, need, s);
        if (st != KDA_OK) return st;
        int* dst = device_status_ptr();
        if (!dst) return KDA_ERR_CUDA;
        return from_cuda(launch_kda_tc_varlen(a, cu_seqlens, n_seqs, ws.ptr, dst, s));
    }
    // CUDA-core path: one launch per non-empty sample on its slice of the packed axis
    const size_t es = dtype == KDA_F32 ? 4 : 2, eo = o_dtype == KDA_F32 ? 4 : 2;
    for (int i = 0; i < n_seqs; ++i) {
        const int t0 = cu_seqlens[i], len = cu_seqlens[i + 1] - t0;
        if (len == 0) continue;
        const size_t kq = (size_t)t0 * H * Dk, kv = (size_t)t0 * H * Dv, kb = (size_t)t0 * H;
        KdaArgs ai = a;
        ai.T = len;
        ai.q = (const char*)q + kq * es;
        ai.k = (const char*)k + kq * es;
        ai.g = (const char*)g + kq * es;
        ai.v = (const char*)v + kv * es;
        ai.beta = (const char*)beta + kb * es;
        ai.o = (char*)o + kv * eo;
        ai.S0 = S0 ? S0 + (size_t)i * H * Dk * Dv : nullptr;
        ai.ST = S_T ? S_T + (size_t)i * H * Dk * Dv : nullptr;
        const cudaError_t e = launch_kda_generic(ai, s);
        if (e != cudaSuccess) return KDA_ERR_CUDA;
    }
    return KDA_OK;
}

// ---- backward ---------------------------------------------------------------------------
size_t kda_backward_workspace_size(int B, int T, int H, int Dk, int Dv)
{
    if (B < 0 || T < 0 || H <= 0 || !dim_ok(Dk) || !dim_ok(Dv)) return 0;
    return kda_bwd_workspace_bytes(B, T, H, Dk, Dv);
}

kda_status kda_backward(const void* q, const void* k, const void* v, const void* g, const void* beta,
                        const float* S0, const void* d_o, const float* dS_T, float* dq, float* dk, float* dv,
                        float* dg, float* dbeta, float* dS0, int B, int T, int H, int Dk, int Dv,
                        kda_dtype dtype, kda_dtype do_dtype, void* workspace, size_t workspace_bytes,
                        kda_stream_t stream)
{
    if (B < 0 || T < 0 || H <= 0) return KDA_ERR_INVALID_ARG;
    if ((dtype != KDA_F32 && dtype != KDA_BF16) || (do_dtype != KDA_F32 && do_dtype != KDA_BF16))
        return KDA_ERR_INVALID_ARG;
    if (!dim_ok(Dk) || !dim_ok(Dv) || B > 65535 || H > 65535) return KDA_ERR_UNSUPPORTED;
    if ((int64_t)B * T > 0 && (!q || !k || !v || !g || !beta || !d_o || !dq || !dk || !dv || !dg || !dbeta))
        return KDA_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    if (B == 0) return KDA_OK;
    if (T == 0) {   // no tokens: dS0 = dS_T
        if (!dS0) return KDA_OK;
        const size_t bytes = (size_t)B * H * Dk * Dv * sizeof(float);
        return from_cuda(dS_T ? cudaMemcpyAsync(dS0, dS_T, bytes, cudaMemcpyDeviceToDevice, s)
                              : cudaMemsetAsync(dS0, 0, bytes, s));
    }
    int* status = device_status_ptr();
    if (!status) return KDA_ERR_CUDA;
    const KdaBwdArgs a{q, k, v, g, beta, S0, d_o, dS_T, dq, dk, dv, dg, dbeta, dS0, B, T, H, Dk, Dv,
                       et_of(dtype), et_of(do_dtype), status};
    Workspace ws;
    kda_status st = ws.acquire(workspace, workspace_bytes, kda_bwd_workspace_bytes(B, T, H, Dk, Dv), s);
    if (st != KDA_OK) return st;
    return from_cuda(launch_kda_bwd(a, ws.ptr, s));
}

static kda_status check_segments(const msc_segment* segs, int n_segs, int T, int Kt,
                                 const float* w_text, int n_text, const float* w_image,
                                 int n_image, const float* w_video, int n_video)
{
    if (n_segs < 0 || (n_segs > 0 && !segs)) return KDA_ERR_INVALID_ARG;
    if (Kt < 1 || Kt > 8) return KDA_ERR_UNSUPPORTED;
    int64_t prev_end = 0;
    for (int i = 0; i < n_segs; ++i) {
        const msc_segment& sg = segs[i];
        if (sg.reserved != 0) return KDA_ERR_INVALID_ARG;
        int64_t len;
        if (sg.modality == MSC_TEXT) {
            if (sg.F != 1 || sg.Hgt != 1 || sg.Wid < 1) return KDA_ERR_INVALID_ARG;
            if (!w_text || sg.weight_set < 0 || sg.weight_set >= n_text) return KDA_ERR_INVALID_ARG;
            len = sg.Wid;
        } else if (sg.modality == MSC_IMAGE) {
            if (sg.F != 1 || sg.Hgt < 1 || sg.Wid < 1) return KDA_ERR_INVALID_ARG;
            if (!w_image || sg.weight_set < 0 || sg.weight_set >= n_image) return KDA_ERR_INVALID_ARG;
            len = (int64_t)sg.Hgt * sg.Wid;
        } else if (sg.modality == MSC_VIDEO) {
            if (sg.F < 1 || sg.Hgt < 1 || sg.Wid < 1) return KDA_ERR_INVALID_ARG;
            if (!w_video || sg.weight_set < 0 || sg.weight_set >= n_video) return KDA_ERR_INVALID_ARG;
            len = (int64_t)sg.F * sg.Hgt * sg.Wid;
        } else {
            return KDA_ERR_INVALID_ARG;
        }
        if (sg.start < prev_end || sg.start + len > T) return KDA_ERR_INVALID_ARG;
        prev_end = sg.start + len;
    }
    return KDA_OK;
}

static int64_t seg_len(const msc_segment& sg)
{
    return sg.modality == MSC_TEXT ? sg.Wid
         : sg.modality == MSC_IMAGE ? (int64_t)sg.Hgt * sg.Wid : (int64_t)sg.F * sg.Hgt * sg.Wid;
}

// Zeroes the token ranges of y that no segment covers.
static cudaError_t zero_gaps(void* y, int B, int T, int C, size_t esz, const msc_segment* segs,
                             int n_segs, cudaStream_t s)
{
    std::vector<std::pair<int64_t, int64_t>> gaps;
    int64_t pos = 0;
    for (int i = 0; i < n_segs; ++i) {
        if (segs[i].start > pos) gaps.push_back({pos, segs[i].start});
        pos = segs[i].start + seg_len(segs[i]);
    }
    if (pos < T) gaps.push_back({pos, T});
    for (auto& gp : gaps)
        for (int b = 0; b < B; ++b) {
            char* base = (char*)y + (((int64_t)b * T + gp.first) * C) * esz;
            cudaError_t e = cudaMemsetAsync(base, 0, (size_t)(gp.second - gp.first) * C * esz, s);
            if (e != cudaSuccess) return e;
        }
    return cudaSuccess;
}

static const float* seg_weights(const msc_segment& sg, int C, int Kt, const float* wt,
                                const float* wi, const float* wv)
{
    if (sg.modality == MSC_TEXT) return wt + (int64_t)sg.weight_set * C * Kt;
    if (sg.modality == MSC_IMAGE) return wi + (int64_t)sg.weight_set * C * 9;
    return wv + (int64_t)sg.weight_set * C * 27;
}

static ConvSeg to_conv_seg(const msc_segment& sg)
{
    return ConvSeg{sg.modality, sg.start, sg.F, sg.Hgt, sg.Wid, sg.weight_set};
}

kda_status mshortconv_forward(const void* x, void* y, int B, int T, int C, kda_dtype dtype,
                              const msc_segment* segs, int n_segs, int Kt,
                              const float* w_text, int n_text_sets,
                              const float* w_image, int n_image_sets,
                              const float* w_video, int n_video_sets,
                              kda_stream_t stream)
{
    if (B < 0 || T < 0 || C <= 0 || (C % 8) != 0) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if ((int64_t)B * T > 0 && (!x || !y)) return KDA_ERR_INVALID_ARG;
    if (x && x == y) return KDA_ERR_INVALID_ARG;
    kda_status st = check_segments(segs, n_segs, T, Kt, w_text, n_text_sets, w_image,
                                   n_image_sets, w_video, n_video_sets);
    if (st != KDA_OK) return st;
    if ((int64_t)B * T == 0) return KDA_OK;
    cudaStream_t s = (cudaStream_t)stream;
    const size_t esz = dtype == KDA_F32 ? 4 : 2;
    cudaError_t e = zero_gaps(y, B, T, C, esz, segs, n_segs, s);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    for (int i = 0; i < n_segs; ++i) {
        const ElemType et = dtype == KDA_F32 ? ET_F32 : ET_BF16;
        const void* xs[1] = {x};
        void* ys[1] = {y};
        const float* wsel[1] = {seg_weights(segs[i], C, Kt, w_text, w_image, w_video)};
        const int nd[1] = {0};
        e = launch_conv_segment_multi(1, xs, ys, B, T, C, et, et, to_conv_seg(segs[i]), Kt, wsel, nd, s);
        if (e != cudaSuccess) return KDA_ERR_CUDA;
    }
    return KDA_OK;
}

// The conv backward after validation: dw zeroed then accumulated, dx zeroed then written
// over the segments.  x, dy: [B, T, C] of element type et.
static kda_status conv_backward_run(const void* x, const void* dy, float* dx, int B, int T, int C, ElemType et,
                                    const msc_segment* segs, int n_segs, int Kt, const float* w_text, int n_text_sets,
                                    const float* w_image, int n_image_sets, const float* w_video, int n_video_sets,
                                    float* dw_text, float* dw_image, float* dw_video, cudaStream_t s)
{
    cudaError_t e = cudaSuccess;
    // weight gradients are sums over rows and segments: zeroed, then accumulated
    if (dw_text && n_text_sets > 0) e = cudaMemsetAsync(dw_text, 0, (size_t)n_text_sets * C * Kt * sizeof(float), s);
    if (e == cudaSuccess && dw_image && n_image_sets > 0)
        e = cudaMemsetAsync(dw_image, 0, (size_t)n_image_sets * C * 9 * sizeof(float), s);
    if (e == cudaSuccess && dw_video && n_video_sets > 0)
        e = cudaMemsetAsync(dw_video, 0, (size_t)n_video_sets * C * 27 * sizeof(float), s);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    if ((int64_t)B * T == 0) return KDA_OK;
    if (cudaMemsetAsync(dx, 0, (size_t)B * T * C * sizeof(float), s) != cudaSuccess) return KDA_ERR_CUDA;
    for (int i = 0; i < n_segs; ++i) {
        const msc_segment& sg = segs[i];
        float* dw_all = sg.modality == MSC_TEXT ? dw_text : sg.modality == MSC_IMAGE ? dw_image : dw_video;
        const int ntaps = sg.modality == MSC_TEXT ? Kt : sg.modality == MSC_IMAGE ? 9 : 27;
        float* dw = dw_all ? dw_all + (int64_t)sg.weight_set * C * ntaps : nullptr;
        e = launch_conv_backward_segment(x, dy, dx, seg_weights(sg, C, Kt, w_text, w_image, w_video), dw, B, T, C,
                                         et, to_conv_seg(sg), Kt, s);
        if (e != cudaSuccess) return KDA_ERR_CUDA;
    }
    return KDA_OK;
}

kda_status mshortconv_backward(const void* x, const void* dy, float* dx, int B, int T, int C, kda_dtype dtype,
                               const msc_segment* segs, int n_segs, int Kt, const float* w_text, int n_text_sets,
                               const float* w_image, int n_image_sets, const float* w_video, int n_video_sets,
                               float* dw_text, float* dw_image, float* dw_video, kda_stream_t stream)
{
    if (B < 0 || T < 0 || C <= 0 || (C % 8) != 0) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    const bool want_dw = dw_text || dw_image || dw_video;
    if ((int64_t)B * T > 0 && (!dy || !dx || (want_dw && !x))) return KDA_ERR_INVALID_ARG;
    kda_status st = check_segments(segs, n_segs, T, Kt, w_text, n_text_sets, w_image,
                                   n_image_sets, w_video, n_video_sets);
    if (st != KDA_OK) return st;
    return conv_backward_run(x, dy, dx, B, T, C, dtype == KDA_F32 ? ET_F32 : ET_BF16, segs, n_segs, Kt, w_text,
                             n_text_sets, w_image, n_image_sets, w_video, n_video_sets, dw_text, dw_image, dw_video,
                             (cudaStream_t)stream);
}

// The fused path keeps q, k, v between the conv and the scan as fp16 (fp32 inputs:
// fp32) in the workspace.
static KdaArgs fused_kda_args(int B, int T, int H, int D, kda_dtype dtype, kda_dtype o_dtype,
                              int chunk)
{
    KdaArgs a{};
    a.B = B; a.T = T; a.H = H; a.Dk = D; a.Dv = D;
    a.chunk = chunk ? chunk : default_chunk(dtype, D);
    a.in_t = dtype == KDA_F32 ? ET_F32 : ET_F16;
    a.gb_t = et_of(dtype);
    a.out_t = et_of(o_dtype);
    return a;
}

size_t kda_mshortconv_workspace_size(int B, int T, int H, int D, kda_dtype dtype,
                                     kda_dtype o_dtype, int chunk)
{
    if (B < 0 || T < 0 || H <= 0 || !dim_ok(D)) return 0;
    const size_t qkv = align256((size_t)B * T * H * D * (dtype == KDA_F32 ? 4 : 2));
    return 3 * qkv + align256(kda_ws_bytes(fused_kda_args(B, T, H, D, dtype, o_dtype, chunk)));
}

kda_status kda_mshortconv_forward(const void* xq, const void* xk, const void* xv,
                                  const msc_segment* segs, int n_segs, int Kt,
                                  const float* const wq[3], const float* const wk[3],
                                  const float* const wv[3],
                                  const void* g, const void* beta, const float* S0,
                                  void* o, float* S_T, int B, int T, int H, int D,
                                  kda_dtype dtype, kda_dtype o_dtype, int chunk,
                                  void* workspace, size_t workspace_bytes,
                                  kda_stream_t stream)
{
    if (!wq || !wk || !wv) return KDA_ERR_INVALID_ARG;
    kda_status st = check_kda_args(xq, xk, xv, g, beta, o, B, T, H, D, D, dtype, o_dtype, chunk);
    if (st != KDA_OK) return st;
    const int C = H * D;
    for (const float* const* w : {wq, wk, wv}) {
        st = check_segments(segs, n_segs, T, Kt, w[0], 1, w[1], 1, w[2], 1);
        if (st != KDA_OK) return st;
    }
    if (B == 0) return KDA_OK;
    cudaStream_t s = (cudaStream_t)stream;
    if (T == 0)
        return kda_forward(xq, xk, xv, g, beta, S0, o, S_T, B, T, H, D, D, dtype, o_dtype,
                           chunk, nullptr, 0, stream);
    const size_t need = kda_mshortconv_workspace_size(B, T, H, D, dtype, o_dtype, chunk);
    Workspace ws;
    st = ws.acquire(workspace, workspace_bytes, need, s);
    if (st != KDA_OK) return st;
    const size_t esz = dtype == KDA_F32 ? 4 : 2;
    const size_t qkv = align256((size_t)B * T * H * D * esz);
    const ElemType in_t = dtype == KDA_F32 ? ET_F32 : ET_BF16;
    const ElemType mid_t = dtype == KDA_F32 ? ET_F32 : ET_F16;
    char* base = (char*)ws.ptr;
    void* qb = base;
    void* kb = base + qkv;
    void* vb = base + 2 * qkv;
    void* kws = base + 3 * qkv;
    const void* xs[3] = {xq, xk, xv};
    void* ys[3] = {qb, kb, vb};
    const float* const* ws3[3] = {wq, wk, wv};
    for (int tsr = 0; tsr < 3; ++tsr) {
        cudaError_t e = zero_gaps(ys[tsr], B, T, C, esz, segs, n_segs, s);  // esz: fp16 = bf16 size
        if (e != cudaSuccess) return KDA_ERR_CUDA;
    }
    const int norms[3] = {D, D, 0};
    for (int i = 0; i < n_segs; ++i) {
        msc_segment sg = segs[i];
        sg.weight_set = 0;
        const float* wsel[3];
        for (int tsr = 0; tsr < 3; ++tsr) wsel[tsr] = seg_weights(sg, C, Kt, ws3[tsr][0], ws3[tsr][1], ws3[tsr][2]);
        cudaError_t e = launch_conv_segment_multi(3, xs, ys, B, T, C, in_t, mid_t, to_conv_seg(sg), Kt, wsel, norms, s);
        if (e != cudaSuccess) return KDA_ERR_CUDA;
    }
    KdaArgs a = fused_kda_args(B, T, H, D, dtype, o_dtype, chunk);
    a.q = qb; a.k = kb; a.v = vb; a.g = g; a.beta = beta; a.S0 = S0; a.o = o; a.ST = S_T;
    return run_kda(a, kws, need - 3 * qkv, s);
}

}  // extern "C"

// ---- backward of the fused path --------------------------------------------------------
namespace {
struct FusedBwdLayout {
    size_t x32, g32, b32, y, qk, d, bws, total;   // offsets (bytes)
};
FusedBwdLayout fused_bwd_layout(int B, int T, int H, int D, kda_dtype dtype)
{
    const size_t tok = (size_t)B * T * H * D, f = sizeof(float);
    const bool widen = dtype != KDA_F32;
    FusedBwdLayout l{};
    size_t off = 0;
    l.x32 = off; off += widen ? 3 * align256(tok * f) : 0;
    l.g32 = off; off += widen ? align256(tok * f) : 0;
    l.b32 = off; off += widen ? align256((size_t)B * T * H * f) : 0;
    l.y = off;   off += 3 * align256(tok * f);   // conv outputs y_q, y_k, y_v
    l.qk = off;  off += 2 * align256(tok * f);   // q, k
    l.d = off;   off += 3 * align256(tok * f);   // dq, dk, dv
    l.bws = off; off += align256(kda_bwd_workspace_bytes(B, T, H, D, D));
    l.total = off;
    return l;
}
}  // namespace

extern "C" {

size_t kda_mshortconv_backward_workspace_size(int B, int T, int H, int D, kda_dtype dtype)
{
    if (B < 0 || T < 0 || H <= 0 || !dim_ok(D) || (dtype != KDA_F32 && dtype != KDA_BF16)) return 0;
    if ((int64_t)B * T == 0) return 0;
    return fused_bwd_layout(B, T, H, D, dtype).total;
}

kda_status kda_mshortconv_backward(const void* xq, const void* xk, const void* xv, const msc_segment* segs,
                                   int n_segs, int Kt, const float* const wq[3], const float* const wk[3],
                                   const float* const wv[3], const void* g, const void* beta, const float* S0,
                                   const void* d_o, kda_dtype do_dtype, const float* dS_T, float* dxq, float* dxk,
                                   float* dxv, float* const dwq[3], float* const dwk[3], float* const dwv[3],
                                   float* dg, float* dbeta, float* dS0, int B, int T, int H, int D, kda_dtype dtype,
                                   void* workspace, size_t workspace_bytes, kda_stream_t stream)
{
    if (!wq || !wk || !wv || !dwq || !dwk || !dwv) return KDA_ERR_INVALID_ARG;
    if (B < 0 || T < 0 || H <= 0) return KDA_ERR_INVALID_ARG;
    if ((dtype != KDA_F32 && dtype != KDA_BF16) || (do_dtype != KDA_F32 && do_dtype != KDA_BF16))
        return KDA_ERR_INVALID_ARG;
    if (!dim_ok(D) || B > 65535 || H > 65535) return KDA_ERR_UNSUPPORTED;
    if ((int64_t)B * T > 0 && (!xq || !xk || !xv || !g || !beta || !d_o || !dxq || !dxk || !dxv || !dg || !dbeta))
        return KDA_ERR_INVALID_ARG;
    const int C = H * D;
    for (const float* const* w : {wq, wk, wv}) {
        const kda_status st = check_segments(segs, n_segs, T, Kt, w[0], 1, w[1], 1, w[2], 1);
        if (st != KDA_OK) return st;
    }
    if (B == 0) return KDA_OK;
    cudaStream_t s = (cudaStream_t)stream;
    if (T == 0) {   // no tokens: zero weight gradients, dS0 = dS_T
        for (float* const* dw : {dwq, dwk, dwv})
            for (int m = 0; m < 3; ++m)
                if (dw[m] && cudaMemsetAsync(dw[m], 0, (size_t)C * (m == 0 ? Kt : m == 1 ? 9 : 27) * sizeof(float), s) !=
                                 cudaSuccess)
                    return KDA_ERR_CUDA;
        return kda_backward(nullptr, nullptr, nullptr, nullptr, nullptr, S0, nullptr, dS_T, nullptr, nullptr, nullptr,
                            nullptr, nullptr, dS0, B, 0, H, D, D, dtype, do_dtype, nullptr, 0, stream);
    }
    const FusedBwdLayout L = fused_bwd_layout(B, T, H, D, dtype);
    Workspace ws;
    kda_status st = ws.acquire(workspace, workspace_bytes, L.total, s);
    if (st != KDA_OK) return st;
    char* base = (char*)ws.ptr;
    const size_t tok = (size_t)B * T * C;
    const size_t tb = align256(tok * sizeof(float));
    // 0. fp32 copies of bf16 inputs
    const void* xs[3] = {xq, xk, xv};
    const float* x32[3];
    const float *g32 = (const float*)g, *b32 = (const float*)beta;
    cudaError_t e = cudaSuccess;
    if (dtype == KDA_BF16) {
        for (int i = 0; i < 3 && e == cudaSuccess; ++i) {
            float* dst = (float*)(base + L.x32 + i * tb);
            e = launch_to_f32(xs[i], ET_BF16, dst, (int64_t)tok, s);
            x32[i] = dst;
        }
        if (e == cudaSuccess) e = launch_to_f32(g, ET_BF16, (float*)(base + L.g32), (int64_t)tok, s);
        if (e == cudaSuccess) e = launch_to_f32(beta, ET_BF16, (float*)(base + L.b32), (int64_t)B * T * H, s);
        g32 = (const float*)(base + L.g32);
        b32 = (const float*)(base + L.b32);
    } else {
        for (int i = 0; i < 3; ++i) x32[i] = (const float*)xs[i];
    }
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    // 1. conv outputs, fp32
    float* y[3];
    const float* const* ws3[3] = {wq, wk, wv};
    for (int i = 0; i < 3; ++i) {
        y[i] = (float*)(base + L.y + i * tb);
        e = zero_gaps(y[i], B, T, C, sizeof(float), segs, n_segs, s);
        for (int j = 0; j < n_segs && e == cudaSuccess; ++j) {
            msc_segment sg = segs[j];
            sg.weight_set = 0;
            e = launch_conv_segment(x32[i], y[i], B, T, C, ET_F32, ET_F32, to_conv_seg(sg), Kt,
                                    seg_weights(sg, C, Kt, ws3[i][0], ws3[i][1], ws3[i][2]), 0, s);
        }
        if (e != cudaSuccess) return KDA_ERR_CUDA;
    }
    // 2. q, k = unit rows per (token, head)
    float* q = (float*)(base + L.qk);
    float* k = (float*)(base + L.qk + tb);
    e = launch_l2norm_rows(y[0], q, (int64_t)B * T * H, D, s);
    if (e == cudaSuccess) e = launch_l2norm_rows(y[1], k, (int64_t)B * T * H, D, s);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    // 3. the scan's backward
    float* dq = (float*)(base + L.d);
    float* dk = (float*)(base + L.d + tb);
    float* dv = (float*)(base + L.d + 2 * tb);
    int* status = device_status_ptr();
    if (!status) return KDA_ERR_CUDA;
    const KdaBwdArgs a{q, k, y[2], g32, b32, S0, d_o, dS_T, dq, dk, dv, dg, dbeta, dS0, B, T, H, D, D, ET_F32,
                       do_dtype == KDA_F32 ? ET_F32 : ET_BF16, status};
    e = launch_kda_bwd(a, base + L.bws, s);
    // 4. through the norms
    if (e == cudaSuccess) e = launch_l2norm_bwd_rows(y[0], dq, (int64_t)B * T * H, D, s);
    if (e == cudaSuccess) e = launch_l2norm_bwd_rows(y[1], dk, (int64_t)B * T * H, D, s);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    // 5. the conv backward of each tensor (one weight set per modality)
    std::vector<msc_segment> segs0(segs, segs + n_segs);
    for (auto& sg : segs0) sg.weight_set = 0;
    const float* dys[3] = {dq, dk, dv};
    float* dxs[3] = {dxq, dxk, dxv};
    float* const* dws[3] = {dwq, dwk, dwv};
    for (int i = 0; i < 3; ++i) {
        st = conv_backward_run(x32[i], dys[i], dxs[i], B, T, C, ET_F32, segs0.data(), n_segs, Kt, ws3[i][0], 1,
                               ws3[i][1], 1, ws3[i][2], 1, dws[i][0], dws[i][1], dws[i][2], s);
        if (st != KDA_OK) return st;
    }
    return KDA_OK;
}

}  // extern "C"
