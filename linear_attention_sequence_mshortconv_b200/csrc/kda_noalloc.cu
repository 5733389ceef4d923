// kda_forward_noalloc: the KDA forward scan without any device allocation.
//
// kda_forward needs scratch memory on its tensor-core path (the per-segment state maps
// and segment start states); it either takes it from the caller or allocates it with
// cudaMallocAsync.  Some callers can do neither: code that runs inside a host framework
// which owns every byte of device memory through its own allocator and forbids raw
// allocation in its call path (plugin interfaces of inference engines, serving loops
// that run on a fixed, pre-planned memory budget), or code that must not risk an
// allocation failing or stalling in the middle of a call.  For them this entry point
// takes its scratch from one fixed array compiled into the library instead.
//
// The array lives in device memory of every GPU on which the library's module is
// loaded, and stays there until the process exits.  All calls on a device share it,
// and it keeps whatever the last call left in it: every byte a call reads from it is
// written earlier by the same call, so nothing needs clearing, but calls whose work
// can overlap on the GPU (different streams, no ordering between them) race on it.

#include <mutex>

#include "internal.h"

namespace kda {
namespace {

constexpr size_t kNoAllocScratchBytes = KDA_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDev = 64;
void* g_scratch_ptr[kMaxDev];
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device.  In host code the
// array's name is only a host-side stand-in; the address a kernel can use comes from
// cudaGetSymbolAddress, fetched once per device with that device current.
cudaError_t scratch_address(void** out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

bool dim_ok(int d) { return d == 32 || d == 64 || d == 128; }

}  // namespace
}  // namespace kda

extern "C" kda_status kda_forward_noalloc(const void* q, const void* k, const void* v, const void* g,
                                          const void* beta, const float* S0, void* o, float* S_T,
                                          int B, int T, int H, int Dk, int Dv, kda_dtype dtype,
                                          kda_dtype o_dtype, int chunk, kda_stream_t stream)
{
    using namespace kda;
    if (B < 0 || T < 0 || H <= 0) return KDA_ERR_INVALID_ARG;
    if ((dtype != KDA_F32 && dtype != KDA_BF16) || (o_dtype != KDA_F32 && o_dtype != KDA_BF16))
        return KDA_ERR_INVALID_ARG;
    if (!dim_ok(Dk) || !dim_ok(Dv)) return KDA_ERR_UNSUPPORTED;
    if (chunk != 0 && chunk != 16 && chunk != 32 && chunk != 64 && chunk != 128) return KDA_ERR_UNSUPPORTED;
    if ((int64_t)B * T > 0 && (!q || !k || !v || !g || !beta || !o)) return KDA_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    if (B == 0) return KDA_OK;
    if (T == 0) {
        if (!S_T) return KDA_OK;
        const size_t bytes = (size_t)B * H * Dk * Dv * sizeof(float);
        const cudaError_t e = S0 ? cudaMemcpyAsync(S_T, S0, bytes, cudaMemcpyDeviceToDevice, s)
                                 : cudaMemsetAsync(S_T, 0, bytes, s);
        return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
    }
    const ElemType et = dtype == KDA_F32 ? ET_F32 : ET_BF16;
    KdaArgs a{q, k, v, g, beta, S0, o, S_T, B, T, H, Dk, Dv,
              chunk ? chunk : (dtype == KDA_F32 ? 16 : 64), et, o_dtype == KDA_F32 ? ET_F32 : ET_BF16, et};
    if (!kda_tc_supported(a)) {
        // the CUDA-core path uses no scratch memory
        return launch_kda_generic(a, s) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
    }
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess) return KDA_ERR_CUDA;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const size_t need = kda_tc_workspace_bytes(B, T, H, a.chunk, sms);
    if (need > kNoAllocScratchBytes) return KDA_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return KDA_ERR_CUDA;
    int* status = device_status_ptr();
    if (!status) return KDA_ERR_CUDA;
    return launch_kda_tc(a, scratch, need, status, s) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}
