// Output side of Eq. 15 (Chimera paper, section 3.3) before the output projection W_o:
// y = Sigmoid(gate) * gamma_h * RMSNorm(o) per (token, head), in place on o.  Used after
// the CUDA-core scan and after the tensor-core scan with an fp32 output; the tensor-core
// scan with a bf16 output applies the same epilogue in its output stage instead.

#include "internal.h"

namespace kda {
namespace {

__device__ __forceinline__ float ld_el(const float* p) { return *p; }
__device__ __forceinline__ float ld_el(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st_el(float* p, float v) { *p = v; }
__device__ __forceinline__ void st_el(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// One warp per (token, head) row of Dv (32, 64 or 128) channels; lane l holds channels
// l, l + 32, ... (coalesced).
template <typename TO, typename TG>
__global__ void __launch_bounds__(256)
gate_rmsnorm_kernel(TO* __restrict__ o, const TG* __restrict__ gate, const float* __restrict__ gamma, float eps,
                    int64_t rows, int H, int Dv)
{
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (row >= rows) return;
    const int lane = threadIdx.x & 31, h = (int)(row % H), per = Dv >> 5;
    TO* orow = o + row * Dv;
    const TG* grow = gate + row * Dv;
    float v[4], gt[4], ss = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (i < per) {
            v[i] = ld_el(orow + lane + 32 * i);
            gt[i] = ld_el(grow + lane + 32 * i);
            ss = fmaf(v[i], v[i], ss);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float m = ss / (float)Dv + eps;
    const float inv = m > 0.f ? rsqrtf(m) : 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (i < per) {
            const int c = lane + 32 * i;
            const float gm = gamma ? gamma[(int64_t)h * Dv + c] : 1.f;
            const float sg = 1.f / (1.f + __expf(-gt[i]));
            st_el(orow + c, v[i] * inv * gm * sg);
        }
    }
}

template <typename TO, typename TG>
cudaError_t launch_typed(const KdaArgs& a, cudaStream_t s)
{
    const int64_t rows = (int64_t)a.B * a.T * a.H;
    if (rows == 0) return cudaSuccess;
    ProfileScope prof("gate_norm", s);
    count_launch();
    gate_rmsnorm_kernel<TO, TG><<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(
        (TO*)a.o, (const TG*)a.gate, a.gamma, a.eps, rows, a.H, a.Dv);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gate_rmsnorm(const KdaArgs& a, cudaStream_t s)
{
    const bool o32 = a.out_t == ET_F32, g32 = a.in_t == ET_F32;
    if (o32 && g32) return launch_typed<float, float>(a, s);
    if (o32 && !g32) return launch_typed<float, __nv_bfloat16>(a, s);
    if (!o32 && g32) return launch_typed<__nv_bfloat16, float>(a, s);
    return launch_typed<__nv_bfloat16, __nv_bfloat16>(a, s);
}

}  // namespace kda
