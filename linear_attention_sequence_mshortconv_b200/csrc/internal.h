// Internal declarations shared by the translation units of libkda (not installed).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kda.h"

namespace kda {

// ---- element types ----------------------------------------------------------------
// Public tensors are fp32 or bf16 (kda_dtype).  fp16 is used internally for the
// fused path's conv outputs (q, k, v between the conv and the scan): its 11-bit
// significand keeps the extra rounding well inside the parity bound, where a bf16
// intermediate alone costs about 2% of RMS(o) in max error.
enum ElemType : int { ET_F32 = 0, ET_BF16 = 1, ET_F16 = 2 };

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_f32(__half x) { return __half2float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}
template <> __device__ __forceinline__ __half from_f32<__half>(float x) { return __float2half_rn(x); }

// ---- launch accounting and optional per-kernel event timing ------------------------
void count_launch();
// Test hook (kda_debug_drop_handoff): non-zero makes the tensor-core scan withhold one
// hand-off between its warp roles per CTA, so a bounded wait runs out.
int debug_drop_handoff();
// Records CUDA events around the kernels launched in its lifetime when profiling is
// enabled (kda_profile_enable); a no-op otherwise.
class ProfileScope {
  public:
    ProfileScope(const char* name, cudaStream_t s);
    ~ProfileScope();
  private:
    const char* name_;
    cudaStream_t s_;
    cudaEvent_t a_ = nullptr, b_ = nullptr;
};

// ---- device status word -------------------------------------------------------------
// Codes a kernel may record (first writer wins).
// DEV_RANGE: an input outside a kernel's documented domain (the scan's backward: a
// 32-token chunk whose decay on some key channel is 80 or more in natural-log units).
enum : int { DEV_OK = 0, DEV_TIMEOUT = 1, DEV_RANGE = 2 };
// Address of this device's status word (set up once per device; thread-safe).
int* device_status_ptr();

// ---- launchers (each returns cudaGetLastError() of its launches) ------------------
struct KdaArgs {
    const void *q, *k, *v, *g, *beta;
    const float* S0;
    void* o;
    float* ST;
    int B, T, H, Dk, Dv, chunk;
    ElemType in_t;   // q, k, v
    ElemType out_t;  // o
    ElemType gb_t;   // g, beta
    // output side of Eq. 15 (gated path only): o <- Sigmoid(gate) * gamma * RMSNorm(o)
    const void* gate = nullptr;   // [B,T,H,Dv], dtype of q (nullptr: plain readout)
    const float* gamma = nullptr; // [H,Dv] fp32 or nullptr (ones)
    float eps = 0.f;
};

// In-place gated RMSNorm of o (a.gate != nullptr), one warp per (token, head).
cudaError_t launch_gate_rmsnorm(const KdaArgs& a, cudaStream_t s);

// Generic chunkwise scan on CUDA cores in fp32 (any supported dtype/shape).
cudaError_t launch_kda_generic(const KdaArgs& a, cudaStream_t s);

// Tensor-core path (bf16, Dk = Dv = 128).  Workspace bytes it needs:
size_t kda_tc_workspace_bytes(int B, int T, int H, int chunk, int num_sms);
bool kda_tc_supported(const KdaArgs& a);
// The uniform-batch split of the tensor-core path: P segments of L chunks per head (P = 1:
// one pass per head; otherwise the output pass of segment 0 runs beside the state pass of
// segments 1..P-2, and the output pass of segments 1..P-1 follows the combine).
void kda_tc_plan(int B, int T, int H, int num_sms, int* P, int* L);
cudaError_t launch_kda_tc(const KdaArgs& a, void* ws, size_t ws_bytes, int* status,
                          cudaStream_t s);
// Packed samples: a.B = 1, a.T = cu[n] tokens; host array cu[0..n] of sample offsets.
size_t kda_tc_varlen_workspace_bytes(const int* cu, int n, int H, int num_sms);
cudaError_t launch_kda_tc_varlen(const KdaArgs& a, const int* cu, int n, void* ws, int* status, cudaStream_t s);
// One shard of a sequence cut across devices (a.B rows of a.T tokens each).  The state
// pass over all of the shard's P segments leaves the per-segment maps in the workspace:
// head bh's segments 0..P-2 at maps + (bh*(P-1) + p)*2*D*D, its last segment at
// tail + bh*2*D*D ([N | M] blocks of D x D fp32 each).  The output pass then takes the
// shard's entry state as a.S0 and reuses those maps.
struct TcShardMaps {
    int P;
    const float* maps;
    const float* tail;
};
size_t kda_tc_sp_workspace_bytes(int B, int T, int H, int num_sms);
cudaError_t launch_kda_tc_sp_state(const KdaArgs& a, void* ws, int* status, cudaStream_t s, TcShardMaps* out);
cudaError_t launch_kda_tc_sp_output(const KdaArgs& a, void* ws, int* status, cudaStream_t s);

// Backward of the scan (fp32 on CUDA cores, any supported dtype / Dk / Dv): gradients
// in fp32; dq, dk, dg, dbeta are zeroed and then accumulated by the launch.
struct KdaBwdArgs {
    const void *q, *k, *v, *g, *beta;
    const float* S0;
    const void* dout;
    const float* dST;
    float *dq, *dk, *dv, *dg, *dbeta, *dS0;
    int B, T, H, Dk, Dv;
    ElemType in_t, do_t;
    int* status;   // device status word (DEV_RANGE is recorded here)
};
size_t kda_bwd_workspace_bytes(int B, int T, int H, int Dk, int Dv);
cudaError_t launch_kda_bwd(const KdaBwdArgs& a, void* ws, cudaStream_t s);

struct ConvSeg {
    int32_t modality;
    int64_t start;
    int32_t F, Hgt, Wid, weight_set;
};
// Depthwise modality-aware conv of one segment; optional per-head L2 normalisation
// (head width D, 0 = none).  x, y: [B,T,C].
cudaError_t launch_conv_segment(const void* x, void* y, int B, int T, int C, ElemType in_t,
                                ElemType out_t, const ConvSeg& seg, int Kt, const float* w,
                                int norm_D, cudaStream_t s);
// The same for nt <= 3 tensors sharing the segment (weights ws[i], norm width norm_Ds[i]);
// image and video segments of bf16 input go to one launch of the tiled kernel.
cudaError_t launch_conv_segment_multi(int nt, const void* const* xs, void* const* ys, int B, int T, int C,
                                      ElemType in_t, ElemType out_t, const ConvSeg& seg, int Kt,
                                      const float* const* ws, const int* norm_Ds, cudaStream_t s);

// Backward of the conv of one segment: dx over the segment's tokens (written), dw (this
// segment's weight set, accumulated with atomics; nullptr = skip).  x, dy: [B,T,C] in_t.
cudaError_t launch_conv_backward_segment(const void* x, const void* dy, float* dx, const float* w, float* dw, int B,
                                         int T, int C, ElemType in_t, const ConvSeg& seg, int Kt, cudaStream_t s);

// Elementwise pieces of the fused backward: widen to fp32 (bf16/fp16/fp32 source), and
// per-row unit norm of rows of D values and its derivative (in place on d).
cudaError_t launch_to_f32(const void* x, ElemType t, float* y, int64_t n, cudaStream_t s);
cudaError_t launch_l2norm_rows(const float* x, float* y, int64_t rows, int D, cudaStream_t s);
cudaError_t launch_l2norm_bwd_rows(const float* x, float* d, int64_t rows, int D, cudaStream_t s);

}  // namespace kda
