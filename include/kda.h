/*
 * kda.h -- C ABI of libkda: the Kimi Delta Attention (KDA) forward scan and the
 * modality-aware short convolution (mShortConv) that feeds it, for NVIDIA B200
 * (sm_100a).
 *
 * The operations are those of the Chimera paper ("Chimera: hybrid attention +
 * Chinchilla scaling", pchao.org translation):
 *   - section 3.3, Eq. 14 -- per head, with S_t in R^{Dk x Dv} the state AFTER token t,
 *         S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
 *     alpha_t in (0,1)^{Dk} a per-key-channel forget gate, beta_t in (0,1) one scalar
 *     per head and token; the parenthesisation (decay, then erase, then write) is the
 *     one printed in LaTeX by the agifrontier summary of the paper;
 *   - section 3.3, Eq. 15 (inner term) -- the readout o_t = S_t^T q_t;
 *   - section 3.3 -- the state restarts from S_0 = 0 at a packed-sample boundary
 *     (here: at the start of every batch row, or from the caller's S0);
 *   - section 3.3, Eq. 13 and section 3.4 -- (Q,K,V) = mShortConv(...): a depthwise
 *     convolution applied inside each modality segment of the packed stream, causal
 *     1-D for text, 3x3 spatial for an image, 3x3x3 for video (causal in time,
 *     symmetric in space, per the agifrontier summary), with visual tokens in the
 *     time-first raster order of Eq. 12, m = f*H*W + r*W + c.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller, contiguous,
 *     token-major; the library never frees or retains them.
 *   - Calls are asynchronous on `stream` (NULL = the legacy default stream).
 *     Argument errors are detected on the host and returned before any launch.
 *     Launch failures return KDA_ERR_CUDA.  Faults detected by the kernels on the
 *     device (a bounded wait that ran out; an input outside the backward's decay domain)
 *     are recorded in a per-device status word read by kda_last_device_error() after the
 *     caller synchronises.
 *   - Floating point: inputs are bf16 or fp32 (kda_dtype); all accumulation and the
 *     recurrent state are fp32.  The fp32 path computes in fp32 on CUDA cores; the
 *     bf16 path converts its tiles on chip to fp16 tensor-core operands (11-bit
 *     significand) with fp32 accumulation.
 *   - CUDA graphs: the forward calls (except kda_forward_varlen), the backward calls,
 *     kda_sp_prefix and kda_sp_output enqueue only launches, memsets, device copies and
 *     event waits, so a stream capture can record them once the first call on the device
 *     has run outside capture (it creates per-device resources) and given a workspace
 *     (a NULL workspace is allocated stream-ordered inside the call).
 *     kda_forward_varlen and kda_sp_transition copy a host-planned work table to the
 *     device in every call and cannot be captured.
 *   - The gate is passed as g = ln(alpha) (g <= 0, finite), not as alpha: alpha close
 *     to 1 is not representable in bf16 (the spacing just below 1 is 2^-8), while its
 *     logarithm is.
 *   - No 1/sqrt(Dk) scaling and no normalisation happen inside kda_forward; q and k
 *     are used as given.
 */
#ifndef LIBKDA_KDA_H
#define LIBKDA_KDA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; declared here so the header needs no CUDA include. */
typedef struct CUstream_st* kda_stream_t;

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,   /* null pointer, negative size, bad segment table, ... */
    KDA_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. Dk not in {32,64,128}) */
    KDA_ERR_CUDA = 3,          /* a CUDA runtime call or kernel launch failed */
    KDA_ERR_TIMEOUT = 4,       /* device side: a bounded wait ran out (see kda_last_device_error) */
    KDA_ERR_WORKSPACE = 5      /* caller-provided workspace smaller than required */
} kda_status;

typedef enum { KDA_F32 = 0, KDA_BF16 = 1 } kda_dtype;

/* Human-readable name of a status code (static storage, never NULL). */
const char* kda_status_string(kda_status s);

/* Reads and clears the calling thread's current device's status word, in which
 * kernels record device-side failures (KDA_OK if none; the first one recorded wins):
 * KDA_ERR_TIMEOUT (a bounded wait ran out), KDA_ERR_UNSUPPORTED (kda_backward or
 * kda_mshortconv_backward met a chunk outside its decay domain).  Synchronous: it waits
 * for all work on the device to finish. */
kda_status kda_last_device_error(void);

/* Bytes of device workspace kda_forward needs for this problem (0 if none).  The
 * value depends only on the arguments and the current device's SM count. */
size_t kda_forward_workspace_size(int B, int T, int H, int Dk, int Dv, kda_dtype dtype,
                                  kda_dtype o_dtype, int chunk);

/*
 * kda_forward -- KDA forward scan (Eq. 14) with readout o_t = S_t^T q_t (Eq. 15).
 *
 *   q, k, g : [B, T, H, Dk]  dtype          g = ln(alpha), finite, <= 0 (any such value:
 *                                            a per-channel decay as strong as alpha =
 *                                            e^-80 on single tokens is computed, no range
 *                                            is rejected)
 *   v       : [B, T, H, Dv]  dtype          on the tensor-core path (bf16, Dk = Dv = 128,
 *                                            chunk 64) the MMA operands are fp16, so the
 *                                            entries of v, of the state and of the
 *                                            pseudo-values must stay below ~6e4 in
 *                                            magnitude (beyond, o is not finite); the
 *                                            fp32 CUDA-core path has no such limit
 *   beta    : [B, T, H]      dtype          erase/write strength, one per (token, head)
 *   S0      : [B, H, Dk, Dv] fp32, or NULL  initial state (NULL = zeros)
 *   o       : [B, T, H, Dv]  o_dtype        written for every token
 *   S_T     : [B, H, Dk, Dv] fp32, or NULL  final state (NULL = not written)
 *   Dk, Dv  : each in {32, 64, 128}
 *   o_dtype : KDA_BF16 or KDA_F32.  The output is accumulated in fp32 and rounded
 *             once to o_dtype (round to nearest even); a bf16 o is exactly the fp32 o
 *             of the same call rounded.  (bf16 output rounding alone is up to 2^-9 of
 *             |o|, which for heavy-tailed outputs exceeds a few percent of RMS(o).)
 *   chunk   : tokens per chunk of the chunkwise evaluation: 0 = the default for
 *             the dtype (64 for bf16, 16 for fp32), else one of {16, 32, 64, 128}.  The
 *             result does not depend on it beyond rounding.  The tensor-core kernel runs
 *             chunk 64 only; any other chunk runs on the fp32 CUDA-core kernels (128 on
 *             one that takes the key channels in blocks of 32), which are much slower.
 *   workspace, workspace_bytes : device scratch of at least
 *             kda_forward_workspace_size(...) bytes, 256-byte aligned; or NULL, in
 *             which case the library takes and returns it with cudaMallocAsync /
 *             cudaFreeAsync on `stream`.  The workspace must not be used by
 *             another call that may run concurrently.
 *
 * Batch rows are independent scans (each starts from its S0 slice or zero).  T may
 * be any non-negative length (0: o untouched, S_T = S0).  o must not alias an input.
 */
kda_status kda_forward(const void* q, const void* k, const void* v, const void* g,
                       const void* beta, const float* S0, void* o, float* S_T,
                       int B, int T, int H, int Dk, int Dv, kda_dtype dtype,
                       kda_dtype o_dtype, int chunk, void* workspace, size_t workspace_bytes,
                       kda_stream_t stream);

/* Size of the scratch array compiled into the library for kda_forward_noalloc. */
#define KDA_NOALLOC_SCRATCH_BYTES (32u << 20)

/*
 * kda_forward_gated -- kda_forward followed by the output side of Eq. 15 (Chimera
 * paper, section 3.3) before the output projection W_o:
 *     y[b,t,h,:] = Sigmoid(gate[b,t,h,:]) * gamma[h,:] * r / sqrt(mean(r^2) + eps),
 *     r = S_t^T q_t (the readout kda_forward would write), mean over the head's Dv values.
 *   gate  : [B,T,H,Dv] device, dtype `dtype`; the pre-sigmoid values W_gate x (the
 *           projection itself is outside this library).  Required when B*T > 0.
 *   gamma : [H,Dv] fp32 device, the RMSNorm gain per head; NULL = all ones.
 *   eps   : >= 0 and finite; a row with mean(r^2) + eps == 0 yields zeros.
 *   o     : receives y (o_dtype).  Every other argument, the workspace and the errors
 *           are those of kda_forward; S_T is unaffected by the epilogue.
 * On the tensor-core path with a bf16 output the epilogue runs inside the scan's output
 * stage (r never reaches global memory); otherwise a separate kernel rewrites o in place.
 */
kda_status kda_forward_gated(const void* q, const void* k, const void* v, const void* g,
                             const void* beta, const float* S0, const void* gate, const float* gamma,
                             float eps, void* o, float* S_T, int B, int T, int H, int Dk, int Dv,
                             kda_dtype dtype, kda_dtype o_dtype, int chunk, void* workspace,
                             size_t workspace_bytes, kda_stream_t stream);

/*
 * kda_forward_varlen -- kda_forward over packed samples: n_seqs sequences laid end to end
 * on one token axis, the state reset at the start of every sample (Eq. 14 runs from S0
 * of that sample, section 3.3: a sample starts from the zero state).
 *   cu_seqlens : HOST array of n_seqs + 1 int32 offsets, cu_seqlens[0] = 0, non-decreasing;
 *                sample i is tokens [cu_seqlens[i], cu_seqlens[i+1]) (empty samples allowed).
 *   q, k, g    : [T_total, H, Dk] with T_total = cu_seqlens[n_seqs]; v, o: [T_total, H, Dv];
 *   beta       : [T_total, H];  all device memory, dtypes as for kda_forward.
 *   S0, S_T    : [n_seqs, H, Dk, Dv] fp32 or NULL (zeros / not written); an empty
 *                sample's S_T is its S0.
 *   workspace  : as for kda_forward, sized by kda_forward_varlen_workspace_size (which
 *                depends on the offsets).
 * Errors as for kda_forward; bad offsets give KDA_ERR_INVALID_ARG.
 */
size_t kda_forward_varlen_workspace_size(const int32_t* cu_seqlens, int n_seqs, int H, int Dk, int Dv,
                                         kda_dtype dtype, kda_dtype o_dtype, int chunk);
kda_status kda_forward_varlen(const void* q, const void* k, const void* v, const void* g, const void* beta,
                              const float* S0, void* o, float* S_T, const int32_t* cu_seqlens, int n_seqs,
                              int H, int Dk, int Dv, kda_dtype dtype, kda_dtype o_dtype, int chunk,
                              void* workspace, size_t workspace_bytes, kda_stream_t stream);

/*
 * kda_forward_noalloc -- kda_forward that allocates no device memory.  The paper has
 * no counterpart to this call; it exists for callers that cannot allocate during a
 * call: code inside a host framework that owns all device memory through its own
 * allocator and forbids raw allocation in its call path (inference-engine plugins,
 * serving loops on a fixed memory plan), or code that must not risk an allocation
 * failing or stalling mid-call.
 *
 * Same arguments and results as kda_forward, minus the workspace.  Its scratch comes
 * from one array of KDA_NOALLOC_SCRATCH_BYTES compiled into the library, held in the
 * device memory of every GPU on which the library is loaded until the process exits.
 *   - The first call on a device looks up that array's device address (once per
 *     device, with the device current) and, when the tensor-core split has more than
 *     one segment, creates the auxiliary stream and two events of its first wave (see
 *     kda_forward_plan); make that first call before any stream capture.
 *   - All calls on a device share the array and it keeps the last call's contents.
 *     Every byte a call reads from it is written earlier in the same call, so nothing
 *     needs clearing; calls whose GPU work may overlap (different streams without
 *     ordering between them) race on it.
 *   - A problem whose scratch need exceeds KDA_NOALLOC_SCRATCH_BYTES returns
 *     KDA_ERR_WORKSPACE before any launch (on a 148-SM B200 every shape fits: the
 *     need is at most about 28 MiB).
 */
kda_status kda_forward_noalloc(const void* q, const void* k, const void* v, const void* g,
                               const void* beta, const float* S0, void* o, float* S_T,
                               int B, int T, int H, int Dk, int Dv, kda_dtype dtype,
                               kda_dtype o_dtype, int chunk, kda_stream_t stream);

/*
 * Sequence-parallel forward: each of the B rows is cut along time into R consecutive
 * shards, one per device (the paper runs one long stream per device and names no
 * multi-device scheme; this follows from Eq. 14 of section 3.3 being affine in the
 * state).  Over a shard, S_out = M S_in + N with
 *   M = prod_t (I - beta_t k_t k_t^T) Diag(alpha_t)   (latest token leftmost), [D, D]
 *   N = the state the shard reaches from S_in = 0,    [D, D]  (state layout [Dk, Dv])
 * A rank r runs kda_sp_transition on its shard, the ranks exchange the [N | M] blocks
 * (an all-gather: the library does no communication), kda_sp_prefix folds shards
 * 0..r-1 over the row's S0 into the shard's entry state, and kda_sp_output scans the
 * shard from it.  Concatenating the ranks' o gives kda_forward's o of the whole rows;
 * the last rank's S_T is the rows' final state.  Dk = Dv = D in {32, 64, 128}; the
 * other arguments are as for kda_forward on the shard ([B, T_r, H, D] tensors).
 *
 * kda_sp_workspace_size -- bytes of device workspace kda_sp_transition and
 *   kda_sp_output need (0 if none).  The workspace is required (the calls allocate
 *   nothing), 256-byte aligned, and is the same buffer for both calls of a shard.
 */
size_t kda_sp_workspace_size(int B, int T, int H, int D, kda_dtype dtype, int chunk);

/*
 * kda_sp_transition -- this shard's affine map.
 *   MN : [B, H, 2, D, D] fp32 (device, written): block 0 = N, block 1 = M, row-major,
 *        so S_out[i][j] = sum_c M[i][c] S_in[c][j] + N[i][j].
 * On the tensor-core route the per-segment maps of the shard stay in the workspace for
 * kda_sp_output: pass that call the same workspace, unmodified, and the same q, k, v, g,
 * beta.  T = 0 gives N = 0, M = I.  Errors: KDA_ERR_INVALID_ARG (null tensor, bad
 * sizes), KDA_ERR_UNSUPPORTED (D, chunk, B*H > 65535), KDA_ERR_WORKSPACE (workspace null
 * or smaller than kda_sp_workspace_size), KDA_ERR_CUDA.
 */
kda_status kda_sp_transition(const void* q, const void* k, const void* v, const void* g,
                             const void* beta, float* MN, int B, int T, int H, int D,
                             kda_dtype dtype, int chunk, void* workspace,
                             size_t workspace_bytes, kda_stream_t stream);

/*
 * kda_sp_prefix -- the entry state of shard r:
 *   S_in = (M_{r-1} (... (M_0 S0 + N_0) ...) + N_{r-1})
 *   MN_all : [R, B, H, 2, D, D] fp32 (device): every rank's kda_sp_transition result,
 *            in rank order (may be NULL when r = 0).
 *   S0     : [B, H, D, D] fp32 or NULL (zeros) -- the rows' initial state.
 *   S_in   : [B, H, D, D] fp32 (device, written).
 * Errors: KDA_ERR_INVALID_ARG (r outside [0, R), null S_in), KDA_ERR_UNSUPPORTED (D),
 * KDA_ERR_CUDA.
 */
kda_status kda_sp_prefix(const float* MN_all, int R, int r, const float* S0, float* S_in,
                         int B, int H, int D, kda_stream_t stream);

/*
 * kda_sp_output -- the scan of this shard from S_in (as kda_forward with S0 = S_in):
 * o [B, T, H, D] in o_dtype and, if S_T is not NULL, the shard's final state.  On the
 * tensor-core route it reads the segment maps kda_sp_transition left in the workspace
 * (one output pass instead of a full scan); otherwise it runs the whole scan.
 * Errors: as kda_sp_transition.
 */
kda_status kda_sp_output(const void* q, const void* k, const void* v, const void* g,
                         const void* beta, const float* S_in, void* o, float* S_T,
                         int B, int T, int H, int D, kda_dtype dtype, kda_dtype o_dtype,
                         int chunk, void* workspace, size_t workspace_bytes,
                         kda_stream_t stream);

/*
 * kda_backward -- gradients of the scan of kda_forward (the paper gives only the forward;
 * this is its reverse-mode derivative).  For a loss L with dL/do = d_o and dL/dS_T = dS_T:
 *   q, k, v, g, beta, S0, B, T, H, Dk, Dv, dtype : exactly as passed to kda_forward.
 *   d_o   : [B, T, H, Dv] in do_dtype (device).
 *   dS_T  : [B, H, Dk, Dv] fp32 or NULL (zeros).
 *   dq, dk, dg : [B, T, H, Dk] fp32 (device, written);  dv : [B, T, H, Dv] fp32;
 *   dbeta : [B, T, H] fp32;  dS0 : [B, H, Dk, Dv] fp32 or NULL (not written).
 * The gradient of g is that of the natural-log decay (alpha = e^g).  The call reruns
 * the forward to store each 32-token chunk's entry state and chunk factors in the
 * workspace (kda_backward_workspace_size bytes: B*H*ceil(T/32)*(Dk*Dv + Dv/16*2048)*4),
 * then sweeps the chunks in
 * reverse; arithmetic is fp32.  Per key channel the decay over each 32-token chunk
 * (tokens 32n .. 32n+31 of a row) must satisfy |sum g| < 80.  A call with a chunk beyond
 * that still runs, but its gradients are not finite and kda_last_device_error() then
 * returns KDA_ERR_UNSUPPORTED (the device records it; the host sees it after a sync).
 * workspace: as for kda_forward (NULL: a stream-ordered allocation inside the call).
 * Errors: KDA_ERR_INVALID_ARG (null tensor with work to do, bad sizes or dtypes),
 * KDA_ERR_UNSUPPORTED (Dk or Dv outside {32, 64, 128}; B or H > 65535),
 * KDA_ERR_WORKSPACE, KDA_ERR_CUDA.
 */
size_t kda_backward_workspace_size(int B, int T, int H, int Dk, int Dv);
kda_status kda_backward(const void* q, const void* k, const void* v, const void* g,
                        const void* beta, const float* S0, const void* d_o,
                        const float* dS_T, float* dq, float* dk, float* dv, float* dg,
                        float* dbeta, float* dS0, int B, int T, int H, int Dk, int Dv,
                        kda_dtype dtype, kda_dtype do_dtype, void* workspace,
                        size_t workspace_bytes, kda_stream_t stream);

/* Modalities of a packed-stream segment (section 3.4). */
typedef enum { MSC_TEXT = 0, MSC_IMAGE = 1, MSC_VIDEO = 2 } msc_modality;

/* One modality segment of a packed row.  The same table applies to every batch
 * row.  Tokens of the segment are [start, start + len) with len = Wid (text),
 * Hgt*Wid (image) or F*Hgt*Wid (video, time-first raster order, Eq. 12).
 * weight_set selects the kernel among the sets of that modality. */
typedef struct {
    int32_t modality;     /* msc_modality */
    int32_t reserved;     /* must be 0 */
    int64_t start;
    int32_t F, Hgt, Wid;  /* text: F = Hgt = 1, Wid = length; image: F = 1 */
    int32_t weight_set;
} msc_segment;

/*
 * mshortconv_forward -- depthwise modality-aware short convolution (section 3.4).
 *
 *   x, y     : [B, T, C] dtype (device).  y must not alias x.
 *   segs     : HOST array of n_segs segments, in increasing start order, without
 *              overlap, inside [0, T).  Tokens covered by no segment get y = 0.
 *   Kt       : text kernel length, 1..8.
 *   w_text   : [n_text_sets, C, Kt] fp32 (device); y[t] = sum_j w[c,j] x[t-(Kt-1)+j]
 *   w_image  : [n_image_sets, C, 3, 3] fp32;  y[r,s] = sum_{a,e} w[c,a,e] x[r-1+a, s-1+e]
 *   w_video  : [n_video_sets, C, 3, 3, 3] fp32;
 *              y[f,r,s] = sum_{tau,a,e} w[c,tau,a,e] x[f-2+tau, r-1+a, s-1+e]
 *              Positions outside the segment (before its first token/frame, outside
 *              its grid) read as zero: no kernel crosses a segment boundary.
 *   n_*_sets : number of weight sets of each modality (bounds weight_set).
 * A weight pointer may be NULL only if no segment uses that modality.  C must be a
 * multiple of 8.  No bias, no activation.
 */
kda_status mshortconv_forward(const void* x, void* y, int B, int T, int C, kda_dtype dtype,
                              const msc_segment* segs, int n_segs, int Kt,
                              const float* w_text, int n_text_sets,
                              const float* w_image, int n_image_sets,
                              const float* w_video, int n_video_sets,
                              kda_stream_t stream);

/*
 * mshortconv_backward -- gradients of mshortconv_forward (section 3.4; the paper gives only
 * the forward).  For a loss L with dL/dy = dy:
 *   x, dy    : [B, T, C] dtype (device); x is read only for the weight gradients.
 *   dx       : [B, T, C] fp32 (device, written; 0 at tokens no segment covers).
 *   segs ... w_video, n_*_sets : exactly as passed to mshortconv_forward.
 *   dw_text, dw_image, dw_video : fp32 with the layouts of w_text, w_image, w_video
 *              (device, written: zeroed, then summed over rows and segments), or NULL
 *              to skip that modality's weight gradient.
 * Inside a segment y[p] = sum_tap w[c,tap] x[p + off(tap)], so dx[p] = sum_tap w[c,tap]
 * dy[p - off(tap)] and dw[c,tap] = sum_{rows,p} dy[p] x[p + off(tap)], with positions
 * outside the segment reading zero.  Errors: as mshortconv_forward.
 */
kda_status mshortconv_backward(const void* x, const void* dy, float* dx, int B, int T, int C,
                               kda_dtype dtype, const msc_segment* segs, int n_segs, int Kt,
                               const float* w_text, int n_text_sets,
                               const float* w_image, int n_image_sets,
                               const float* w_video, int n_video_sets,
                               float* dw_text, float* dw_image, float* dw_video,
                               kda_stream_t stream);

/* Bytes of workspace kda_mshortconv_forward needs. */
size_t kda_mshortconv_workspace_size(int B, int T, int H, int D, kda_dtype dtype,
                                     kda_dtype o_dtype, int chunk);

/*
 * kda_mshortconv_forward -- Eq. 13 feeding Eq. 14: q = L2norm_h(mShortConv(x_q)),
 * k = L2norm_h(mShortConv(x_k)), v = mShortConv(x_v), then kda_forward(q,k,v,g,beta).
 *
 *   xq, xk, xv : [B, T, H*D] dtype (device), the projected inputs before the conv.
 *   segs, n_segs, Kt : as for mshortconv_forward (one table for all three tensors).
 *   wq, wk, wv : each an array of 3 device pointers {w_text, w_image, w_video} with
 *                the layouts of mshortconv_forward and ONE weight set per modality.
 *   L2norm_h   : per (token, head) division by the Euclidean norm of the D channels
 *                of that head (no epsilon; an all-zero vector stays zero).
 *   g, beta, S0, o, S_T, o_dtype, chunk : as for kda_forward with Dk = Dv = D.
 *   q, k, v are kept between the conv and the scan in the workspace as fp16 for
 *   bf16 inputs (fp32 for fp32 inputs).
 *   workspace  : as for kda_forward, sized by kda_mshortconv_workspace_size.
 */
kda_status kda_mshortconv_forward(const void* xq, const void* xk, const void* xv,
                                  const msc_segment* segs, int n_segs, int Kt,
                                  const float* const wq[3], const float* const wk[3],
                                  const float* const wv[3],
                                  const void* g, const void* beta, const float* S0,
                                  void* o, float* S_T, int B, int T, int H, int D,
                                  kda_dtype dtype, kda_dtype o_dtype, int chunk,
                                  void* workspace, size_t workspace_bytes,
                                  kda_stream_t stream);

/*
 * kda_mshortconv_backward -- gradients of kda_mshortconv_forward (the paper gives only the
 * forward): for dL/do = d_o and dL/dS_T = dS_T, the gradients of x_q, x_k, x_v, of the
 * three tensors' conv weights, of g, beta and S0.
 *   xq ... D, dtype : exactly as passed to kda_mshortconv_forward.
 *   d_o   : [B, T, H, D] in do_dtype;  dS_T : [B, H, D, D] fp32 or NULL (zeros).
 *   dxq, dxk, dxv : [B, T, H*D] fp32 (written).
 *   dwq, dwk, dwv : each an array of 3 pointers {text, image, video}, fp32 with the
 *                   layouts of wq[i] (one weight set), or NULL entries to skip.
 *   dg : [B, T, H, D] fp32;  dbeta : [B, T, H] fp32;  dS0 : [B, H, D, D] fp32 or NULL.
 * The chain rule runs in fp32: the conv outputs are recomputed, q and k normalised, the
 * scan's backward (as kda_backward) gives dq, dk, dv, the norm's derivative
 * dy = (dq - q (q . dq)) / |y| per (token, head) (0 where |y| = 0) maps dq, dk back, and
 * the conv backward (as mshortconv_backward) gives dx and the weight gradients.
 * workspace: kda_mshortconv_backward_workspace_size bytes (NULL: allocated in the call).
 * Errors: as kda_backward and mshortconv_backward.
 */
size_t kda_mshortconv_backward_workspace_size(int B, int T, int H, int D, kda_dtype dtype);
kda_status kda_mshortconv_backward(const void* xq, const void* xk, const void* xv,
                                   const msc_segment* segs, int n_segs, int Kt,
                                   const float* const wq[3], const float* const wk[3],
                                   const float* const wv[3], const void* g, const void* beta,
                                   const float* S0, const void* d_o, kda_dtype do_dtype,
                                   const float* dS_T, float* dxq, float* dxk, float* dxv,
                                   float* const dwq[3], float* const dwk[3], float* const dwv[3],
                                   float* dg, float* dbeta, float* dS0, int B, int T, int H, int D,
                                   kda_dtype dtype, void* workspace, size_t workspace_bytes,
                                   kda_stream_t stream);

/* ---- diagnostics ---------------------------------------------------------------- */

/* How kda_forward (ungated) splits a uniform batch on the tensor-core path on the current
 * device: each head's ceil(T/64) chunks form *segments runs; segments 1.. hold
 * *chunks_per_segment chunks each (the last may be shorter), or, with three or more
 * segments where that shortens them, segments 1.. hold exactly *chunks_per_segment and
 * segment 0 the rest, up to 4% more (its output pass runs beside the state pass of the
 * others, whose chunks cost ~4% more).  With more than one segment, segment 0's output pass
 * ("kda_tc_output_first") runs beside the state pass of segments 1..P-2 ("kda_tc_state"),
 * and the output pass of segments 1..P-1 ("kda_tc_output") follows the combine
 * ("kda_tc_combine").  Both are 0 when the call would not take the tensor-core path.
 * The first kda_forward on a device with more than one segment creates an auxiliary
 * stream and two events for that overlap; make it before any stream capture.
 * Returns KDA_ERR_INVALID_ARG for null outputs or bad sizes. */
kda_status kda_forward_plan(int B, int T, int H, int Dk, int Dv, kda_dtype dtype,
                            kda_dtype o_dtype, int chunk, int* segments,
                            int* chunks_per_segment);

/* Number of kernels this library has launched in this process (all devices). */
uint64_t kda_kernel_launches(void);

/* Test hook for the device-side failure path (the paper has no counterpart; this is
 * how the timeout handling is exercised without a fault or a hang).  While `on` is
 * non-zero, every later launch of the tensor-core scan withholds, in each CTA, the
 * first "every tile of the chunk ready" signal to the warps that run the state chain.
 * Their bounded wait (2 s) then runs out: the CTA records the timeout in the device
 * status word, stops waiting, drains its own tensor-core and TMA work, frees its tensor
 * memory and exits.  The call still returns KDA_OK (errors on the device are reported
 * asynchronously); o and S_T are undefined; kda_last_device_error() then returns
 * KDA_ERR_TIMEOUT, and later calls with the hook off run normally.  Off by default;
 * process-wide; not for production use. */
void kda_debug_drop_handoff(int on);

/* Measures this GPU's fp32 fused-multiply-add rate (FMAs per second) with a synthetic
 * kernel of independent FMA chains on every SM, timed with CUDA events on the default
 * stream (synchronous; allocates 4 bytes).  It is the denominator of the conv's
 * plain-ALU roofline in the benchmark; the paper has no counterpart.  Returns 0, or -1
 * on a CUDA error. */
int kda_fma_probe(double* fma_per_s);

/* When `on` is non-zero, every later call records a pair of CUDA events on its
 * stream around each of its kernels, keyed by kernel name.  Off by default. */
void kda_profile_enable(int on);

/* Waits for the recorded events and returns, for kernel `name`, the summed
 * device time in milliseconds and the number of launches timed since the last
 * collection; clears that kernel's record.  Returns 0, or -1 if `name` has no
 * record.  Names: "kda_generic", "kda_tc_state", "kda_tc_combine",
 * "kda_tc_output", "kda_tc_output_first", "conv", "gate_norm", "kda_sp_fold",
 * "kda_bwd", "conv_bwd". */
int kda_profile_collect(const char* name, double* total_ms, int* launches);

#ifdef __cplusplus
}
#endif
#endif /* LIBKDA_KDA_H */
