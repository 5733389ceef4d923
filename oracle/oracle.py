"""fp64 CPU oracle for the KDA forward scan and mShortConv -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may
import this module.  The product path (the CUDA library and its Python binding) never
does, and shares no code with it.

The arithmetic lives in ``kda_oracle.c`` (plain loops in double precision); this file
only builds it with gcc and marshals arrays.  What each routine computes, and the
passages of the Chimera paper it follows, is stated in that file's header:

* ``kda_forward``: Eq. 14 of the paper, section 3.3 (decay, rank-one erase, write, in
  that order), read out as o_t = S_t^T q_t with S_t the state after token t.
* ``mshortconv``: section 3.4 -- per-segment depthwise conv, 1-D causal for text,
  3x3 spatial for an image, 3x3x3 causal-in-time / symmetric-in-space for video,
  zero padding inside each segment, time-first raster order of Eq. 12.
* ``l2norm_heads``: unit-norm rows per head (no epsilon; zero stays zero).
* ``kda_forward_varlen``: packed samples on one token axis, each scanned from its own
  S0 (zero by default): the reset at a sample start of section 3.3.
* ``gated_rmsnorm`` / ``kda_forward_gated``: the output side of Eq. 15 (section 3.3),
  Sigmoid(gate) * RMSNorm(S_t^T q_t) per (token, head), before the output projection
  W_o (numpy, fp64).
* ``mshortconv_backward``: the adjoint of ``mshortconv`` (linear in x and in w): dx and
  the weight gradients per modality, by the same per-segment taps read backwards (numpy,
  fp64).
* ``l2norm_heads_backward`` / ``fused_backward``: the derivative of the per-head unit
  normalisation and the chain rule through the fused forward (conv -> norm -> scan),
  composed from the other backward routines (numpy, fp64).
* ``kda_backward``: the reverse-mode derivative of the token recurrence of Eq. 14 with
  the readout of Eq. 15 (the paper gives only the forward; the paper trains with it).
  Plain reverse sweep over the tokens in fp64 (numpy), from the states of a forward
  sweep.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

DT_F32, DT_BF16, DT_F64 = 0, 1, 2
MOD_TEXT, MOD_IMAGE, MOD_VIDEO = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile kda_oracle.c into liboracle.so next to it (gcc, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class Segment(ctypes.Structure):
    _fields_ = [("modality", ctypes.c_int32), ("pad0", ctypes.c_int32),
                ("start", ctypes.c_int64), ("F", ctypes.c_int32), ("Hgt", ctypes.c_int32),
                ("Wid", ctypes.c_int32), ("weight_set", ctypes.c_int32)]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P, I, L = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
            lib.oracle_kda_forward.restype = I
            lib.oracle_kda_forward.argtypes = [P, P, P, P, P, I, P, P, L, L, L, P,
                                               I, I, I, I, I, P, I, I]
            lib.oracle_mshortconv.restype = I
            lib.oracle_mshortconv.argtypes = [P, I, P, I, I, I, I, I, P, I, I, P, P, P, I]
            lib.oracle_l2norm_heads.restype = None
            lib.oracle_l2norm_heads.argtypes = [P, L, I, I]
            _lib = lib
    return _lib


def default_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return max(1, os.cpu_count() or 1)


def _as_input(a):
    """Return (contiguous numpy array, dtype code) holding the values at stored precision.

    Accepts numpy arrays (float32 / float64) or torch CPU tensors (float32, bfloat16,
    float64).  bf16 is passed as its raw 16-bit patterns; the C side widens them
    exactly."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().contiguous().cpu()
            if a.dtype == torch.bfloat16:
                return a.view(torch.int16).numpy().view(np.uint16), DT_BF16
            if a.dtype == torch.float32:
                return a.numpy(), DT_F32
            if a.dtype == torch.float64:
                return a.numpy(), DT_F64
            raise TypeError(f"unsupported tensor dtype {a.dtype}")
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(a)
    if a.dtype == np.float32:
        return a, DT_F32
    if a.dtype == np.float64:
        return a, DT_F64
    if a.dtype == np.uint16:
        return a, DT_BF16
    raise TypeError(f"unsupported array dtype {a.dtype}")


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def kda_forward(q, k, v, g, beta, S0=None, *, pairs=None, want_o=True, nthreads=None):
    """Token-by-token KDA scan in fp64.

    q, k, g: [B,T,H,Dk]; v: [B,T,H,Dv]; beta: [B,T,H]; S0: [B,H,Dk,Dv] or None (zeros).
    All five inputs must share one storage dtype.  ``pairs`` optionally restricts the
    work to a list of (b, h) pairs; outputs of other pairs are left at zero.

    Returns (o [B,T,H,Dv] float64 or None, S_T [B,H,Dk,Dv] float64).
    """
    lib = _load()
    arrs = [_as_input(x) for x in (q, k, v, g, beta)]
    dts = {d for _, d in arrs}
    if len(dts) != 1:
        raise TypeError("q, k, v, g, beta must share one dtype")
    dt = dts.pop()
    (qa, _), (ka, _), (va, _), (ga, _), (ba, _) = arrs
    B, T, H, Dk = qa.shape
    Dv = va.shape[-1]
    if ka.shape != (B, T, H, Dk) or ga.shape != (B, T, H, Dk) or va.shape != (B, T, H, Dv) \
            or ba.shape != (B, T, H):
        raise ValueError("shape mismatch")
    s0 = None
    if S0 is not None:
        s0 = np.ascontiguousarray(np.asarray(S0, dtype=np.float64))
        if s0.shape != (B, H, Dk, Dv):
            raise ValueError("S0 shape")
    o = np.zeros((B, T, H, Dv), dtype=np.float64) if want_o else None
    ST = np.zeros((B, H, Dk, Dv), dtype=np.float64)
    pr = None
    npairs = 0
    if pairs is not None:
        pr = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32).reshape(-1, 2))
        npairs = pr.shape[0]
    nt = nthreads or default_threads()
    rc = lib.oracle_kda_forward(_ptr(qa), _ptr(ka), _ptr(va), _ptr(ga), _ptr(ba), dt, _ptr(s0),
                                _ptr(o), T * H * Dv, H * Dv, Dv, _ptr(ST),
                                B, T, H, Dk, Dv, _ptr(pr), npairs, nt)
    if rc != 0:
        raise ValueError("oracle_kda_forward rejected its arguments")
    return o, ST


def kda_forward_head(q, k, v, g, beta, b, h, S0_head=None, nthreads=1):
    """One (b, h) scan over the full length; returns (o [T,Dv], S_T [Dk,Dv]) in fp64.

    Memory is O(T*Dv) for the output of that head only, so full-length streams can be
    checked one head at a time."""
    lib = _load()
    arrs = [_as_input(x) for x in (q, k, v, g, beta)]
    dt = arrs[0][1]
    (qa, _), (ka, _), (va, _), (ga, _), (ba, _) = arrs
    B, T, H, Dk = qa.shape
    Dv = va.shape[-1]
    s0 = None
    if S0_head is not None:
        s0 = np.zeros((B, H, Dk, Dv), dtype=np.float64)
        s0[b, h] = np.asarray(S0_head, dtype=np.float64)
    o = np.zeros((T, Dv), dtype=np.float64)
    ST = np.zeros((B, H, Dk, Dv), dtype=np.float64) if B * H * Dk * Dv <= (1 << 24) else None
    pr = np.array([[b, h]], dtype=np.int32)
    if ST is None:
        raise ValueError("state buffer too large")
    # o[b*o_sb + t*o_st + h*o_sh]: address the single-head buffer with o_sb = o_sh = 0.
    rc = lib.oracle_kda_forward(_ptr(qa), _ptr(ka), _ptr(va), _ptr(ga), _ptr(ba), dt, _ptr(s0),
                                _ptr(o), 0, Dv, 0, _ptr(ST), B, T, H, Dk, Dv, _ptr(pr), 1, nthreads)
    if rc != 0:
        raise ValueError("oracle_kda_forward rejected its arguments")
    return o, ST[b, h].copy()


def make_segments(table):
    """table: iterable of (modality, start, F, Hgt, Wid, weight_set) -> ctypes array."""
    rows = list(table)
    arr = (Segment * max(1, len(rows)))()
    for i, (m, s, F, Hh, W, ws) in enumerate(rows):
        arr[i] = Segment(int(m), 0, int(s), int(F), int(Hh), int(W), int(ws))
    return arr, len(rows)


def mshortconv(x, segments, Kt, w_text=None, w_image=None, w_video=None, *, c_range=None,
               nthreads=None):
    """Direct-loop mShortConv in fp64.  x: [B,T,C] (fp32 / bf16 / fp64); weights fp32:
    text [n,C,Kt], image [n,C,3,3], video [n,C,3,3,3].  Returns y [B,T,C'] float64 for
    the channel range c_range=(lo,hi) (all channels by default); positions outside
    every segment are zero."""
    lib = _load()
    xa, dt = _as_input(x)
    B, T, C = xa.shape
    lo, hi = c_range if c_range is not None else (0, C)
    y = np.zeros((B, T, C), dtype=np.float64)
    segs, n = make_segments(segments)

    def wp(w):
        if w is None:
            return None, None
        try:
            import torch
            if isinstance(w, torch.Tensor):
                w = w.detach().cpu().float().numpy()
        except ImportError:  # pragma: no cover
            pass
        w = np.ascontiguousarray(np.asarray(w, dtype=np.float32))
        return w, _ptr(w)

    wt, pt = wp(w_text)
    wi, pi = wp(w_image)
    wv, pv = wp(w_video)
    nt = nthreads or default_threads()
    rc = lib.oracle_mshortconv(_ptr(xa), dt, _ptr(y), B, T, C, lo, hi,
                               ctypes.cast(segs, ctypes.c_void_p), n, int(Kt), pt, pi, pv, nt)
    if rc != 0:
        raise ValueError("oracle_mshortconv rejected its arguments")
    return y[:, :, lo:hi]


def l2norm_heads(x, H):
    """Unit-normalise every head slice of the last axis (length H*D); returns a copy."""
    a = np.array(x, dtype=np.float64, copy=True, order="C")
    D = a.shape[-1] // H
    lib = _load()
    rows = a.size // (H * D)
    lib.oracle_l2norm_heads(_ptr(a), rows, H, D)
    return a


def fused_forward(xq, xk, xv, segments, Kt, wq, wk, wv, g, beta, H, S0=None, *, pairs=None,
                  nthreads=None):
    """mShortConv of x_q, x_k, x_v (each [B,T,H*D]) -> L2-normalised q, k per head ->
    KDA scan (Eq. 13 feeding Eq. 14).  w* = (w_text, w_image, w_video) per tensor."""
    yq = mshortconv(xq, segments, Kt, *wq, nthreads=nthreads)
    yk = mshortconv(xk, segments, Kt, *wk, nthreads=nthreads)
    yv = mshortconv(xv, segments, Kt, *wv, nthreads=nthreads)
    B, T, C = yq.shape
    D = C // H
    q = l2norm_heads(yq, H).reshape(B, T, H, D)
    k = l2norm_heads(yk, H).reshape(B, T, H, D)
    v = yv.reshape(B, T, H, D)
    return kda_forward(q, k, v, _to_f64(g), _to_f64(beta), S0, pairs=pairs, nthreads=nthreads)


def kda_forward_varlen(q, k, v, g, beta, cu_seqlens, S0=None, *, nthreads=None):
    """Packed samples: q, k, g [T,H,Dk], v [T,H,Dv], beta [T,H]; sample i is tokens
    [cu[i], cu[i+1]) and runs kda_forward from S0[i] (zeros if S0 is None).  Returns
    (o [T,H,Dv], S_T [n,H,Dk,Dv]) in fp64."""
    cu = [int(x) for x in cu_seqlens]
    n = len(cu) - 1
    T, H, Dk = q.shape
    Dv = v.shape[-1]
    o = np.zeros((T, H, Dv))
    S_T = np.zeros((n, H, Dk, Dv))
    for i in range(n):
        a, b = cu[i], cu[i + 1]
        s0 = None if S0 is None else _to_f64(S0)[i:i + 1]
        if b == a:
            S_T[i] = 0.0 if s0 is None else s0[0]
            continue
        sl = lambda t: t[a:b][None]
        oi, si = kda_forward(sl(q), sl(k), sl(v), sl(g), sl(beta), s0, nthreads=nthreads)
        o[a:b] = oi[0]
        S_T[i] = si[0]
    return o, S_T


def gated_rmsnorm(o, gate, gamma=None, eps=1e-6):
    """Output side of Eq. 15 before W_o: for every (token, head) row r of o [..., H, Dv],
    y = sigmoid(gate_r) * gamma_h * r / sqrt(mean(r^2) + eps).  The RMS runs over the
    head's Dv channels; gamma [H, Dv] is the RMSNorm gain (None = ones); gate has o's
    shape and holds the pre-sigmoid values W_gate x.  fp64 throughout."""
    r = _to_f64(o)
    gt = _to_f64(gate)
    H, Dv = r.shape[-2], r.shape[-1]
    gm = np.ones((H, Dv)) if gamma is None else _to_f64(gamma).reshape(H, Dv)
    rms = np.sqrt(np.mean(r * r, axis=-1, keepdims=True) + float(eps))
    sig = 1.0 / (1.0 + np.exp(-gt))
    with np.errstate(invalid="ignore", divide="ignore"):
        y = np.where(rms > 0, r / rms, 0.0)
    return sig * gm * y


def kda_forward_gated(q, k, v, g, beta, gate, gamma=None, eps=1e-6, S0=None, *, pairs=None, nthreads=None):
    """kda_forward followed by gated_rmsnorm of its readout; returns (y, S_T)."""
    o, S_T = kda_forward(q, k, v, g, beta, S0, pairs=pairs, nthreads=nthreads)
    return gated_rmsnorm(o, gate, gamma, eps), S_T


def l2norm_heads_backward(x, dy, H):
    """Gradient through y = x / |x| per head slice (length D of the last axis H*D):
    dx = (dy - y (y . dy)) / |x|, and 0 where |x| = 0 (y = 0 there, a constant)."""
    X, G = _to_f64(x), _to_f64(dy)
    shp = X.shape
    D = shp[-1] // H
    Xh, Gh = X.reshape(-1, H, D), G.reshape(-1, H, D)
    n = np.sqrt(np.sum(Xh * Xh, axis=-1, keepdims=True))
    with np.errstate(invalid="ignore", divide="ignore"):
        Y = np.where(n > 0, Xh / n, 0.0)
        dX = np.where(n > 0, (Gh - Y * np.sum(Y * Gh, axis=-1, keepdims=True)) / n, 0.0)
    return dX.reshape(shp)


def fused_backward(xq, xk, xv, segments, Kt, wq, wk, wv, g, beta, H, do, S0=None, dS_T=None):
    """Gradients of L = sum(do * o) + sum(dS_T * S_T) through fused_forward: returns
    (dxq, dxk, dxv, dwq, dwk, dwv, dg, dbeta, dS0), each dw* a tuple (text, image, video)
    like w*.  Chain rule: the scan's backward on (q, k, v), then the norm's backward on
    dq, dk, then the conv's backward per tensor."""
    yq = mshortconv(xq, segments, Kt, *wq)
    yk = mshortconv(xk, segments, Kt, *wk)
    yv = mshortconv(xv, segments, Kt, *wv)
    B, T, C = yq.shape
    D = C // H
    q = l2norm_heads(yq, H).reshape(B, T, H, D)
    k = l2norm_heads(yk, H).reshape(B, T, H, D)
    v = yv.reshape(B, T, H, D)
    dq, dk, dv, dg, dbeta, dS0 = kda_backward(q, k, v, _to_f64(g), _to_f64(beta), do, S0, dS_T)
    dyq = l2norm_heads_backward(yq, dq.reshape(B, T, C), H)
    dyk = l2norm_heads_backward(yk, dk.reshape(B, T, C), H)
    gq = mshortconv_backward(xq, dyq, segments, Kt, *wq)
    gk = mshortconv_backward(xk, dyk, segments, Kt, *wk)
    gv = mshortconv_backward(xv, dv.reshape(B, T, C), segments, Kt, *wv)
    return gq[0], gk[0], gv[0], gq[1:], gk[1:], gv[1:], dg, dbeta, dS0


def _taps(modality, Kt):
    """(tap index, (df, dr, ds)) with y[f, r, s] += w[tap] * x[f + df, r + dr, s + ds]:
    text j -> (0, 0, j - (Kt-1)); image (a, e) -> (0, a-1, e-1); video (tau, a, e) ->
    (tau-2, a-1, e-1), taps numbered in the weight layout's row-major order."""
    if modality == MOD_TEXT:
        return [(j, (0, 0, j - (Kt - 1))) for j in range(Kt)]
    if modality == MOD_IMAGE:
        return [(3 * a + e, (0, a - 1, e - 1)) for a in range(3) for e in range(3)]
    return [(9 * tau + 3 * a + e, (tau - 2, a - 1, e - 1)) for tau in range(3) for a in range(3) for e in range(3)]


def mshortconv_backward(x, dy, segments, Kt, w_text=None, w_image=None, w_video=None):
    """Gradients of L = sum(dy * mshortconv(x)) with respect to x and to the weights.

    x, dy: [B,T,C]; weights as for mshortconv.  Returns (dx [B,T,C], dw_text, dw_image,
    dw_video) in fp64, each dw with its weight's shape (None where the weight is None).
    Inside a segment laid out as [F, Hgt, Wid] (text: [1, 1, len]),
    y[p] = sum_tap w[c, tap] x[p + off(tap)] over in-segment positions, so
      dx[p + off]       += w[c, tap] dy[p]
      dw[c, tap]        += sum over rows b and positions p of dy[p] x[p + off]
    for every tap whose shifted position stays inside the segment; tokens outside every
    segment get dx = 0."""
    X, DY = _to_f64(x), _to_f64(dy)
    B, T, C = X.shape
    dx = np.zeros((B, T, C))
    ws = {}
    for m, w in ((MOD_TEXT, w_text), (MOD_IMAGE, w_image), (MOD_VIDEO, w_video)):
        ws[m] = None if w is None else _to_f64(w)
    dws = {m: (None if w is None else np.zeros_like(w)) for m, w in ws.items()}
    for (m, s0, F, Hh, Wd, wset) in segments:
        F, Hh, Wd = (1, 1, Wd) if m == MOD_TEXT else ((1, Hh, Wd) if m == MOD_IMAGE else (F, Hh, Wd))
        n = F * Hh * Wd
        xs = X[:, s0:s0 + n].reshape(B, F, Hh, Wd, C)
        gs = DY[:, s0:s0 + n].reshape(B, F, Hh, Wd, C)
        dxs = np.zeros_like(xs)
        wm = ws[m][wset].reshape(C, -1)
        dwm = dws[m][wset].reshape(C, -1)
        for tap, (df, dr, ds) in _taps(m, Kt):
            # output positions p whose p + off lies in the segment
            f0, f1 = max(0, -df), min(F, F - df)
            r0, r1 = max(0, -dr), min(Hh, Hh - dr)
            c0, c1 = max(0, -ds), min(Wd, Wd - ds)
            if f0 >= f1 or r0 >= r1 or c0 >= c1:
                continue
            g_out = gs[:, f0:f1, r0:r1, c0:c1]
            x_in = xs[:, f0 + df:f1 + df, r0 + dr:r1 + dr, c0 + ds:c1 + ds]
            dxs[:, f0 + df:f1 + df, r0 + dr:r1 + dr, c0 + ds:c1 + ds] += wm[:, tap] * g_out
            dwm[:, tap] += np.einsum("bfrsc,bfrsc->c", g_out, x_in)
        dx[:, s0:s0 + n] = dxs.reshape(B, n, C)
    return dx, dws[MOD_TEXT], dws[MOD_IMAGE], dws[MOD_VIDEO]


def kda_backward(q, k, v, g, beta, do, S0=None, dS_T=None, *, block=64):
    """Gradients of L = sum(do * o) + sum(dS_T * S_T) through the scan of kda_forward.

    q, k, g: [B,T,H,Dk]; v, do: [B,T,H,Dv]; beta: [B,T,H]; S0, dS_T: [B,H,Dk,Dv] or
    None (zeros).  Inputs are read at their stored precision.  Returns fp64
    (dq, dk, dv, dg, dbeta, dS0) with the shapes of q, k, v, g, beta, S0.

    Per token t, with a = exp(g_t), X = Diag(a) S_{t-1}, w = v_t - X^T k_t:
      S_t = X + beta_t k_t w^T,   o_t = S_t^T q_t.
    The reverse sweep carries G = dL/dS_t (starting from dS_T):
      G      += q_t do_t^T                     (readout)
      dq_t    = S_t do_t
      dv_t    = beta_t G^T k_t
      dbeta_t = k_t^T G w
      dk_t    = beta_t (G w - X G^T k_t)
      dX      = G - beta_t k_t (k_t^T G)
      dg_t    = a * rowsum(dX * S_{t-1})       (dX/dg through X = Diag(e^g) S_{t-1})
      G       = Diag(a) dX                     (dL/dS_{t-1})
    and dS0 = G after token 1.  States are kept every `block` tokens and the ones in
    between recomputed by the same forward steps."""
    Q, K, V, Gl, Bt, dO = (_to_f64(x) for x in (q, k, v, g, beta, do))
    B, T, H, Dk = Q.shape
    Dv = V.shape[-1]
    s0 = None if S0 is None else _to_f64(S0)
    dst = None if dS_T is None else _to_f64(dS_T)
    dq, dk, dg = np.zeros_like(Q), np.zeros_like(K), np.zeros_like(Gl)
    dv, dbeta = np.zeros_like(V), np.zeros_like(Bt)
    dS0 = np.zeros((B, H, Dk, Dv))

    def step(S, b, t, h):
        X = np.exp(Gl[b, t, h])[:, None] * S
        kk = K[b, t, h]
        return X + Bt[b, t, h] * np.outer(kk, V[b, t, h] - kk @ X)

    for b in range(B):
        for h in range(H):
            S = np.zeros((Dk, Dv)) if s0 is None else s0[b, h].copy()
            ckpt = {}
            for t in range(T):
                if t % block == 0:
                    ckpt[t] = S.copy()
                S = step(S, b, t, h)
            G = np.zeros((Dk, Dv)) if dst is None else dst[b, h].copy()
            for t0 in reversed(range(0, T, block)):
                states = [ckpt[t0]]            # states[i] = S_{t0 + i - 1}, the state before token t0+i
                for t in range(t0, min(T, t0 + block)):
                    states.append(step(states[-1], b, t, h))
                for t in reversed(range(t0, min(T, t0 + block))):
                    S_prev, S_t = states[t - t0], states[t - t0 + 1]
                    a = np.exp(Gl[b, t, h])
                    kk, bt = K[b, t, h], Bt[b, t, h]
                    X = a[:, None] * S_prev
                    w = V[b, t, h] - kk @ X
                    G = G + np.outer(Q[b, t, h], dO[b, t, h])
                    dq[b, t, h] = S_t @ dO[b, t, h]
                    Gk = G.T @ kk
                    dv[b, t, h] = bt * Gk
                    dbeta[b, t, h] = Gk @ w
                    dk[b, t, h] = bt * (G @ w - X @ Gk)
                    dX = G - bt * np.outer(kk, Gk)
                    dg[b, t, h] = a * np.sum(dX * S_prev, axis=1)
                    G = a[:, None] * dX
            dS0[b, h] = G
    return dq, dk, dv, dg, dbeta, dS0


def _to_f64(a):
    """Widen an input (torch tensor or numpy array, bf16 bit patterns included) to fp64
    at its stored precision."""
    arr, dt = _as_input(a)
    if dt == DT_BF16:
        return (arr.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return arr.astype(np.float64)
