"""Comparison helpers shared by the GPU parity tests (no method arithmetic here).

Tolerances (written once, used by every parity test):
  * fp32 inputs: max |gpu - oracle| <= 1e-4 * max |oracle|, per (b, h), for o and S_T.
  * bf16 inputs: max |gpu - oracle| <= 2e-2 * RMS(oracle), per (b, h), for o and S_T,
    with the oracle fed the same bf16-rounded inputs (o computed in fp32).
  * a bf16 output o: element-wise |gpu - oracle| <= 2e-2 * RMS(oracle) + 2^-9 |oracle|
    (the same bound plus the rounding of o to bf16).
The relative-to-max form for fp32 avoids an ill-posed element-wise relative error near
zero; the bf16 bound covers bf16 operand and output rounding after fp32 accumulation.
"""
import numpy as np
import torch

FP32_REL = 1e-4
BF16_RMS = 2e-2


def tol_for(dtype) -> str:
    return "fp32" if dtype == torch.float32 else "bf16"


def compare(gpu: np.ndarray, ref: np.ndarray, kind: str, what: str = ""):
    """gpu, ref: arrays of one (b, h) slice.  Returns (err, bound); asserts err <= bound."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite values in the GPU result"
    err = float(np.abs(gpu - ref).max()) if gpu.size else 0.0
    if kind == "fp32":
        bound = FP32_REL * float(np.abs(ref).max()) if ref.size else 0.0
    else:
        bound = BF16_RMS * float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    assert err <= bound + 1e-30, f"{what}: max|diff| {err:.3e} > bound {bound:.3e}"
    return err, bound


BF16_HALF_ULP = 2.0 ** -9   # round-to-nearest bf16: relative error at most 2^-9


def compare_bf16_output(gpu: np.ndarray, ref: np.ndarray, what: str = ""):
    """A bf16 output o against the oracle: element-wise |gpu - ref| <= 2e-2 * RMS(ref) +
    2^-9 * |ref|, the bf16-input bound plus the rounding of o itself to bf16 (which alone
    reaches 2.3-2.5% of RMS on the video clip's heavy-tailed outputs).  Returns the
    worst ratio to that bound."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite values in the GPU result"
    if not ref.size:
        return 0.0
    bound = BF16_RMS * float(np.sqrt(np.mean(ref * ref))) + BF16_HALF_ULP * np.abs(ref)
    ratio = float((np.abs(gpu - ref) / bound).max())
    assert ratio <= 1.0, f"{what}: |diff| exceeds 2e-2 RMS + 2^-9 |ref| by x{ratio:.3f}"
    return ratio


def compare_heads(o_gpu, o_ref, S_gpu, S_ref, kind, pairs=None, what=""):
    """Per-(b,h) comparison of o [B,T,H,Dv] and S_T [B,H,Dk,Dv]."""
    B, T, H, _ = o_ref.shape
    pairs = pairs if pairs is not None else [(b, h) for b in range(B) for h in range(H)]
    worst = 0.0
    for (b, h) in pairs:
        e, bd = compare(o_gpu[b, :, h], o_ref[b, :, h], kind, f"{what} o[b={b},h={h}]")
        worst = max(worst, e / bd if bd > 0 else 0.0)
        if S_gpu is not None and S_ref is not None:
            e, bd = compare(S_gpu[b, h], S_ref[b, h], kind, f"{what} S_T[b={b},h={h}]")
            worst = max(worst, e / bd if bd > 0 else 0.0)
    return worst


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)
