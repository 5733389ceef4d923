"""Writes the golden fixtures of this directory: exact rational results of the plain
definitions, computed with Python fractions (no floating point, no oracle, no CUDA).

* kda_exact.json -- the state recurrence of Eq. 14 of the Chimera paper (section 3.3),
  S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T, with the readout
  o_t = S_t^T q_t of Eq. 15, for T = 4 tokens, d_k = 2, d_v = 3, a nonzero S0 and one
  token with beta = 0.
* conv_exact.json -- the per-segment depthwise conv of section 3.4 on integers: a text
  segment (kernel 4, causal, zero before the segment), a 3 x 3 image and a 2-frame 2 x 2
  video (3 x 3 x 3 kernel, frames f-2..f), one channel each.

Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
from fractions import Fraction as F

HERE = os.path.dirname(os.path.abspath(__file__))


def s(x):
    return f"{x.numerator}/{x.denominator}"


def kda_case():
    alpha = [[F(3, 4), F(1, 2)], [F(7, 8), F(1, 1)], [F(1, 2), F(3, 4)], [F(15, 16), F(5, 8)]]
    beta = [F(1, 2), F(0), F(1, 1), F(3, 4)]
    k = [[F(1), F(0)], [F(1, 2), F(1, 2)], [F(0), F(1)], [F(3, 5), F(4, 5)]]
    q = [[F(1), F(1)], [F(-1), F(2)], [F(1, 2), F(-1, 2)], [F(0), F(1)]]
    v = [[F(1), F(-2), F(3)], [F(2), F(0), F(-1)], [F(-1), F(1), F(1)], [F(1, 2), F(1, 4), F(-1, 4)]]
    S = [[F(1, 2), F(0), F(-1)], [F(1), F(1, 4), F(0)]]
    S0 = [row[:] for row in S]
    outs = []
    for t in range(4):
        dk, dv = 2, 3
        X = [[alpha[t][i] * S[i][j] for j in range(dv)] for i in range(dk)]            # Diag(alpha) S
        kX = [sum(k[t][i] * X[i][j] for i in range(dk)) for j in range(dv)]            # k^T X
        S = [[X[i][j] - beta[t] * k[t][i] * kX[j] + beta[t] * k[t][i] * v[t][j] for j in range(dv)]
             for i in range(dk)]
        outs.append([sum(S[i][j] * q[t][i] for i in range(dk)) for j in range(dv)])
    g = lambda M: [[s(x) for x in row] for row in M]
    return {"cite": "Chimera paper, section 3.3, Eq. 14 (state update) and Eq. 15 (readout S_t^T q_t)",
            "alpha": g(alpha), "beta": [s(b) for b in beta], "k": g(k), "q": g(q), "v": g(v),
            "S0": g(S0), "o": g(outs), "S_T": g(S)}


def conv_case():
    # text: kernel w[0..3], y[t] = sum_j w[j] x[t-3+j], zero before the segment
    wt = [1, -2, 3, 4]
    xt = [2, -1, 0, 5, 3]
    yt = [sum(wt[j] * (xt[t - 3 + j] if t - 3 + j >= 0 else 0) for j in range(4)) for t in range(5)]
    # image 3x3: y[r][c] = sum_{a,e} w[a][e] x[r-1+a][c-1+e], zero outside
    wi = [[1, 0, -1], [2, 1, 0], [0, -1, 3]]
    xi = [[1, 2, 0], [-1, 3, 1], [2, 0, -2]]
    inside = lambda r, c, H, W: 0 <= r < H and 0 <= c < W
    yi = [[sum(wi[a][e] * (xi[r - 1 + a][c - 1 + e] if inside(r - 1 + a, c - 1 + e, 3, 3) else 0)
               for a in range(3) for e in range(3)) for c in range(3)] for r in range(3)]
    # video 2 frames of 2x2: y[f][r][c] = sum w[tau][a][e] x[f-2+tau][r-1+a][c-1+e]
    wv = [[[(tau + 1) * (a - e) + (a * e) % 3 for e in range(3)] for a in range(3)] for tau in range(3)]
    xv = [[[1, -1], [2, 0]], [[0, 3], [-2, 1]]]
    yv = [[[sum(wv[tau][a][e] * (xv[f - 2 + tau][r - 1 + a][c - 1 + e]
                                  if f - 2 + tau >= 0 and inside(r - 1 + a, c - 1 + e, 2, 2) else 0)
                for tau in range(3) for a in range(3) for e in range(3)) for c in range(2)] for r in range(2)]
          for f in range(2)]
    return {"cite": "Chimera paper, section 3.4 (modality-aware short convolution; Eq. 12 raster order)",
            "text": {"w": wt, "x": xt, "y": yt}, "image": {"w": wi, "x": xi, "y": yi},
            "video": {"w": wv, "x": xv, "y": yv}}


if __name__ == "__main__":
    with open(os.path.join(HERE, "kda_exact.json"), "w") as f:
        json.dump(kda_case(), f, indent=1)
    with open(os.path.join(HERE, "conv_exact.json"), "w") as f:
        json.dump(conv_case(), f, indent=1)
