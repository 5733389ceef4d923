"""Pins of the oracle's backward (kda_backward) to things other than itself.

* Finite differences: central differences of the (separately pinned) forward oracle's
  L = sum(do * o) + sum(dS_T * S_T) with respect to every input element.
* Automatic differentiation: torch.autograd through a plain fp64 token loop of Eq. 14
  written here, with Dk != Dv so that a transposed operand cannot pass.
* Closed form: with beta = 0 the scan is pure decay, S_t = Diag(prod_{r<=t} alpha_r) S0,
  so dv = dk = 0, dq_t = S_t do_t and dS0 = sum_t Diag(c_t) q_t do_t^T + Diag(c_T) dS_T
  with c_t = prod_{r<=t} alpha_r.
"""
import numpy as np
import torch

from oracle import oracle as O

NAMES = ("q", "k", "v", "g", "beta", "S0")


def _inputs(B, T, H, Dk, Dv, seed):
    gen = torch.Generator().manual_seed(seed)
    x = lambda *s: torch.randn(*s, generator=gen, dtype=torch.float64)
    q, k, v = x(B, T, H, Dk), x(B, T, H, Dk), x(B, T, H, Dv)
    g = -torch.rand(B, T, H, Dk, generator=gen, dtype=torch.float64)
    beta = torch.rand(B, T, H, generator=gen, dtype=torch.float64)
    do, S0, dST = x(B, T, H, Dv), x(B, H, Dk, Dv), x(B, H, Dk, Dv)
    return [q, k, v, g, beta, S0], do, dST


def test_backward_matches_finite_differences():
    args, do, dST = _inputs(1, 7, 1, 3, 2, seed=0)
    grads = O.kda_backward(*args[:5], do, args[5].numpy(), dST.numpy(), block=3)

    def L():
        o, S = O.kda_forward(*args[:5], args[5].numpy())
        return float((o * do.numpy()).sum() + (S * dST.numpy()).sum())

    eps = 1e-6
    for name, a, gr in zip(NAMES, args, grads):
        flat = a.view(-1)
        fd = np.zeros(flat.numel())
        for j in range(flat.numel()):
            old = flat[j].item()
            flat[j] = old + eps
            lp = L()
            flat[j] = old - eps
            lm = L()
            flat[j] = old
            fd[j] = (lp - lm) / (2 * eps)
        err = np.abs(fd - gr.reshape(-1)).max()
        assert err <= 1e-7 * max(1.0, np.abs(fd).max()), (name, err)


def _torch_scan(q, k, v, g, beta, S0):
    B, T, H, Dk = q.shape
    outs, finals = [], []
    for b in range(B):
        ob, fb = [], []
        for h in range(H):
            S = S0[b, h]
            oh = []
            for t in range(T):
                kk = k[b, t, h]
                S = torch.exp(g[b, t, h])[:, None] * S
                S = S - beta[b, t, h] * torch.outer(kk, kk @ S) + beta[b, t, h] * torch.outer(kk, v[b, t, h])
                oh.append(S.T @ q[b, t, h])
            ob.append(torch.stack(oh))
            fb.append(S)
        outs.append(torch.stack(ob, dim=1))
        finals.append(torch.stack(fb))
    return torch.stack(outs), torch.stack(finals)


def test_backward_matches_autograd_of_a_token_loop():
    args, do, dST = _inputs(2, 20, 2, 5, 4, seed=1)
    leaves = [a.clone().requires_grad_(True) for a in args]
    o, S = _torch_scan(*leaves)
    ((o * do).sum() + (S * dST).sum()).backward()
    grads = O.kda_backward(*args[:5], do, args[5].numpy(), dST.numpy(), block=8)
    for name, leaf, gr in zip(NAMES, leaves, grads):
        ref = leaf.grad.numpy()
        assert gr.shape == ref.shape, name
        assert np.abs(gr - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max()), name


def test_backward_pure_decay_closed_form():
    args, do, dST = _inputs(1, 9, 2, 4, 3, seed=2)
    q, k, v, g, beta, S0 = args
    beta = torch.zeros_like(beta)
    dq, dk, dv, dg, dbeta, dS0 = O.kda_backward(q, k, v, g, beta, do, S0.numpy(), dST.numpy(), block=4)
    assert np.all(dv == 0.0) and np.all(dk == 0.0)
    c = np.cumprod(np.exp(g.numpy()), axis=1)            # [B,T,H,Dk]
    s0, qn, don = S0.numpy(), q.numpy(), do.numpy()
    for h in range(2):
        ref_dS0 = c[0, -1, h][:, None] * dST.numpy()[0, h]
        for t in range(9):
            S_t = c[0, t, h][:, None] * s0[0, h]
            assert np.allclose(dq[0, t, h], S_t @ don[0, t, h], rtol=1e-13, atol=1e-13)
            ref_dS0 = ref_dS0 + c[0, t, h][:, None] * np.outer(qn[0, t, h], don[0, t, h])
        assert np.allclose(dS0[0, h], ref_dS0, rtol=1e-13, atol=1e-13)


def test_backward_checkpoint_block_does_not_change_the_result():
    args, do, dST = _inputs(1, 13, 1, 4, 4, seed=3)
    a = O.kda_backward(*args[:5], do, args[5].numpy(), dST.numpy(), block=64)
    b = O.kda_backward(*args[:5], do, args[5].numpy(), dST.numpy(), block=5)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
