"""Pins of the w / beta prologue oracle (oracle/wbeta.py) against things other than itself.

- the forward, rebuilt from library routines: torch's depthwise conv1d for the
  3-tap causal short convolution, F.normalize for the L2 normalisation (the same
  max(|z|, eps) guard), torch.sigmoid (Paper-Notes "关键设计");
- every gradient against autograd of that formulation, and against central finite
  differences;
- closed forms: u = 0, b = 0 gives beta = 1; an identity first factor with the
  identity filter gives normalize(x Bw); the one-step-delay filter shifts w by one
  position; unit norms; the clip;
- causality of the convolution, and the scale invariants: w does not change when
  z is scaled, and z is linear in each of A, Bw and f, so sum(A dA), sum(Bw dBw)
  and sum(f df) vanish;
- mutations planted in a copy of the oracle source are caught.
"""
import os
import types

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle.wbeta as wb

TOL = 1e-10


def case(rng, B=2, L=9, D=7, r=3, H=2, d=4, beta_max=2.0, scale=1.0):
    x = rng.standard_normal((B, L, D)) * scale
    A = rng.standard_normal((D, r)) / np.sqrt(D)
    Bw = rng.standard_normal((r, H * d)) / np.sqrt(r)
    f = rng.standard_normal((H * d, 3))
    u = rng.standard_normal((D, H)) / np.sqrt(D)
    b = rng.standard_normal(H)
    return x, A, Bw, f, u, b, H, beta_max


def torch_forward(x, A, Bw, f, u, b, H, beta_max):
    """The prologue from library routines (fp64 autograd leaves in, w and beta out)."""
    B, L, D = x.shape
    Hd = Bw.shape[1]
    wt = (x @ A) @ Bw                                     # [B, L, Hd]
    # causal 3-tap depthwise convolution: left-pad 2 and cross-correlate with the
    # taps reversed (conv1d weight tap j meets wt_{t + j - 2} = wt_{t - k} for k = 2 - j)
    z = F.conv1d(F.pad(wt.transpose(1, 2), (2, 0)), f.flip(1).unsqueeze(1), groups=Hd)
    z = z.transpose(1, 2).reshape(B, L, H, Hd // H)
    w = F.normalize(z, p=2.0, dim=-1, eps=wb.EPS).permute(0, 2, 1, 3)
    beta = torch.clamp(2.0 * torch.sigmoid(x @ u + b), max=beta_max).permute(0, 2, 1)
    return w, beta


def leaves(args):
    return [torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in args[:6]]


def test_forward_matches_library_routines():
    rng = np.random.default_rng(0)
    args = case(rng, beta_max=1.5)
    w, beta = wb.fwd(*args)
    tw, tbeta = torch_forward(*leaves(args), args[6], args[7])
    np.testing.assert_allclose(w, tw.detach().numpy(), atol=TOL, rtol=0)
    np.testing.assert_allclose(beta, tbeta.detach().numpy(), atol=TOL, rtol=0)


@pytest.mark.parametrize("beta_max", [2.0, 1.2])
def test_gradients_match_autograd(beta_max):
    rng = np.random.default_rng(1)
    args = list(case(rng, beta_max=beta_max))
    # head 0 gets a zero first tap: its z at t = 0 is 0 (the |z| <= EPS branch)
    args[3][:args[3].shape[0] // args[6], 0] = 0.0
    args = tuple(args)
    B, L = args[0].shape[:2]
    H, d = args[6], args[2].shape[1] // args[6]
    dw = rng.standard_normal((B, H, L, d))
    dbeta = rng.standard_normal((B, H, L))
    ours = wb.bwd(*args, dw=dw, dbeta=dbeta)
    ts = leaves(args)
    tw, tbeta = torch_forward(*ts, H, beta_max)
    loss = (tw * torch.tensor(dw)).sum() + (tbeta * torch.tensor(dbeta)).sum()
    loss.backward()
    for name, t in zip(("dx", "dA", "dBw", "df", "du", "db"), ts):
        np.testing.assert_allclose(ours[name], t.grad.numpy(), atol=TOL, rtol=1e-9, err_msg=name)


def test_gradients_match_finite_differences():
    rng = np.random.default_rng(2)
    args = case(rng, B=1, L=6, D=5, r=2, H=2, d=3, beta_max=1.7)
    B, L = args[0].shape[:2]
    H, d = args[6], args[2].shape[1] // args[6]
    dw = rng.standard_normal((B, H, L, d))
    dbeta = rng.standard_normal((B, H, L))

    def loss(a):
        w, beta = wb.fwd(*a)
        return float(np.sum(w * dw) + np.sum(beta * dbeta))

    g = wb.bwd(*args, dw=dw, dbeta=dbeta)
    h = 1e-6
    for i, name in enumerate(("dx", "dA", "dBw", "df", "du", "db")):
        arr = args[i]
        for _ in range(4):
            idx = tuple(rng.integers(0, s) for s in arr.shape)
            ap = [a.copy() if j == i else a for j, a in enumerate(args[:6])]
            am = [a.copy() if j == i else a for j, a in enumerate(args[:6])]
            ap[i][idx] += h
            am[i][idx] -= h
            num = (loss((*ap, H, args[7])) - loss((*am, H, args[7]))) / (2 * h)
            assert abs(num - g[name][idx]) <= 1e-6 * max(1.0, abs(num)), (name, idx, num, g[name][idx])


def test_closed_forms():
    rng = np.random.default_rng(3)
    x, A, Bw, f, u, b, H, _ = case(rng, D=4, r=4)
    B, L = x.shape[:2]
    d = Bw.shape[1] // H
    # no projection, no bias: beta = 2 sigmoid(0) = 1
    _, beta = wb.fwd(x, A, Bw, f, np.zeros_like(u), np.zeros_like(b), H)
    np.testing.assert_allclose(beta, 1.0, atol=TOL)
    # identity first factor and the identity filter: w = normalize(x Bw) per head
    ident = np.tile([1.0, 0.0, 0.0], (Bw.shape[1], 1))
    w, _ = wb.fwd(x, np.eye(4), Bw, ident, u, b, H)
    ref = (x @ Bw).reshape(B, L, H, d)
    ref = ref / np.linalg.norm(ref, axis=-1, keepdims=True)
    np.testing.assert_allclose(w, ref.transpose(0, 2, 1, 3), atol=TOL)
    # the one-step delay: w_t = normalize(wt_{t-1}), w_0 = 0
    delay = np.tile([0.0, 1.0, 0.0], (Bw.shape[1], 1))
    w1, _ = wb.fwd(x, A, Bw, delay, u, b, H)
    w0, _ = wb.fwd(x, A, Bw, ident, u, b, H)
    np.testing.assert_allclose(w1[:, :, 1:], w0[:, :, :-1], atol=TOL)
    np.testing.assert_allclose(w1[:, :, 0], 0.0, atol=TOL)
    # unit norms, and the clip
    w, beta = wb.fwd(x, A, Bw, f, u, b, H, beta_max=1.1)
    np.testing.assert_allclose(np.linalg.norm(w, axis=-1), 1.0, atol=TOL)
    assert beta.max() <= 1.1 and beta.min() > 0.0


def test_causality():
    rng = np.random.default_rng(4)
    args = case(rng, L=12)
    w0, b0 = wb.fwd(*args)
    x = args[0].copy()
    x[:, 7] += rng.standard_normal(x.shape[2])
    w1, b1 = wb.fwd(x, *args[1:])
    np.testing.assert_array_equal(w0[:, :, :7], w1[:, :, :7])
    np.testing.assert_array_equal(b0[:, :, :7], b1[:, :, :7])
    assert np.abs(w0[:, :, 7] - w1[:, :, 7]).max() > 1e-6


def test_scale_invariants():
    rng = np.random.default_rng(5)
    args = case(rng)
    B, L = args[0].shape[:2]
    H, d = args[6], args[2].shape[1] // args[6]
    g = wb.bwd(*args, dw=rng.standard_normal((B, H, L, d)), dbeta=np.zeros((B, H, L)))
    for name, a in (("dA", args[1]), ("dBw", args[2]), ("df", args[3])):
        s = float(np.sum(a * g[name]))
        assert abs(s) <= 1e-10 * (1.0 + float(np.abs(a * g[name]).sum())), (name, s)


# ---------------------------------------------------------------- planted mistakes
MUTATIONS = {
    "conv reaches forward": ("sum(f[:, k] * _shift(wt, k) for k in range(3))",
                             "sum(f[:, k] * _unshift(wt, k) for k in range(3))"),
    "sigmoid derivative": ("2.0 * sig * (1.0 - sig)", "sig * (1.0 - sig)"),
    "no projection off w": ("(g - w * along)", "g"),
    "adjoint conv direction": ("sum(f[:, k] * _unshift(dz, k) for k in range(3))",
                               "sum(f[:, k] * _shift(dz, k) for k in range(3))"),
    "clip ignored": ("np.where(open_, db_t", "np.where(True, db_t"),
    "filter gradient tap": ("np.sum(dz * _shift(wt, k), axis=(0, 1))",
                            "np.sum(dz * _shift(wt, 2 - k), axis=(0, 1))"),
    "beta projection transposed": ("dx = ds @ u.T", "dx = ds @ u.T * 0.5"),
}


def mutated(before, after):
    src = open(wb.__file__).read()
    assert src.count(before) == 1, before
    mod = types.ModuleType("wbeta_mutant")
    exec(compile(src.replace(before, after), "wbeta_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_a_planted_mistake_is_caught(name, monkeypatch):
    monkeypatch.setattr(wb, "fwd", mutated(*MUTATIONS[name]).fwd)
    monkeypatch.setattr(wb, "bwd", mutated(*MUTATIONS[name]).bwd)
    pins = (test_forward_matches_library_routines,
            lambda: test_gradients_match_autograd(1.2), test_closed_forms)
    caught = False
    for pin in pins:
        try:
            pin()
        except AssertionError:
            caught = True
            break
    assert caught, f"no pin caught the planted mistake: {name}"
