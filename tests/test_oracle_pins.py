"""Pins of the fp64 oracle against things other than itself.

Each test ties the oracle to something the pages or mathematics fix:
explicit d x d matrix products of the Householder-like factors, the UT
identity and full-matrix form printed on the Paper-Notes page ("训练策略"),
a library attention routine (torch SDPA) where PaTH reduces to plain causal
softmax attention, closed forms for repeated w, norm preservation of H at
beta = 2, finite differences and autograd of an explicit-matrix formulation
for every gradient, gradient invariants, decode replay (with and without the
gate's per-key bias), and the cache a prefill leaves (explicit products, the
forward's last row, decode continuing the forward). The mutation
tests at the end plant mistakes in a copy of the oracle source and check that
a pin catches each one.
"""
import math
import os
import re
import tempfile

import numpy as np
import pytest
import torch
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle

RTOL = 1e-11


def rand_case(rng, B=1, H=2, L=9, d=5, beta_hi=2.0, unit_w=True, fox=False):
    q, k, v, w = (rng.standard_normal((B, H, L, d)) for _ in range(4))
    if unit_w:
        w /= np.linalg.norm(w, axis=-1, keepdims=True)
    beta = rng.uniform(0.0, beta_hi, (B, H, L))
    logf = np.log(1.0 / (1.0 + np.exp(-(3.0 + rng.standard_normal((B, H, L)))))) if fox else None
    return q, k, v, w, beta, logf


# ---------------------------------------------------------------- helpers
def householder(w_s, b_s):
    return np.eye(len(w_s)) - b_s * np.outer(w_s, w_s)


def explicit_scores(q, k, w, beta, logf, scale):
    """z_ij = scale q_i^T (H_i ... H_{j+1}) k_j + c_i - c_j from explicit matrices."""
    L, d = q.shape
    c = np.cumsum(logf) if logf is not None else np.zeros(L)
    z = np.full((L, L), -np.inf)
    for i in range(L):
        M = np.eye(d)  # H_i ... H_{j+1}, built by right-multiplying as j decreases
        for j in range(i, -1, -1):
            z[i, j] = scale * q[i] @ M @ k[j] + c[i] - c[j]
            M = M @ householder(w[j], beta[j])
    return z


def ut_inverse(W, beta):
    """T^{-1} = (I + strictLower(D W W^T))^{-1} D (Paper-Notes, UT transform)."""
    n = W.shape[0]
    A = np.tril(beta[:, None] * (W @ W.T), -1)
    return np.linalg.solve(np.eye(n) + A, np.diag(beta))


# ---------------------------------------------------------------- forward pins
def test_scores_equal_explicit_matrix_products(orc):
    rng = np.random.default_rng(1)
    q, k, v, w, beta, logf = rand_case(rng, L=10, d=5, fox=True, unit_w=False)  # w unnormalised
    z = orc.scores(q, k, w, beta, logf, scale=0.7)
    for h in range(2):
        ref = explicit_scores(q[0, h], k[0, h], w[0, h], beta[0, h], logf[0, h], 0.7)
        np.testing.assert_allclose(z[0, h], ref, rtol=RTOL, atol=1e-12)


def test_fwd_equals_softmax_of_explicit_scores(orc):
    rng = np.random.default_rng(2)
    q, k, v, w, beta, logf = rand_case(rng, B=2, H=1, L=11, d=4, fox=True)
    out, lse = orc.fwd(q, k, v, w, beta, logf, scale=0.9)
    for b in range(2):
        z = explicit_scores(q[b, 0], k[b, 0], w[b, 0], beta[b, 0], logf[b, 0], 0.9)
        zt = torch.from_numpy(z)
        ref_lse = torch.logsumexp(zt, dim=-1).numpy()
        ref_out = (torch.softmax(zt, dim=-1) @ torch.from_numpy(v[b, 0])).numpy()
        np.testing.assert_allclose(lse[b, 0], ref_lse, rtol=RTOL)
        np.testing.assert_allclose(out[b, 0], ref_out, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("zero", ["beta", "w"])
def test_beta_or_w_zero_is_causal_softmax_attention(orc, zero):
    rng = np.random.default_rng(3)
    q, k, v, w, beta, _ = rand_case(rng, B=2, H=3, L=33, d=8)
    if zero == "beta":
        beta[:] = 0.0
    else:
        w[:] = 0.0
    out, lse = orc.fwd(q, k, v, w, beta, scale=8 ** -0.5)
    t = [torch.from_numpy(a) for a in (q, k, v)]
    ref = torch.nn.functional.scaled_dot_product_attention(*t, is_causal=True, scale=8 ** -0.5)
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-10, atol=1e-12)


def test_fox_with_beta_zero_is_gated_softmax_attention(orc):
    rng = np.random.default_rng(4)
    q, k, v, w, beta, logf = rand_case(rng, B=1, H=2, L=40, d=6, fox=True)
    beta[:] = 0.0
    out, lse = orc.fwd(q, k, v, w, beta, logf, scale=0.5)
    c = torch.from_numpy(np.cumsum(logf, axis=-1))
    bias = c[..., :, None] - c[..., None, :]
    mask = torch.ones(40, 40, dtype=torch.bool).tril()
    bias = bias.masked_fill(~mask, -math.inf)
    t = [torch.from_numpy(a) for a in (q, k, v)]
    ref = torch.nn.functional.scaled_dot_product_attention(*t, attn_mask=bias, scale=0.5)
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-10, atol=1e-12)


def test_zero_log_gate_is_plain_path(orc):
    rng = np.random.default_rng(5)
    q, k, v, w, beta, _ = rand_case(rng, L=20, d=6)
    a = orc.fwd(q, k, v, w, beta, np.zeros(beta.shape))
    b = orc.fwd(q, k, v, w, beta, None)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_length_one(orc):
    rng = np.random.default_rng(6)
    q, k, v, w, beta, _ = rand_case(rng, B=1, H=3, L=1, d=7)
    out, lse = orc.fwd(q, k, v, w, beta, scale=0.3)
    np.testing.assert_array_equal(out, v)
    np.testing.assert_allclose(lse, 0.3 * np.sum(q * k, axis=-1), rtol=1e-15)


def test_projector_closed_form(orc):
    """beta = 1 and every w_s = u (unit): H = I - u u^T is a projector, so for
    j < i the path product is exactly I - u u^T."""
    rng = np.random.default_rng(7)
    L, d = 12, 5
    q, k = rng.standard_normal((2, 1, 1, L, d))
    u = rng.standard_normal(d)
    u /= np.linalg.norm(u)
    w = np.broadcast_to(u, (1, 1, L, d)).copy()
    z = orc.scores(q, k, w, np.ones((1, 1, L)), scale=1.0)[0, 0]
    Pu = np.eye(d) - np.outer(u, u)
    for i in range(L):
        for j in range(i + 1):
            ref = q[0, 0, i] @ (Pu if j < i else np.eye(d)) @ k[0, 0, j]
            assert abs(z[i, j] - ref) < 1e-12


def test_reflection_parity_closed_form(orc):
    """beta = 2 and every w_s = u (unit): H is a reflection, H^2 = I, so the
    path product is I for even i - j and I - 2 u u^T for odd i - j."""
    rng = np.random.default_rng(8)
    L, d = 13, 6
    q, k = rng.standard_normal((2, 1, 1, L, d))
    u = rng.standard_normal(d)
    u /= np.linalg.norm(u)
    w = np.broadcast_to(u, (1, 1, L, d)).copy()
    z = orc.scores(q, k, w, np.full((1, 1, L), 2.0), scale=1.0)[0, 0]
    R = np.eye(d) - 2 * np.outer(u, u)
    for i in range(L):
        for j in range(i + 1):
            ref = q[0, 0, i] @ (np.eye(d) if (i - j) % 2 == 0 else R) @ k[0, 0, j]
            assert abs(z[i, j] - ref) < 1e-12


def test_reflections_preserve_norms_and_contractions_shrink(orc):
    """beta = 2, |w| = 1: each H is orthogonal, cached key norms never change.
    beta in [0, 2]: |H|_2 <= 1, so norms never grow and |S_ij| <= |q_i||k_j|."""
    rng = np.random.default_rng(9)
    B, H, d, steps = 1, 2, 8, 60
    kc = np.zeros((B, H, steps, d))
    vc = np.zeros((B, H, steps, d))
    kc2 = np.zeros_like(kc)
    vc2 = np.zeros_like(vc)
    norms = []
    for t in range(steps):
        q, kn, vn, w = rng.standard_normal((4, B, H, d))
        w /= np.linalg.norm(w, axis=-1, keepdims=True)
        orc.decode_step(q, kn, vn, w, np.full((B, H), 2.0), kc, vc, t)
        before = np.linalg.norm(kc2[:, :, :t], axis=-1)
        orc.decode_step(q, kn, vn, w, rng.uniform(0, 2, (B, H)), kc2, vc2, t)
        after = np.linalg.norm(kc2[:, :, :t], axis=-1)
        assert np.all(after <= before + 1e-12)
        norms.append(np.linalg.norm(kn, axis=-1))
    final = np.linalg.norm(kc, axis=-1)
    np.testing.assert_allclose(final, np.stack(norms, axis=-1), rtol=1e-13)
    q, k, v, w, beta, _ = rand_case(rng, L=30, d=6, unit_w=True)
    z = orc.scores(q, k, w, beta, scale=1.0)
    bound = np.linalg.norm(q, axis=-1)[..., :, None] * np.linalg.norm(k, axis=-1)[..., None, :]
    low = np.tril(np.ones((30, 30), dtype=bool))
    assert np.all(np.abs(z[..., low]) <= bound[..., low] + 1e-12)


def test_ut_identity_orientation():
    """Paper-Notes "训练策略": I - W^T T^{-1} W equals the product of the H_t.
    It holds for the descending product H_{L-1} ... H_0 (the orientation the
    blockwise path uses); the ascending product differs."""
    rng = np.random.default_rng(10)
    L, d = 9, 6
    W = rng.standard_normal((L, d))
    beta = rng.uniform(0, 2, L)
    P = np.eye(d) - W.T @ ut_inverse(W, beta) @ W
    desc = np.eye(d)
    for t in range(L):
        desc = householder(W[t], beta[t]) @ desc
    asc = np.eye(d)
    for t in range(L):
        asc = asc @ householder(W[t], beta[t])
    np.testing.assert_allclose(P, desc, atol=1e-13)
    assert np.abs(P - asc).max() > 1e-3


def test_full_matrix_form_matches_oracle(orc):
    """Paper-Notes "训练策略": lower(QK^T) - lower(QW^T) T^{-1} strictLower(WK^T)
    equals the oracle's logits on and below the diagonal."""
    rng = np.random.default_rng(11)
    q, k, v, w, beta, _ = rand_case(rng, B=1, H=1, L=14, d=5)
    Q, K, W, b = q[0, 0], k[0, 0], w[0, 0], beta[0, 0]
    A = np.tril(Q @ K.T) - np.tril(Q @ W.T) @ ut_inverse(W, b) @ np.tril(W @ K.T, -1)
    z = orc.scores(q, k, w, beta, scale=1.0)[0, 0]
    low = np.tril(np.ones((14, 14), dtype=bool))
    np.testing.assert_allclose(z[low], A[low], atol=1e-12)
    assert np.abs(A[~low]).max() < 1e-11  # zero up to the solve's rounding


# ---------------------------------------------------------------- backward pins
def torch_explicit_loss(q, k, v, w, beta, logf, dout, scale):
    """sum(o * dO) of PaTH(-FoX) written with explicit d x d matrices (autograd)."""
    B, H, L, d = q.shape
    total = q.new_zeros(())
    eye = torch.eye(d, dtype=q.dtype)
    for b in range(B):
        for h in range(H):
            c = torch.cumsum(logf[b, h], 0) if logf is not None else q.new_zeros(L)
            Hs = [eye - beta[b, h, s] * torch.outer(w[b, h, s], w[b, h, s]) for s in range(L)]
            rows = []
            for i in range(L):
                M = eye
                zs = []
                for j in range(i, -1, -1):
                    zs.append(scale * (q[b, h, i] @ M @ k[b, h, j]) + c[i] - c[j])
                    M = M @ Hs[j]
                z = torch.stack(zs[::-1])
                p = torch.softmax(z, 0)
                rows.append(p @ v[b, h, : i + 1])
            o = torch.stack(rows)
            total = total + (o * dout[b, h]).sum()
    return total


@pytest.mark.parametrize("fox", [False, True])
def test_bwd_equals_autograd_of_explicit_matrices(orc, fox):
    rng = np.random.default_rng(12 + fox)
    q, k, v, w, beta, logf = rand_case(rng, B=1, H=2, L=8, d=4, fox=fox, unit_w=fox)
    dout = rng.standard_normal(q.shape)
    g = orc.bwd(q, k, v, w, beta, dout, logf, scale=0.8)
    ts = [torch.tensor(a, requires_grad=True) for a in (q, k, v, w, beta)]
    tl = torch.tensor(logf, requires_grad=True) if fox else None
    loss = torch_explicit_loss(*ts, tl, torch.from_numpy(dout), 0.8)
    grads = torch.autograd.grad(loss, ts + ([tl] if fox else []))
    names = ["dq", "dk", "dv", "dw", "dbeta"] + (["dlog_f"] if fox else [])
    for n, ref in zip(names, grads):
        np.testing.assert_allclose(g[n], ref.numpy(), rtol=1e-9, atol=1e-11, err_msg=n)


def test_bwd_equals_central_finite_differences(orc):
    rng = np.random.default_rng(14)
    q, k, v, w, beta, logf = rand_case(rng, B=1, H=1, L=7, d=3, fox=True)
    dout = rng.standard_normal(q.shape)
    g = orc.bwd(q, k, v, w, beta, dout, logf, scale=0.6)
    args = dict(q=q, k=k, v=v, w=w, beta=beta, log_f=logf)

    def loss(a):
        o, _ = orc.fwd(a["q"], a["k"], a["v"], a["w"], a["beta"], a["log_f"], scale=0.6)
        return float(np.sum(o * dout))

    eps = 1e-6
    for name, gname in [("q", "dq"), ("k", "dk"), ("v", "dv"), ("w", "dw"), ("beta", "dbeta"),
                        ("log_f", "dlog_f")]:
        base = args[name]
        fd = np.zeros_like(base)
        for idx in np.ndindex(base.shape):
            plus = {**args, name: base.copy()}
            minus = {**args, name: base.copy()}
            plus[name][idx] += eps
            minus[name][idx] -= eps
            fd[idx] = (loss(plus) - loss(minus)) / (2 * eps)
        np.testing.assert_allclose(g[gname], fd, rtol=1e-6, atol=1e-8, err_msg=gname)


def test_gradient_invariants(orc):
    """Symmetries of the loss fix these sums exactly: q -> a q, k -> k / a;
    w -> a w, beta -> beta / a^2; v -> v + const; and position 0's w, beta and
    log f never enter a logit."""
    rng = np.random.default_rng(15)
    q, k, v, w, beta, logf = rand_case(rng, B=2, H=2, L=37, d=7, fox=True)
    dout = rng.standard_normal(q.shape)
    g = orc.bwd(q, k, v, w, beta, dout, logf)
    np.testing.assert_allclose(np.sum(q * g["dq"], axis=(-1, -2)),
                               np.sum(k * g["dk"], axis=(-1, -2)), rtol=1e-10)
    np.testing.assert_allclose(np.sum(w * g["dw"], axis=(-1, -2)),
                               2 * np.sum(beta * g["dbeta"], axis=-1), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(g["dv"].sum(axis=-2), dout.sum(axis=-2), rtol=1e-10)
    assert np.all(g["dw"][..., 0, :] == 0) and np.all(g["dbeta"][..., 0] == 0)
    assert np.all(np.abs(g["dlog_f"][..., 0]) < 1e-10)
    # w -> -w: H unchanged, so outputs unchanged and dw flips sign
    g2 = orc.bwd(q, k, v, -w, beta, dout, logf)
    np.testing.assert_allclose(g2["dw"], -g["dw"], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(g2["dbeta"], g["dbeta"], rtol=1e-12, atol=1e-14)
    o1, _ = orc.fwd(q, k, v, w, beta, logf)
    o2, _ = orc.fwd(q, k, v, -w, beta, logf)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- decode pins
def test_decode_replay_equals_forward_rows(orc):
    """Paper-Notes "训练策略", inference paragraph: updating the cached keys in
    place and attending with the raw query reproduces the training forward."""
    rng = np.random.default_rng(16)
    q, k, v, w, beta, _ = rand_case(rng, B=2, H=2, L=25, d=6)
    out, _ = orc.fwd(q, k, v, w, beta, scale=0.4)
    kc = np.zeros((2, 2, 25, 6))
    vc = np.zeros((2, 2, 25, 6))
    for t in range(25):
        o = orc.decode_step(q[:, :, t], k[:, :, t], v[:, :, t], w[:, :, t], beta[:, :, t], kc, vc,
                            t, scale=0.4)
        np.testing.assert_allclose(o, out[:, :, t], rtol=1e-11, atol=1e-13)


def test_round_bf16_matches_library_conversion(orc):
    rng = np.random.default_rng(17)
    x = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 2 ** -130, 3e-39]),
    ]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    got = np.array([orc.round_bf16(float(a)) for a in x])
    np.testing.assert_array_equal(got, ref)


def test_decode_bf16_cache_is_rounded_update(orc):
    rng = np.random.default_rng(18)
    B, H, cap, d, n = 1, 2, 40, 8, 30
    base = torch.randn(B, H, cap, d).bfloat16().double().numpy()
    base[:, :, n:] = 0
    q, kn, vn, w = (torch.randn(B, H, d).bfloat16().double().numpy() for _ in range(4))
    beta = rng.uniform(0, 1.99, (B, H))
    k64, v64 = base.copy(), base.copy()
    kb, vb = base.copy(), base.copy()
    orc.decode_step(q, kn, vn, w, beta, k64, v64, n)
    orc.decode_step(q, kn, vn, w, beta, kb, vb, n, round_bf16=True)
    ref = np.vectorize(orc.round_bf16)(k64[:, :, :n])
    np.testing.assert_array_equal(kb[:, :, :n], ref)
    np.testing.assert_array_equal(kb[:, :, n], kn)


def test_gated_decode_replay_equals_forward_rows(orc):
    """PaTH-FoX decode: each cached key carries its gate bias c_t - c_j, grown in
    place by log f_t at every step (Paper-Notes "PaTH-FoX 扩展" logit term, carried
    like the in-place key update of "训练策略"); replay reproduces the forward."""
    rng = np.random.default_rng(19)
    q, k, v, w, beta, logf = rand_case(rng, B=2, H=2, L=21, d=6, fox=True)
    out, _ = orc.fwd(q, k, v, w, beta, logf, scale=0.5)
    kc, vc, gc = np.zeros((2, 2, 21, 6)), np.zeros((2, 2, 21, 6)), np.zeros((2, 2, 21))
    for t in range(21):
        o = orc.decode_step(q[:, :, t], k[:, :, t], v[:, :, t], w[:, :, t], beta[:, :, t], kc, vc,
                            t, scale=0.5, log_f=logf[:, :, t], g_cache=gc)
        np.testing.assert_allclose(o, out[:, :, t], rtol=1e-11, atol=1e-13)


# ---------------------------------------------------------------- prefill cache pins
def test_prefill_cache_equals_explicit_products(orc):
    """Row j of the cache after positions 0..L-1 is H_{L-1} ... H_{j+1} k_j, and its gate
    bias is the sum of log f_s over s = j+1..L-1 (Paper-Notes "训练策略", inference
    paragraph; "PaTH-FoX 扩展")."""
    rng = np.random.default_rng(20)
    B, H, L, d, cap = 2, 2, 11, 5, 14
    q, k, v, w, beta, logf = rand_case(rng, B=B, H=H, L=L, d=d, fox=True)
    kc, vc, gc = orc.prefill_cache(k, v, w, beta, logf, capacity=cap)
    for b in range(B):
        for h in range(H):
            M = np.eye(d)  # H_{L-1} ... H_{j+1}, built by right-multiplying as j decreases
            for j in range(L - 1, -1, -1):
                np.testing.assert_allclose(kc[b, h, j], M @ k[b, h, j], rtol=1e-12, atol=1e-13)
                assert gc[b, h, j] == pytest.approx(math.fsum(logf[b, h, j + 1:]), rel=1e-12,
                                                    abs=1e-13)
                M = M @ householder(w[b, h, j], beta[b, h, j])
    np.testing.assert_array_equal(vc[:, :, :L], v)
    assert not kc[:, :, L:].any() and not vc[:, :, L:].any() and not gc[:, :, L:].any()
    kc2, _, gc2 = orc.prefill_cache(k, v, w, beta, None, capacity=cap)
    np.testing.assert_array_equal(kc2, kc)
    assert gc2 is None


def test_prefill_cache_last_row_attention_is_forward_row(orc):
    """Softmax attention of q_{L-1} over the prefill cache (logits scale q.k_j + g_j, a
    library softmax) gives the forward's last output row and log-sum-exp."""
    rng = np.random.default_rng(21)
    q, k, v, w, beta, logf = rand_case(rng, B=1, H=3, L=13, d=4, fox=True)
    out, lse = orc.fwd(q, k, v, w, beta, logf, scale=0.7)
    kc, vc, gc = orc.prefill_cache(k, v, w, beta, logf)
    z = torch.from_numpy(0.7 * np.einsum("bhd,bhjd->bhj", q[:, :, -1], kc) + gc)
    p = torch.softmax(z, -1).numpy()
    np.testing.assert_allclose(np.einsum("bhj,bhjd->bhd", p, vc), out[:, :, -1], rtol=1e-11,
                               atol=1e-13)
    np.testing.assert_allclose(torch.logsumexp(z, -1).numpy(), lse[:, :, -1], rtol=1e-11)


@pytest.mark.parametrize("fox", [False, True])
def test_decode_after_prefill_continues_the_forward(orc, fox):
    """A prefill of the first L0 positions followed by decode steps reproduces the
    forward rows L0.. of the whole sequence."""
    rng = np.random.default_rng(22)
    L0, L = 9, 14
    q, k, v, w, beta, logf = rand_case(rng, B=2, H=2, L=L, d=5, fox=fox)
    out, _ = orc.fwd(q, k, v, w, beta, logf, scale=0.6)
    head = lambda a: None if a is None else a[:, :, :L0]
    kc, vc, gc = orc.prefill_cache(head(k), head(v), head(w), head(beta), head(logf), capacity=L)
    for t in range(L0, L):
        o = orc.decode_step(q[:, :, t], k[:, :, t], v[:, :, t], w[:, :, t], beta[:, :, t], kc, vc,
                            t, scale=0.6, log_f=None if logf is None else logf[:, :, t],
                            g_cache=gc)
        np.testing.assert_allclose(o, out[:, :, t], rtol=1e-11, atol=1e-13)


# ---------------------------------------------------------------- randomized pins
# The fixed-seed pins above, over random shapes, beta in [0, 2], unnormalised w
# and gate on / off (hypothesis draws the case; numpy draws the values from its seed).
CASES = st.tuples(st.integers(1, 9), st.integers(1, 5), st.floats(0.0, 2.0),
                  st.booleans(), st.booleans(), st.integers(0, 2 ** 31 - 1))


@settings(max_examples=40, deadline=None)
@given(CASES)
def test_random_scores_equal_explicit_products(case):
    L, d, beta_hi, unit_w, fox, seed = case
    rng = np.random.default_rng(seed)
    q, k, v, w, beta, logf = rand_case(rng, B=1, H=1, L=L, d=d, beta_hi=beta_hi, unit_w=unit_w,
                                       fox=fox)
    z = oracle.scores(q, k, w, beta, logf, scale=0.9)[0, 0]
    ref = explicit_scores(q[0, 0], k[0, 0], w[0, 0], beta[0, 0],
                          None if logf is None else logf[0, 0], 0.9)
    np.testing.assert_allclose(z, ref, rtol=1e-10, atol=1e-10)


@settings(max_examples=25, deadline=None)
@given(CASES)
def test_random_decode_and_prefill_agree_with_forward(case):
    L, d, beta_hi, unit_w, fox, seed = case
    rng = np.random.default_rng(seed)
    q, k, v, w, beta, logf = rand_case(rng, B=1, H=2, L=L, d=d, beta_hi=beta_hi, unit_w=unit_w,
                                       fox=fox)
    out, _ = oracle.fwd(q, k, v, w, beta, logf, scale=0.7)
    kc, vc, gc = np.zeros((1, 2, L, d)), np.zeros((1, 2, L, d)), np.zeros((1, 2, L))
    for t in range(L):
        o = oracle.decode_step(q[:, :, t], k[:, :, t], v[:, :, t], w[:, :, t], beta[:, :, t],
                               kc, vc, t, scale=0.7,
                               log_f=None if logf is None else logf[:, :, t],
                               g_cache=gc if fox else None)
        np.testing.assert_allclose(o, out[:, :, t], rtol=1e-9, atol=1e-11)
    pk, pv, pg = oracle.prefill_cache(k, v, w, beta, logf)
    np.testing.assert_allclose(pk, kc, rtol=1e-12, atol=1e-13)
    np.testing.assert_array_equal(pv, vc)
    if fox:
        np.testing.assert_allclose(pg, gc, rtol=1e-12, atol=1e-13)


@settings(max_examples=15, deadline=None)
@given(CASES)
def test_random_gradient_invariants(case):
    L, d, beta_hi, unit_w, fox, seed = case
    rng = np.random.default_rng(seed)
    q, k, v, w, beta, logf = rand_case(rng, B=1, H=1, L=L, d=d, beta_hi=beta_hi, unit_w=unit_w,
                                       fox=fox)
    dout = rng.standard_normal(q.shape)
    g = oracle.bwd(q, k, v, w, beta, dout, logf, scale=0.8)
    # scaling q by s and k by 1/s leaves every logit unchanged: sum q.dq = sum k.dk
    assert math.isclose(float(np.sum(q * g["dq"])), float(np.sum(k * g["dk"])),
                        rel_tol=1e-8, abs_tol=1e-9)
    # H depends on w only through beta w w^T: sum w.dw = 2 sum beta dbeta
    assert math.isclose(float(np.sum(w * g["dw"])), float(2 * np.sum(beta * g["dbeta"])),
                        rel_tol=1e-8, abs_tol=1e-9)
    # the rows of softmax sum to one: sum over keys of dv is sum over queries of dout
    np.testing.assert_allclose(g["dv"].sum(axis=-2), dout.sum(axis=-2), rtol=1e-9, atol=1e-10)


# ---------------------------------------------------------------- planted mistakes
MUTATIONS = [
    # (name, regex on the source, replacement, pin that must fail)
    ("h_sign", r"x\[e\] -= a \* w_s\[e\]", "x[e] += a * w_s[e]", "scores"),
    ("append_before_update", r"for \(int j = 0; j < t; \+\+j\) apply_h",
     "for (int j = 0; j < t - 1; ++j) apply_h", "scores"),
    ("gate_sign", r"\(c\[t\] - c\[j\]\)", "(c[j] - c[t])", "fox_fwd"),
    ("dw_drop_term", r"b \* \(ux \* g\[e\] \+ gu \* x\[e\]\)", "b * (ux * g[e])", "grad"),
    ("dbeta_sign", r"a->dbeta\[j \+ 1\] -= gu \* ux", "a->dbeta[j + 1] += gu * ux", "grad"),
    ("dc_key_sign", r"a->dc\[j\] -= dz", "a->dc[j] += dz", "grad"),
    ("g_transport_sign", r"g\[e\] -= b \* gu \* u\[e\]", "g[e] += b * gu * u[e]", "grad"),
    ("round_ties_away", r"nearbyint\(x / ulp\)", "round(x / ulp)", "round"),
    ("decode_gate_not_carried", r"if \(g\) g\[j\] \+= \*logf_t;", ";", "gated_decode"),
    ("prefill_skips_newest_key", r"for \(int j = t - 1; j >= 0; --j\)",
     "for (int j = t - 2; j >= 0; --j)", "prefill"),
    ("prefill_gate_sign", r"if \(g\) g\[j\] \+= log_f\[in0 \+ t\];",
     "if (g) g[j] -= log_f[in0 + t];", "prefill"),
]


def _mutant(tmpdir, name, pattern, repl):
    src = open(oracle.SOURCE).read()
    mutated, n = re.subn(pattern, repl, src)
    assert n >= 1, f"mutation {name} did not apply"
    path = os.path.join(tmpdir, f"{name}.c")
    with open(path, "w") as f:
        f.write(mutated)
    return oracle.Oracle(oracle.compile_source(path, os.path.join(tmpdir, f"lib{name}.so")))


def _pin_passes(orc, pin):
    rng = np.random.default_rng(99)
    try:
        if pin == "scores":
            q, k, v, w, beta, _ = rand_case(rng, B=1, H=1, L=8, d=4)
            z = orc.scores(q, k, w, beta, scale=1.0)[0, 0]
            ref = explicit_scores(q[0, 0], k[0, 0], w[0, 0], beta[0, 0], None, 1.0)
            np.testing.assert_allclose(z, ref, rtol=1e-10, atol=1e-12)
        elif pin == "fox_fwd":
            q, k, v, w, beta, logf = rand_case(rng, B=1, H=1, L=8, d=4, fox=True)
            z = orc.scores(q, k, w, beta, logf, scale=1.0)[0, 0]
            ref = explicit_scores(q[0, 0], k[0, 0], w[0, 0], beta[0, 0], logf[0, 0], 1.0)
            np.testing.assert_allclose(z, ref, rtol=1e-10, atol=1e-12)
        elif pin == "grad":
            q, k, v, w, beta, logf = rand_case(rng, B=1, H=1, L=6, d=3, fox=True)
            dout = rng.standard_normal(q.shape)
            g = orc.bwd(q, k, v, w, beta, dout, logf, scale=0.8)
            ts = [torch.tensor(a, requires_grad=True) for a in (q, k, v, w, beta, logf)]
            loss = torch_explicit_loss(*ts, torch.from_numpy(dout), 0.8)
            grads = torch.autograd.grad(loss, ts)
            for n, ref in zip(["dq", "dk", "dv", "dw", "dbeta", "dlog_f"], grads):
                np.testing.assert_allclose(g[n], ref.numpy(), rtol=1e-9, atol=1e-11)
        elif pin == "gated_decode":
            q, k, v, w, beta, logf = rand_case(rng, B=1, H=1, L=7, d=4, fox=True)
            z = explicit_scores(q[0, 0], k[0, 0], w[0, 0], beta[0, 0], logf[0, 0], 1.0)
            kc, vc, gc = np.zeros((1, 1, 7, 4)), np.zeros((1, 1, 7, 4)), np.zeros((1, 1, 7))
            for t in range(7):
                o = orc.decode_step(q[:, :, t], k[:, :, t], v[:, :, t], w[:, :, t],
                                    beta[:, :, t], kc, vc, t, scale=1.0, log_f=logf[:, :, t],
                                    g_cache=gc)
                p = torch.softmax(torch.from_numpy(z[t, :t + 1]), -1).numpy()
                np.testing.assert_allclose(o[0, 0], p @ v[0, 0, :t + 1], rtol=1e-10, atol=1e-12)
        elif pin == "prefill":
            q, k, v, w, beta, logf = rand_case(rng, B=1, H=1, L=7, d=4, fox=True)
            kc, _, gc = orc.prefill_cache(k, v, w, beta, logf)
            M = np.eye(4)
            for j in range(6, -1, -1):
                np.testing.assert_allclose(kc[0, 0, j], M @ k[0, 0, j], rtol=1e-10, atol=1e-12)
                np.testing.assert_allclose(gc[0, 0, j], logf[0, 0, j + 1:].sum(), rtol=1e-10,
                                           atol=1e-12)
                M = M @ householder(w[0, 0, j], beta[0, 0, j])
        elif pin == "round":
            x = np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8)], dtype=np.float32)
            ref = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
            np.testing.assert_array_equal([orc.round_bf16(float(a)) for a in x], ref)
    except AssertionError:
        return False
    return True


def test_pins_pass_on_the_real_oracle(orc):
    for pin in {m[3] for m in MUTATIONS}:
        assert _pin_passes(orc, pin), pin


@pytest.mark.parametrize("mutation", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_planted_mistakes(mutation):
    name, pattern, repl, pin = mutation
    with tempfile.TemporaryDirectory() as tmp:
        bad = _mutant(tmp, name, pattern, repl)
        assert not _pin_passes(bad, pin), f"pin '{pin}' missed planted mistake '{name}'"
