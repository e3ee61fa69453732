"""The w / beta prologue of PaTH attention in fp64: the plain reference (test
infrastructure only; the CUDA library never calls it and shares no code with it).

What it computes (Paper-Notes "关键设计": w_t comes from a low-rank linear layer,
a short convolution with filter size 3 and L2 normalisation, and
beta_t = 2 sigmoid(u^T x_t + b); the same beta on the gist.science page, section 2
"Kernmechanisme"), per sequence b, position t and head h, with the plainest
readings where the pages leave a step open:

- low-rank linear layer: wt_t = (x_t A) Bw, A [D, r], Bw [r, H d]; no bias and no
  activation between the two factors;
- short convolution: one filter of 3 taps per channel c of the H d channels,
  causal: z_t[c] = sum_{k=0..2} f[c, k] wt_{t-k}[c], with wt before the start of the
  sequence taken as 0 (tap k reaches k positions back);
- L2 normalisation of each head's d channels: w_t^h = z_t^h / max(|z_t^h|, EPS);
- beta_t^h = min(2 sigmoid(x_t . u_h + b_h), beta_max), U = [u_1 .. u_H] is [D, H];
  beta_max = 2 leaves beta unclipped (bf16 training clips it below 2: atlas.scime.ai
  "Limitations", gist.science section 6).

Layouts: x [B, L, D]; w [B, H, L, d]; beta [B, H, L] (the attention's inputs).
The backward is the chain rule through these steps, written out by hand below;
tests/test_oracle_wbeta.py pins it against autograd of a formulation built from
library routines, finite differences and invariants.
"""
from __future__ import annotations

import numpy as np

EPS = 1e-6


def _f64(a):
    if a is None:
        return None
    if hasattr(a, "detach"):
        a = a.detach().double().cpu().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _shift(a, k):
    """a[:, t - k] along the sequence axis 1, zero before the start."""
    if k == 0:
        return a
    out = np.zeros_like(a)
    out[:, k:] = a[:, :-k]
    return out


def _unshift(a, k):
    """a[:, t + k] along the sequence axis 1, zero past the end."""
    if k == 0:
        return a
    out = np.zeros_like(a)
    out[:, :-k] = a[:, k:]
    return out


def forward(x, A, Bw, f, u, b, H, beta_max=2.0):
    """w [B, H, L, d], beta [B, H, L] and the intermediates the backward reads."""
    x, A, Bw, f, u, b = (_f64(t) for t in (x, A, Bw, f, u, b))
    Bn, L, D = x.shape
    Hd = Bw.shape[1]
    d = Hd // H
    y = x @ A                                  # [B, L, r]
    wt = y @ Bw                                # [B, L, H d]
    z = sum(f[:, k] * _shift(wt, k) for k in range(3))
    zh = z.reshape(Bn, L, H, d)
    nrm = np.sqrt(np.sum(zh * zh, axis=-1))     # [B, L, H]
    m = np.maximum(nrm, EPS)
    w = zh / m[..., None]
    s = x @ u + b                              # [B, L, H]
    sig = 1.0 / (1.0 + np.exp(-s))
    beta_raw = 2.0 * sig
    beta = np.minimum(beta_raw, beta_max)
    cache = dict(x=x, A=A, Bw=Bw, f=f, u=u, y=y, wt=wt, nrm=nrm, w=w, sig=sig, beta_raw=beta_raw,
                 H=H, d=d, beta_max=beta_max)
    return w.transpose(0, 2, 1, 3).copy(), beta.transpose(0, 2, 1).copy(), cache


def backward(cache, dw, dbeta):
    """Gradients of sum(w * dw) + sum(beta * dbeta) with respect to x, A, Bw, f, u, b."""
    dw, dbeta = _f64(dw), _f64(dbeta)
    x, A, Bw, f, u = (cache[k] for k in ("x", "A", "Bw", "f", "u"))
    H, d = cache["H"], cache["d"]
    Bn, L, D = x.shape
    # beta = min(2 sigmoid(s), beta_max): no gradient where the clip holds
    db_t = dbeta.transpose(0, 2, 1)            # [B, L, H]
    open_ = cache["beta_raw"] < cache["beta_max"]
    sig = cache["sig"]
    ds = np.where(open_, db_t * 2.0 * sig * (1.0 - sig), 0.0)
    du = x.reshape(-1, D).T @ ds.reshape(-1, H)
    db = ds.reshape(-1, H).sum(axis=0)
    dx = ds @ u.T
    # w = z / max(|z|, EPS): the part of dw along w drops out where |z| > EPS
    g = dw.transpose(0, 2, 1, 3)               # [B, L, H, d]
    w, nrm = cache["w"], cache["nrm"]
    along = np.sum(w * g, axis=-1, keepdims=True)
    big = (nrm > EPS)[..., None]
    dzh = np.where(big, (g - w * along) / np.maximum(nrm, EPS)[..., None], g / EPS)
    dz = dzh.reshape(Bn, L, H * d)
    # causal 3-tap convolution: its adjoint reaches forward in time
    wt = cache["wt"]
    dwt = sum(f[:, k] * _unshift(dz, k) for k in range(3))
    df = np.stack([np.sum(dz * _shift(wt, k), axis=(0, 1)) for k in range(3)], axis=1)
    # wt = (x A) Bw
    y = cache["y"]
    dBw = y.reshape(-1, y.shape[-1]).T @ dwt.reshape(-1, H * d)
    dy = dwt @ Bw.T
    dA = x.reshape(-1, D).T @ dy.reshape(-1, dy.shape[-1])
    dx = dx + dy @ A.T
    return dict(dx=dx, dA=dA, dBw=dBw, df=df, du=du, db=db)


def fwd(x, A, Bw, f, u, b, H, beta_max=2.0):
    w, beta, _ = forward(x, A, Bw, f, u, b, H, beta_max)
    return w, beta


def bwd(x, A, Bw, f, u, b, H, beta_max=2.0, *, dw, dbeta):
    return backward(forward(x, A, Bw, f, u, b, H, beta_max)[2], dw, dbeta)
