"""Seeded synthetic inputs for PaTH attention (shared by the tests, the oracle
checks and the benchmark; holds none of the method's arithmetic).

Recipe (one PyTorch CPU generator, ``manual_seed(seed)``, draws in fp32 in the
order q, k, v, w, x_beta, z_f, dO, then the decode tensors):
- q, k, v, dO ~ N(0, 1);
- w rows ~ N(0, 1), L2-normalised in fp32 (the model layer normalises w);
- beta = 2 sigmoid(x), x ~ N(0, 1), clipped to [0, 1.99] for the bf16
  workloads (bf16 training needs clipped beta); beta stays fp32;
- log f = logsigmoid(z), z ~ N(3, 1), fp32 (PaTH-FoX only);
- everything stored in the workload dtype is rounded (nearest even) from the
  fp32 draw, so both sides read identical bytes.

Workloads named after what they are (sizes from the problem statement's
headline shapes):
- ``fwd_fp32_tiny``      fp32 forward, B=1 H=1 L=64 d=16, beta unclipped
- ``fwd_bf16_l1024``     bf16 forward, B=2 H=4 L=1024 d=64
- ``fwdbwd_bf16_l4096``  bf16 forward+backward, B=8 H=24 L=4096 d=64
- ``fox_fwdbwd_l16384``  bf16 PaTH-FoX forward+backward, B=1 H=24 L=16384 d=64
- ``fwdbwd_bf16_l4096_d128``  bf16 forward+backward at head dim 128, B=8 H=12 L=4096
  (the headline's model width as 12 heads of 128)
- ``decode_bf16_c16k``   bf16 decode, B=32 H=32 d=128, cache 16384 -> 16448, 64 steps
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    L: int
    d: int
    dtype: torch.dtype
    fox: bool = False
    clip_beta: bool = True
    backward: bool = False
    # decode only
    n0: int = 0
    steps: int = 0


WORKLOADS = {
    w.name: w
    for w in (
        Workload("fwd_fp32_tiny", 1, 1, 64, 16, torch.float32, clip_beta=False),
        Workload("fwd_bf16_l1024", 2, 4, 1024, 64, torch.bfloat16),
        Workload("fwdbwd_bf16_l4096", 8, 24, 4096, 64, torch.bfloat16, backward=True),
        Workload("fox_fwdbwd_l16384", 1, 24, 16384, 64, torch.bfloat16, fox=True,
                 backward=True),
        Workload("fwdbwd_bf16_l4096_d128", 8, 12, 4096, 128, torch.bfloat16, backward=True),
        Workload("decode_bf16_c16k", 32, 32, 0, 128, torch.bfloat16, n0=16384, steps=64),
    )
}

BETA_CLIP_MAX = 1.99


def _beta(x: torch.Tensor, clip: bool) -> torch.Tensor:
    b = 2.0 * torch.sigmoid(x)
    return b.clamp(0.0, BETA_CLIP_MAX) if clip else b


def make_inputs(B, H, L, d, dtype=torch.bfloat16, seed=0, fox=False, clip_beta=True,
                with_dout=True, out_dtype=None):
    """Training-shape inputs: dict of CPU tensors q, k, v, w [B,H,L,d] (dtype),
    beta [B,H,L] fp32, log_f [B,H,L] fp32 or None, dout [B,H,L,d] (out_dtype,
    default dtype) or None."""
    g = torch.Generator().manual_seed(seed)
    shp = (B, H, L, d)
    q = torch.randn(shp, generator=g)
    k = torch.randn(shp, generator=g)
    v = torch.randn(shp, generator=g)
    w = torch.randn(shp, generator=g)
    w = w / w.norm(dim=-1, keepdim=True).clamp_min(1e-30)
    xb = torch.randn((B, H, L), generator=g)
    zf = torch.randn((B, H, L), generator=g) + 3.0 if fox else None
    do = torch.randn(shp, generator=g) if with_dout else None
    out = dict(q=q.to(dtype), k=k.to(dtype), v=v.to(dtype), w=w.to(dtype),
               beta=_beta(xb, clip_beta).float().contiguous(),
               log_f=torch.nn.functional.logsigmoid(zf).float().contiguous() if fox else None,
               dout=do.to(out_dtype or dtype) if with_dout else None)
    return out


def workload_inputs(name: str, seed: int = 0, heads=None, out_dtype=None):
    """Inputs of a named training workload. ``heads`` (list of flat b*H+h
    indices) keeps only those heads, as B=1 H=len(heads) (same values)."""
    w = WORKLOADS[name]
    x = make_inputs(w.B, w.H, w.L, w.d, w.dtype, seed, fox=w.fox, clip_beta=w.clip_beta,
                    with_dout=True, out_dtype=out_dtype)
    if heads is not None:
        idx = torch.as_tensor(heads)
        for key, t in list(x.items()):
            if t is None:
                continue
            flat = t.reshape(w.B * w.H, *t.shape[2:])
            x[key] = flat[idx].unsqueeze(0).contiguous()
    return x


def make_decode_inputs(B, H, d, n0, capacity, steps, dtype=torch.bfloat16, seed=0,
                       clip_beta=True):
    """Decode inputs: k_cache, v_cache [B,H,capacity,d] (rows >= n0 zero) and a
    list of ``steps`` dicts with q, k_new, v_new, w [B,H,d] (dtype), beta [B,H] fp32."""
    if n0 + steps > capacity:
        raise ValueError("capacity too small for n0 + steps")
    g = torch.Generator().manual_seed(seed)
    kc = torch.zeros((B, H, capacity, d), dtype=dtype)
    vc = torch.zeros((B, H, capacity, d), dtype=dtype)
    if n0:
        kc[:, :, :n0] = torch.randn((B, H, n0, d), generator=g).to(dtype)
        vc[:, :, :n0] = torch.randn((B, H, n0, d), generator=g).to(dtype)
    seq = []
    for _ in range(steps):
        q = torch.randn((B, H, d), generator=g)
        kn = torch.randn((B, H, d), generator=g)
        vn = torch.randn((B, H, d), generator=g)
        w = torch.randn((B, H, d), generator=g)
        w = w / w.norm(dim=-1, keepdim=True).clamp_min(1e-30)
        xb = torch.randn((B, H), generator=g)
        seq.append(dict(q=q.to(dtype), k_new=kn.to(dtype), v_new=vn.to(dtype), w=w.to(dtype),
                        beta=_beta(xb, clip_beta).float().contiguous()))
    return kc, vc, seq
