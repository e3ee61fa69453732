"""GPU parity of the w / beta prologue (path_wbeta_fwd / path_wbeta_bwd, through the C
ABI) against the fp64 oracle (oracle/wbeta.py) on identical input bytes.

Bars (max absolute error, elementwise):
- fp32 inputs and outputs: 1e-4 on w and beta; 1e-4 max(1, max|ref|) on the
  gradients (the parameter gradients are sums over every position).
- bf16 inputs: 2e-2 on w and beta, 2e-2 max(1, max|ref|) on the gradients (the
  low-rank products run on TF32 tensor cores with fp32 accumulation; bf16 inputs
  are exact in TF32), plus one bf16 ulp of the reference where the result is
  stored in bf16 (w, dx).
Every output starts as NaN, so an element no kernel writes cannot pass.
"""
import numpy as np
import pytest
import torch

import oracle.wbeta as wb

from test_gpu_parity import ulp_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def P():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import softmax_attention_block_b200 as P

    P.lib()
    return P


def inputs(B, L, D, r, H, d, dtype, out_dtype, seed):
    g = torch.Generator().manual_seed(seed)
    rn = lambda *s: torch.randn(*s, generator=g)
    x = rn(B, L, D).to(dtype)
    A = (rn(D, r) / D ** 0.5).to(dtype)
    Bw = (rn(r, H * d) / r ** 0.5).to(dtype)
    f = rn(H * d, 3) * 0.5 + torch.tensor([1.0, 0.0, 0.0])
    U = (rn(D, H) * (2.0 / D ** 0.5)).to(dtype)
    b = rn(H)
    dw = rn(B, H, L, d).to(out_dtype)
    dbeta = rn(B, H, L)
    return x, A, Bw, f, U, b, dw, dbeta


def nans(shape, dtype):
    return torch.full(shape, float("nan"), dtype=dtype, device="cuda")


def bar(name, ref, bf16_in, bf16_stored):
    big = max(1.0, float(np.abs(ref).max()))
    base = 1e-4 if not bf16_in else 2e-2
    tol = base if name in ("w", "beta") else base * big
    return tol + (ulp_bf16(ref) if bf16_stored else 0.0)


CASES = [
    # dtype, out dtype, B, L, D, r, H, d, beta_max
    (torch.float32, torch.float32, 2, 37, 48, 8, 3, 16, 2.0),
    (torch.float32, torch.float32, 1, 70, 64, 12, 2, 64, 1.2),
    (torch.bfloat16, torch.float32, 2, 300, 96, 16, 2, 64, 1.99),
    (torch.bfloat16, torch.bfloat16, 1, 260, 128, 32, 2, 64, 1.99),
    (torch.bfloat16, torch.float32, 1, 129, 64, 8, 1, 128, 1.5),
    (torch.bfloat16, torch.float32, 3, 5, 32, 4, 2, 32, 2.0),
]


def run_case(P, dtype, out_dtype, B, L, D, r, H, d, beta_max, seed=0):
    x, A, Bw, f, U, b, dw, dbeta = inputs(B, L, D, r, H, d, dtype, out_dtype, seed)
    dev = [t.cuda() for t in (x, A, Bw, f, U, b, dw, dbeta)]
    ws = torch.full((P.path_wbeta_workspace_bytes(B, L, D, r, H, d, dtype, True, out_dtype),), 0xFF,
                    dtype=torch.uint8, device="cuda")
    w, beta = P.path_wbeta_fwd(*dev[:6], H, beta_max, w=nans((B, H, L, d), out_dtype),
                               beta=nans((B, H, L), torch.float32), workspace=ws, out_dtype=out_dtype)
    grads = dict(dx=nans((B, L, D), out_dtype), dA=nans((D, r), torch.float32),
                 dBw=nans((r, H * d), torch.float32), df=nans((H * d, 3), torch.float32),
                 dU=nans((D, H), torch.float32), db=nans((H,), torch.float32))
    g = P.path_wbeta_bwd(*dev[:6], H, dev[6], dev[7], beta_max, grads=grads, workspace=ws,
                         reuse_fwd_workspace=True)
    torch.cuda.synchronize()
    rw, rbeta = wb.fwd(x, A, Bw, f, U, b, H, beta_max)
    rg = wb.bwd(x, A, Bw, f, U, b, H, beta_max, dw=dw, dbeta=dbeta)
    ours = {"w": w, "beta": beta, "dx": g["dx"], "dA": g["dA"], "dBw": g["dBw"], "df": g["df"],
            "du": g["dU"], "db": g["db"]}
    ref = {"w": rw, "beta": rbeta, **rg}
    bf16_in = dtype == torch.bfloat16
    errs, bad = {}, {}
    for n, r_ in ref.items():
        got = ours[n].float().cpu().double().numpy()
        assert np.isfinite(got).all(), f"{n}: elements never written (NaN sentinel left)"
        diff = np.abs(got - r_)
        stored = out_dtype == torch.bfloat16 and n in ("w", "dx")
        tol = bar(n, r_, bf16_in, stored)
        errs[n] = float(diff.max())
        if not np.all(diff <= tol):
            bad[n] = errs[n]
    print(f"\n[wbeta {dtype} -> {out_dtype} B={B} L={L} D={D} r={r} H={H} d={d} bmax={beta_max}] "
          + " ".join(f"{k}={v:.3g}" for k, v in errs.items()))
    assert not bad, f"over the bar: {bad}"


@pytest.mark.parametrize("case", CASES)
def test_wbeta_matches_oracle(P, case):
    run_case(P, *case)


def test_wbeta_headline_layer_width(P):
    """The layer width of the benchmark workload (24 heads of 64: D = 1536, rank 64) at
    L = 4096 on two sequences, bf16 inputs with fp32 outputs."""
    run_case(P, torch.bfloat16, torch.float32, 2, 4096, 1536, 64, 24, 64, 1.99, seed=1)
