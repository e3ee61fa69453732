"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Tolerances (max absolute error): 1e-4 for fp32 inputs, 2e-2 for bf16 inputs
with fp32 accumulation, on outputs, lse and every gradient. Both sides read
identical input bytes from ``synthetic_inputs``; the oracle sees them exactly
(upcast to fp64).
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic_inputs as si

pytestmark = pytest.mark.gpu

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


@pytest.fixture(scope="module")
def P():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import softmax_attention_block_b200 as P

    P.lib()
    return P


def to_dev(x):
    return {k: (v.cuda() if v is not None else None) for k, v in x.items()}


def maxerr(a, b):
    a = a.detach().float().cpu().double().numpy() if hasattr(a, "detach") else np.asarray(a)
    return float(np.max(np.abs(a - b))) if a.size else 0.0


def run_ours(P, x, backward):
    d = to_dev(x)
    out, lse = P.path_attn_fwd(d["q"], d["k"], d["v"], d["w"], d["beta"], d["log_f"])
    g = None
    if backward:
        g = P.path_attn_bwd(d["q"], d["k"], d["v"], d["w"], d["beta"], out, lse, d["dout"],
                            d["log_f"])
    torch.cuda.synchronize()
    return out, lse, g


def check(P, x, backward, tol, report=""):
    out, lse, g = run_ours(P, x, backward)
    ro, rl = oracle.fwd(x["q"], x["k"], x["v"], x["w"], x["beta"], x["log_f"])
    errs = {"out": maxerr(out, ro), "lse": maxerr(lse, rl)}
    if backward:
        rg = oracle.bwd(x["q"], x["k"], x["v"], x["w"], x["beta"], x["dout"], x["log_f"])
        for n, ref in rg.items():
            errs[n] = maxerr(g[n], ref)
            errs[n + "/max|ref|"] = errs[n] / max(float(np.max(np.abs(ref))), 1e-30)
    print(f"\n[{report}] " + " ".join(f"{k}={v:.3g}" for k, v in errs.items()))
    bad = {k: v for k, v in errs.items() if "/" not in k and not v <= tol}
    assert not bad, f"{report}: over tolerance {tol}: {bad}"
    return errs


def test_fp32_tiny_forward(P):
    x = si.workload_inputs("fwd_fp32_tiny")
    check(P, x, backward=False, tol=1e-4, report="fwd_fp32_tiny")


@pytest.mark.parametrize("L,d,fox", [(1, 16, False), (64, 16, True), (300, 32, True),
                                     (257, 64, False), (130, 128, True)])
def test_fp32_fwd_bwd_shapes(P, L, d, fox):
    x = si.make_inputs(1, 2, L, d, torch.float32, seed=1, fox=fox, clip_beta=False)
    check(P, x, backward=True, tol=1e-4, report=f"fp32 L={L} d={d} fox={fox}")


def test_bf16_l1024_forward(P):
    x = si.workload_inputs("fwd_bf16_l1024")
    check(P, x, backward=False, tol=2e-2, report="fwd_bf16_l1024")


@pytest.mark.parametrize("L,d,fox", [(1, 64, False), (100, 64, True), (128, 64, False),
                                     (257, 64, True), (600, 16, False), (333, 32, True),
                                     (390, 128, True)])
def test_bf16_fwd_bwd_ragged(P, L, d, fox):
    x = si.make_inputs(2, 2, L, d, torch.bfloat16, seed=2, fox=fox)
    check(P, x, backward=True, tol=2e-2, report=f"bf16 L={L} d={d} fox={fox}")


def test_bf16_l1024_fwd_bwd(P):
    x = si.make_inputs(2, 4, 1024, 64, torch.bfloat16, seed=0)
    check(P, x, backward=True, tol=2e-2, report="bf16 l1024 fwd+bwd")


def _sampled_full_size(P, name, heads):
    """Full-size run on the GPU, oracle on a few heads (heads are independent)."""
    w = si.WORKLOADS[name]
    x = si.workload_inputs(name)
    out, lse, g = run_ours(P, x, backward=True)
    flat = lambda t: t.reshape(w.B * w.H, *t.shape[2:])[heads]
    xs = si.workload_inputs(name, heads=heads)
    ro, rl = oracle.fwd(xs["q"], xs["k"], xs["v"], xs["w"], xs["beta"], xs["log_f"])
    rg = oracle.bwd(xs["q"], xs["k"], xs["v"], xs["w"], xs["beta"], xs["dout"], xs["log_f"])
    errs = {"out": maxerr(flat(out), ro[0]), "lse": maxerr(flat(lse), rl[0])}
    for n, ref in rg.items():
        errs[n] = maxerr(flat(g[n]), ref[0])
        errs[n + "/max|ref|"] = errs[n] / max(float(np.max(np.abs(ref))), 1e-30)
    print(f"\n[{name} heads {heads}] " + " ".join(f"{k}={v:.3g}" for k, v in errs.items()))
    bad = {k: v for k, v in errs.items() if "/" not in k and not v <= 2e-2}
    assert not bad, f"{name}: over tolerance: {bad}"


def test_full_size_l4096_sampled_heads(P):
    _sampled_full_size(P, "fwdbwd_bf16_l4096", [0, 77, 191])


def test_full_size_fox_l16384_sampled_heads(P):
    _sampled_full_size(P, "fox_fwdbwd_l16384", [5])


def _decode_check(P, B, H, d, n0, cap, steps, dtype, heads, tol):
    kc, vc, seq = si.make_decode_inputs(B, H, d, n0, cap, steps, dtype, seed=3)
    kd, vd = kc.cuda(), vc.cuda()
    sel = lambda t: t.reshape(B * H, *t.shape[2:])[heads].unsqueeze(0)
    ok = sel(kc).double().numpy().copy()
    ov = sel(vc).double().numpy().copy()
    worst = 0.0
    for t, s in enumerate(seq):
        sd = {k: v.cuda() for k, v in s.items()}
        out = P.path_decode_step(sd["q"], sd["k_new"], sd["v_new"], sd["w"], sd["beta"], kd, vd,
                                 n0 + t)
        ref = oracle.decode_step(sel(s["q"]), sel(s["k_new"]), sel(s["v_new"]), sel(s["w"]),
                                 sel(s["beta"]), ok, ov, n0 + t,
                                 round_bf16=(dtype == torch.bfloat16))
        worst = max(worst, maxerr(sel(out.cpu()), ref))
    torch.cuda.synchronize()
    n = n0 + steps
    kg = sel(kd.cpu())[..., :n, :].double().numpy()
    kref = ok[..., :n, :]
    if dtype == torch.bfloat16:
        # cache entries within 2 bf16 ulps (relative 2^-7) of the oracle's rounded cache
        ulp = np.maximum(np.abs(kref), 1e-30) * 2.0 ** -7
        cache_bad = int(np.sum(np.abs(kg - kref) > 2 * ulp + 1e-6))
    else:
        cache_bad = int(np.sum(np.abs(kg - kref) > 1e-4))
    print(f"\n[decode B={B} H={H} d={d} n0={n0} steps={steps}] out max err {worst:.3g}, "
          f"cache entries beyond tolerance {cache_bad}")
    np.testing.assert_array_equal(sel(vd.cpu())[..., :n, :].double().numpy(), ov[..., :n, :])
    assert worst <= tol
    assert cache_bad == 0


@pytest.mark.parametrize("dtype,d", [(torch.float32, 64), (torch.bfloat16, 64),
                                     (torch.bfloat16, 128)])
def test_decode_small(P, dtype, d):
    _decode_check(P, 2, 3, d, 700, 720, 5, dtype, list(range(6)), TOL[dtype])


def test_decode_from_empty_cache(P):
    _decode_check(P, 1, 2, 64, 0, 40, 30, torch.float32, [0, 1], 1e-4)


def test_decode_full_size_sampled_heads(P):
    _decode_check(P, 32, 32, 128, 16384, 16448, 64, torch.bfloat16, [0, 513, 1023], 2e-2)


def test_launch_counter_advances(P):
    before = P.lib().path_kernel_launch_count()
    x = si.make_inputs(1, 1, 200, 64, torch.bfloat16, seed=5)
    run_ours(P, x, backward=True)
    assert P.lib().path_kernel_launch_count() > before
