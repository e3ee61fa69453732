"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Bars (max absolute error, elementwise, against the oracle on identical input
bytes):
- fp32 inputs and outputs: 1e-4 on out, lse and every gradient.
- bf16 inputs, fp32 accumulate, fp32 outputs (PATH_BF16_F32OUT): 2e-2 on out,
  lse and every gradient.
- bf16 inputs and bf16 outputs (PATH_BF16): 2e-2 plus one bf16 ulp of the
  reference value on the bf16-stored tensors (out, dq, dk, dv, dw): bf16 keeps
  8 significant bits, so a value of magnitude >= 8 cannot be stored closer
  than 2e-2. lse and dbeta (fp32) keep 2e-2. dlog_f (fp32) gets 2e-2 plus
  2^-7 max|dlog_f|: it is a sum of dZ over every (query, key) pair that
  straddles a position, and dZ carries delta = dout . out, which in this mode
  comes from the bf16-rounded out.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synthetic_inputs as si

pytestmark = pytest.mark.gpu

STORED_BF16 = ("out", "dq", "dk", "dv", "dw")


@pytest.fixture(scope="module")
def P():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import softmax_attention_block_b200 as P

    P.lib()
    return P


def to_dev(x):
    return {k: (v.cuda() if v is not None else None) for k, v in x.items()}


def np64(t):
    return t.detach().float().cpu().double().numpy() if hasattr(t, "detach") else np.asarray(t)


def ulp_bf16(x):
    """Spacing of bf16 numbers at |x| (8 significant bits)."""
    a = np.maximum(np.abs(x), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(a)) - 7)


def nans(shape, dtype):
    return torch.full(shape, float("nan"), dtype=dtype, device="cuda")


def assert_all_finite(ts, where):
    """Every element of every tensor was written: they all start as NaN."""
    for n, t in ts.items():
        bad = int((~torch.isfinite(t)).sum())
        assert bad == 0, f"{where}: {n} has {bad} elements never written (NaN sentinel left)"


def run_ours(P, x, backward, out_dtype=None, reuse=False):
    """The library on x. Outputs, gradients and the workspace start filled with NaN
    (the workspace as 0xFF bytes, a NaN in fp32 and fp16), so an element that no kernel
    writes, or a workspace value read before any kernel wrote it, cannot pass."""
    d = to_dev(x)
    B, H, L, D = d["q"].shape
    od = out_dtype or d["q"].dtype
    nb = max(P.path_attn_workspace_bytes(B, H, L, D, d["q"].dtype, bwd, od)
             for bwd in (False, backward))
    ws = torch.full((nb,), 0xFF, dtype=torch.uint8, device="cuda")
    out, lse = P.path_attn_fwd(d["q"], d["k"], d["v"], d["w"], d["beta"], d["log_f"],
                               out=nans(d["q"].shape, od), lse=nans((B, H, L), torch.float32),
                               workspace=ws)
    assert P.lib().path_attn_wait_status(ws.data_ptr(), None) == 0, "forward wait timed out"
    assert_all_finite({"out": out, "lse": lse}, "forward")
    g = None
    if backward:
        grads = {n: nans(d["q"].shape, od) for n in ("dq", "dk", "dv", "dw")}
        grads["dbeta"] = nans((B, H, L), torch.float32)
        if d["log_f"] is not None:
            grads["dlog_f"] = nans((B, H, L), torch.float32)
        g = P.path_attn_bwd(d["q"], d["k"], d["v"], d["w"], d["beta"], out, lse,
                            d["dout"].to(out.dtype), d["log_f"], grads=grads, workspace=ws,
                            reuse_fwd_workspace=reuse)
        assert P.lib().path_attn_wait_status(ws.data_ptr(), None) == 0, "backward wait timed out"
        assert_all_finite(g, "backward")
    torch.cuda.synchronize()
    return out, lse, g


def oracle_results(x, backward):
    ro, rl = oracle.fwd(x["q"], x["k"], x["v"], x["w"], x["beta"], x["log_f"])
    r = {"out": ro, "lse": rl}
    if backward:
        r.update(oracle.bwd(x["q"], x["k"], x["v"], x["w"], x["beta"], x["dout"], x["log_f"]))
    return r


def compare(ours, ref, mode, report):
    """ours/ref: dicts name -> array. mode: 'f32', 'bf16in_f32out' or 'bf16'."""
    errs, bad = {}, {}
    for n, r in ref.items():
        got = np64(ours[n])
        diff = np.abs(got - r)
        errs[n] = float(diff.max()) if diff.size else 0.0
        errs[n + "/max|ref|"] = errs[n] / max(float(np.abs(r).max()), 1e-30)
        if mode == "f32":
            ok = errs[n] <= 1e-4
        elif mode == "bf16in_f32out" or n in ("lse", "dbeta"):
            ok = errs[n] <= 2e-2
        elif n in STORED_BF16:
            ok = bool(np.all(diff <= 2e-2 + ulp_bf16(r)))
        elif n == "dlog_f":
            ok = errs[n] <= 2e-2 + 2.0 ** -7 * float(np.abs(r).max())
        else:
            ok = errs[n] <= 2e-2
        if not ok:
            bad[n] = errs[n]
    print(f"\n[{report} | {mode}] " + " ".join(f"{k}={v:.3g}" for k, v in errs.items()))
    assert not bad, f"{report} ({mode}): over the bar: {bad}"
    return errs


def ours_dict(out, lse, g):
    d = {"out": out, "lse": lse}
    if g:
        d.update(g)
    return d


def check(P, x, backward, modes, report):
    ref = oracle_results(x, backward)
    for mode in modes:
        od = torch.float32 if mode == "bf16in_f32out" else None
        out, lse, g = run_ours(P, x, backward, out_dtype=od)
        compare(ours_dict(out, lse, g), ref, mode, report)


def test_fp32_tiny_forward(P):
    x = si.workload_inputs("fwd_fp32_tiny")
    check(P, x, False, ["f32"], "fwd_fp32_tiny")


@pytest.mark.parametrize("L,d,fox", [(1, 16, False), (64, 16, True), (300, 32, True),
                                     (257, 64, False), (130, 128, True)])
def test_fp32_fwd_bwd_shapes(P, L, d, fox):
    x = si.make_inputs(1, 2, L, d, torch.float32, seed=1, fox=fox, clip_beta=False)
    check(P, x, True, ["f32"], f"fp32 L={L} d={d} fox={fox}")


def test_bf16_l1024_forward(P):
    x = si.workload_inputs("fwd_bf16_l1024")
    check(P, x, False, ["bf16", "bf16in_f32out"], "fwd_bf16_l1024")


@pytest.mark.parametrize("L,d,fox", [(1, 64, False), (100, 64, True), (128, 64, False),
                                     (257, 64, True), (600, 16, False), (333, 32, True),
                                     (390, 128, True)])
def test_bf16_fwd_bwd_ragged(P, L, d, fox):
    x = si.make_inputs(2, 2, L, d, torch.bfloat16, seed=2, fox=fox)
    check(P, x, True, ["bf16", "bf16in_f32out"], f"bf16 L={L} d={d} fox={fox}")


@pytest.mark.parametrize("fox", [False, True])
def test_backward_reusing_forward_workspace(P, fox):
    """A backward that reuses the forward's workspace gives the gradients of one
    that recomputes the block transforms (to summation order), and both meet the bar."""
    x = si.make_inputs(1, 3, 700, 64, torch.bfloat16, seed=4, fox=fox)
    ref = oracle_results(x, True)
    outs = []
    for reuse in (False, True):
        out, lse, g = run_ours(P, x, True, out_dtype=torch.float32, reuse=reuse)
        compare(ours_dict(out, lse, g), ref, "bf16in_f32out", f"reuse={reuse} fox={fox}")
        outs.append(g)
    # dQtil and dP_I accumulate across key tiles by fp32 reductions whose order
    # varies from run to run; the bf16-input path rounds the UT adjoint's
    # operands to TF32 (11 significant bits), where such a last-bit difference
    # can flip a rounding. So the two runs agree to that resolution, not more.
    for n in outs[0]:
        a, b = outs[0][n].float(), outs[1][n].float()
        tol = 2.0 ** -9 * float(a.abs().max()) + 1e-6
        diff = float((a - b).abs().max())
        print(f"[reuse vs recompute | {n}] max diff {diff:.3g} (bound {tol:.3g})")
        assert diff <= tol, (n, diff, tol)


def test_bf16_l1024_fwd_bwd(P):
    x = si.make_inputs(2, 4, 1024, 64, torch.bfloat16, seed=0)
    check(P, x, True, ["bf16", "bf16in_f32out"], "bf16 l1024 fwd+bwd")


def _sampled_full_size(P, name, heads, modes):
    """Full-size run on the GPU (the benchmark's launch), oracle on a few heads
    (heads are independent, so those heads' values are exact comparisons)."""
    w = si.WORKLOADS[name]
    x = si.workload_inputs(name)
    xs = si.workload_inputs(name, heads=heads)
    ref = {k: v[0] for k, v in oracle_results(xs, True).items()}
    flat = lambda t: t.reshape(w.B * w.H, *t.shape[2:])[heads]
    for mode in modes:
        od = torch.float32 if mode == "bf16in_f32out" else None
        out, lse, g = run_ours(P, x, True, out_dtype=od)
        ours = {k: flat(v) for k, v in ours_dict(out, lse, g).items()}
        compare(ours, ref, mode, f"{name} heads {heads}")
        del out, lse, g, ours
        torch.cuda.empty_cache()


def test_full_size_l4096_sampled_heads(P):
    _sampled_full_size(P, "fwdbwd_bf16_l4096", [0, 77, 191], ["bf16", "bf16in_f32out"])


def test_full_size_d128_sampled_heads(P):
    """Head dim 128 at the benchmark's shape (32 blocks per head, 96 heads), oracle on
    the first and last head."""
    _sampled_full_size(P, "fwdbwd_bf16_l4096_d128", [0, 95], ["bf16", "bf16in_f32out"])


def test_forward_is_deterministic_at_full_size(P):
    """The forward has no atomics: repeated calls on the headline workload give the same
    bits (each call starts from a NaN-filled workspace). A softmax warp pair running a
    tile ahead of another once completed the P.V barrier early, which showed up here as
    run-to-run differences in whole 32-row groups of out."""
    x = to_dev(si.workload_inputs("fwdbwd_bf16_l4096"))
    B, H, L, D = x["q"].shape
    ws = torch.empty(P.path_attn_workspace_bytes(B, H, L, D, torch.bfloat16, True),
                     dtype=torch.uint8, device="cuda")
    first = None
    for _ in range(6):
        ws.fill_(0xFF)
        out, lse = P.path_attn_fwd(x["q"], x["k"], x["v"], x["w"], x["beta"], None, workspace=ws)
        torch.cuda.synchronize()
        if first is None:
            first = (out.clone(), lse.clone())
            continue
        assert torch.equal(out, first[0]), "out differs between identical calls"
        assert torch.equal(lse, first[1]), "lse differs between identical calls"


def test_full_size_fox_l16384_sampled_heads(P):
    _sampled_full_size(P, "fox_fwdbwd_l16384", [5], ["bf16in_f32out", "bf16"])


def _decode_check(P, B, H, d, n0, cap, steps, dtype, heads, tol):
    kc, vc, seq = si.make_decode_inputs(B, H, d, n0, cap, steps, dtype, seed=3)
    kd, vd = kc.cuda(), vc.cuda()
    # cache rows past the cached ones start as NaN: each step must write its row
    # before any read of it, and rows past the last step stay untouched
    kd[..., n0:, :] = float("nan")
    vd[..., n0:, :] = float("nan")
    sel = lambda t: t.reshape(B * H, *t.shape[2:])[heads].unsqueeze(0)
    ok = sel(kc).double().numpy().copy()
    ov = sel(vc).double().numpy().copy()
    ok64, ov64 = ok.copy(), ov.copy()  # the same steps without rounding the cache
    worst = 0.0
    for t, s in enumerate(seq):
        sd = {k: v.cuda() for k, v in s.items()}
        out = P.path_decode_step(sd["q"], sd["k_new"], sd["v_new"], sd["w"], sd["beta"], kd, vd,
                                 n0 + t, out=nans(sd["q"].shape, dtype))
        assert_all_finite({"out": out}, f"decode step {t}")
        ref = oracle.decode_step(sel(s["q"]), sel(s["k_new"]), sel(s["v_new"]), sel(s["w"]),
                                 sel(s["beta"]), ok, ov, n0 + t,
                                 round_bf16=(dtype == torch.bfloat16))
        worst = max(worst, float(np.abs(np64(sel(out.cpu())) - ref).max()))
        if dtype == torch.bfloat16:
            oracle.decode_step(sel(s["q"]), sel(s["k_new"]), sel(s["v_new"]), sel(s["w"]),
                               sel(s["beta"]), ok64, ov64, n0 + t)
        if t == 0 and dtype == torch.bfloat16 and n0 > 0:
            # One update from identical caches. The GPU computes k - beta w (w.k) in
            # fp32, the oracle in fp64; both round to bf16. The fp32 result is off by
            # at most ~2^-22 of the row's magnitude, so the two agree within one ulp
            # of the entry, plus (where the update cancels most of the entry and the
            # entry becomes tiny next to its row) 2^-16 of the row's largest entry.
            k1 = np64(sel(kd.cpu())[..., :n0, :])
            r1 = ok[..., :n0, :]
            ctol = (ulp_bf16(np.maximum(np.abs(k1), np.abs(r1)))
                    + 2.0 ** -16 * np.abs(r1).max(axis=-1, keepdims=True))
            assert np.all(np.abs(k1 - r1) <= ctol), "single-step cache update beyond 1 ulp"
    torch.cuda.synchronize()
    n = n0 + steps
    kg = np64(sel(kd.cpu())[..., :n, :])
    kref = ok[..., :n, :]
    if dtype == torch.bfloat16:
        # Over many steps the two bf16 caches drift apart: each rounding flip
        # (one ulp, checked above for a single step) feeds every later update of
        # its row, and rows that the updates shrink keep the absolute difference.
        # The yardstick is the drift that bf16 rounding itself causes: the oracle's
        # bf16 cache against the same steps in fp64. Each GPU row must be within
        # twice that drift of the oracle's bf16 row, plus bf16 resolution (2^-8 of
        # the row's norm).
        rnorm = lambda a: np.sqrt(np.sum(a ** 2, axis=-1))
        diff = rnorm(kg - kref)
        drift = rnorm(kref - ok64[..., :n, :])
        bound = 2.0 * drift + 2.0 ** -8 * rnorm(kref)
        cache_bad = int(np.sum(diff > bound))
        print(f"  worst row: diff / bound = {float(np.max(diff / bound)):.3g}; median rounding "
              f"drift {float(np.median(drift / np.maximum(rnorm(kref), 1e-30))):.3g} of the row")
    else:
        cache_bad = int(np.sum(np.abs(kg - kref) > 1e-4))
    print(f"\n[decode B={B} H={H} d={d} n0={n0} steps={steps}] out max err {worst:.3g}, "
          f"cache entries beyond tolerance {cache_bad}, entries differing "
          f"{int(np.sum(kg != kref))} of {kg.size}")
    np.testing.assert_array_equal(np64(sel(vd.cpu())[..., :n, :]), ov[..., :n, :])
    assert_all_finite({"k_cache": kd[..., :n, :], "v_cache": vd[..., :n, :]}, "decode cache")
    assert bool(torch.isnan(kd[..., n:, :]).all()) and bool(torch.isnan(vd[..., n:, :]).all()), \
        "decode wrote cache rows past the last step"
    assert worst <= tol
    assert cache_bad == 0


@pytest.mark.parametrize("dtype,d", [(torch.float32, 64), (torch.bfloat16, 64),
                                     (torch.bfloat16, 128)])
def test_decode_small(P, dtype, d):
    _decode_check(P, 2, 3, d, 700, 720, 5, dtype, list(range(6)),
                  1e-4 if dtype == torch.float32 else 2e-2)


@pytest.mark.parametrize("dtype,d", [(torch.float32, 64), (torch.bfloat16, 128)])
def test_decode_multi_chunk_ragged(P, dtype, d):
    """Caches of several split chunks with a ragged last one (the chunk length is
    a power of two; 2500 rows cross two boundaries at any of them up to 1024)."""
    _decode_check(P, 1, 3, d, 2500, 2510, 4, dtype, [0, 1, 2],
                  1e-4 if dtype == torch.float32 else 2e-2)


def test_decode_from_empty_cache(P):
    _decode_check(P, 1, 2, 64, 0, 40, 30, torch.float32, [0, 1], 1e-4)


def test_decode_full_size_sampled_heads(P):
    _decode_check(P, 32, 32, 128, 16384, 16448, 64, torch.bfloat16, [0, 513, 1023], 2e-2)


def test_launch_counter_advances(P):
    before = P.lib().path_kernel_launch_count()
    x = si.make_inputs(1, 1, 200, 64, torch.bfloat16, seed=5)
    run_ours(P, x, backward=True)
    assert P.lib().path_kernel_launch_count() > before


# ---------------------------------------------------------------- prefill -> decode
def _cache_bar(got, ref, dtype):
    """fp32 caches: 1e-4. bf16 caches: 2e-2 plus one bf16 ulp of the reference, the
    stored-bf16 rule above (the keys are carried in fp16 through the forward's block
    products and stored in bf16)."""
    diff = np.abs(got - ref)
    if dtype == torch.float32:
        return bool(np.all(diff <= 1e-4)), float(diff.max())
    return bool(np.all(diff <= 2e-2 + ulp_bf16(ref))), float(diff.max())


def _prefill_check(P, x, cap, heads=None):
    dd = to_dev(x)
    dtype = dd["q"].dtype
    B, H, L, d = dd["q"].shape
    # outputs and caches start as NaN: rows 0..L-1 must be written, the rest left alone
    fox = dd["log_f"] is not None
    out, lse, kc, vc, gc = P.path_attn_prefill(
        dd["q"], dd["k"], dd["v"], dd["w"], dd["beta"], cap, dd["log_f"],
        out=nans(dd["q"].shape, dtype), lse=nans((B, H, L), torch.float32),
        k_cache=nans((B, H, cap, d), dtype), v_cache=nans((B, H, cap, d), dtype),
        g_cache=nans((B, H, cap), torch.float32) if fox else None)
    torch.cuda.synchronize()
    assert_all_finite({"out": out, "lse": lse, "k_cache": kc[..., :L, :], "v_cache": vc[..., :L, :]},
                      "prefill")
    if fox:
        assert_all_finite({"g_cache": gc[..., :L]}, "prefill")
    pick = (lambda t: t) if heads is None else (
        lambda t: t.reshape(B * H, *t.shape[2:])[heads].unsqueeze(0))
    xs = x if heads is None else {k: (None if v is None else pick(v)) for k, v in x.items()}
    rk, rv, rg = oracle.prefill_cache(xs["k"], xs["v"], xs["w"], xs["beta"], xs["log_f"],
                                      capacity=cap)
    ref = oracle_results(xs, False)
    mode = "f32" if dtype == torch.float32 else "bf16"
    compare({"out": pick(out), "lse": pick(lse)}, ref, mode, f"prefill fwd L={L} d={d}")
    ok_k, ek = _cache_bar(np64(pick(kc.cpu()))[..., :L, :], rk[..., :L, :], dtype)
    np.testing.assert_array_equal(np64(pick(vc.cpu()))[..., :L, :], rv[..., :L, :])
    eg = 0.0
    if rg is not None:
        eg = float(np.abs(np64(pick(gc.cpu()))[..., :L] - rg[..., :L]).max())
    print(f"\n[prefill cache L={L} d={d} {dtype}] k max err {ek:.3g}, g max err {eg:.3g}")
    assert ok_k, f"key cache beyond the bar (max err {ek:.3g})"
    if rg is not None:
        # g_j = c_{L-1} - c_j from prefix sums kept in fp64 and stored in fp32: two
        # fp32 roundings of |c| and one of the difference, so |err| <= 3 2^-24 max|c|
        cmax = float(np.abs(np.cumsum(np64(xs["log_f"]), axis=-1)).max())
        assert eg <= 4 * 2.0 ** -24 * cmax + 1e-12, (eg, cmax)
    # rows past L are left as the caller had them (NaN here)
    assert bool(torch.isnan(kc[..., L:, :]).all()) and bool(torch.isnan(vc[..., L:, :]).all())
    if gc is not None:
        assert bool(torch.isnan(gc[..., L:]).all())


@pytest.mark.parametrize("dtype,d,L,fox", [(torch.float32, 64, 300, False),
                                           (torch.float32, 128, 130, True),
                                           (torch.bfloat16, 64, 1, False),
                                           (torch.bfloat16, 64, 100, True),
                                           (torch.bfloat16, 64, 700, True),
                                           (torch.bfloat16, 128, 390, False)])
def test_prefill_cache_matches_oracle(P, dtype, d, L, fox):
    x = si.make_inputs(2, 2, L, d, dtype, seed=6, fox=fox,
                       clip_beta=dtype == torch.bfloat16)
    _prefill_check(P, x, L + 9)


def test_prefill_cache_full_size_sampled_heads(P):
    """The headline shape (32 key blocks, so 31 chained block products before the
    last one), oracle on sampled heads."""
    x = si.workload_inputs("fwdbwd_bf16_l4096")
    _prefill_check(P, x, 4096 + 64, heads=[0, 191])


@pytest.mark.parametrize("dtype,d,fox,L0", [(torch.float32, 64, True, 333),
                                            (torch.bfloat16, 64, True, 333),
                                            (torch.bfloat16, 128, False, 333),
                                            (torch.bfloat16, 64, True, 2100)])
def test_decode_after_prefill_continues_the_forward(P, dtype, d, fox, L0):
    """Prefill of the first L0 positions, then (gated) decode steps: the decode outputs
    are the forward rows L0.. of the whole sequence (oracle). L0 = 2100 puts the
    decode over three split chunks, the last one ragged."""
    steps = 4
    x = si.make_inputs(1, 2, L0 + steps, d, dtype, seed=7, fox=fox,
                       clip_beta=dtype == torch.bfloat16)
    ref_out, _ = oracle.fwd(x["q"], x["k"], x["v"], x["w"], x["beta"], x["log_f"])
    dd = to_dev(x)
    head = lambda t: None if t is None else t[:, :, :L0].contiguous()
    col = lambda t, i: None if t is None else t[:, :, i].contiguous()
    _, _, kc, vc, gc = P.path_attn_prefill(head(dd["q"]), head(dd["k"]), head(dd["v"]),
                                           head(dd["w"]), head(dd["beta"]), L0 + steps,
                                           head(dd["log_f"]))
    worst, ok = 0.0, True
    for t in range(L0, L0 + steps):
        o = P.path_decode_step(col(dd["q"], t), col(dd["k"], t), col(dd["v"], t),
                               col(dd["w"], t), col(dd["beta"], t), kc, vc, t,
                               log_f=col(dd["log_f"], t), g_cache=gc)
        r = ref_out[:, :, t]
        diff = np.abs(np64(o.cpu()) - r)
        worst = max(worst, float(diff.max()))
        bar = 1e-4 if dtype == torch.float32 else 2e-2 + ulp_bf16(r)
        ok = ok and bool(np.all(diff <= bar))
    torch.cuda.synchronize()
    print(f"\n[prefill + decode L0={L0} d={d} {dtype} fox={fox}] out max err {worst:.3g}")
    assert ok


def test_hand_worked_example(P):
    """The hand-derived example of tests/golden (d = 2, zero-padded to the kernels' head
    dims: zero columns leave every logit and the first two output columns unchanged),
    forward and prefill cache against the hand values themselves."""
    import json
    import os

    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                           "hand_worked_d2_l3.json")) as f:
        g = json.load(f)

    def pad(key, d):
        a = torch.tensor(g[key], dtype=torch.float32)
        return torch.nn.functional.pad(a, (0, d - a.shape[-1]))[None, None].contiguous().cuda()

    beta = torch.tensor(g["beta"], dtype=torch.float32)[None, None].cuda()
    lf = torch.tensor(g["log_f"], dtype=torch.float32)[None, None].cuda()
    vv = np.array(g["v"], dtype=np.float64)
    for gated in (False, True):
        z = np.array([[-np.inf if x is None else x for x in r]
                      for r in g["logits_gated" if gated else "logits"]])
        p = np.exp(z - z.max(axis=1, keepdims=True))
        ro = (p / p.sum(axis=1, keepdims=True)) @ vv
        for d in (16, 64):
            q, k, v, w = (pad(n, d) for n in ("q", "k", "v", "w"))
            log_f = lf if gated else None
            if d == 64:
                out, _, kc, vc, gc = P.path_attn_prefill(q, k, v, w, beta, 3, log_f,
                                                         scale=g["scale"])
                torch.cuda.synchronize()
                np.testing.assert_allclose(np64(kc.cpu())[0, 0, :, :2], g["k_cache"], atol=1e-5)
                assert not kc[..., 2:].any()
                if gated:
                    np.testing.assert_allclose(np64(gc.cpu())[0, 0], g["g_cache"], atol=1e-5)
            else:
                out, _ = P.path_attn_fwd(q, k, v, w, beta, log_f, scale=g["scale"])
                torch.cuda.synchronize()
            np.testing.assert_allclose(np64(out.cpu())[0, 0, :, :2], ro, atol=1e-5)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("scale", [-0.125, 0.0])
def test_forward_with_non_positive_scale(P, d, scale):
    """Without the gate and with a positive scale the tensor-core softmax keeps the
    logits unscaled and scales the row max instead; a zero or negative scale takes the
    per-element path. Both against the oracle at the same scale."""
    x = si.make_inputs(1, 2, 300, d, torch.bfloat16, seed=13)
    dd = to_dev(x)
    out, lse = P.path_attn_fwd(dd["q"], dd["k"], dd["v"], dd["w"], dd["beta"], None, scale=scale,
                               out_dtype=torch.float32)
    torch.cuda.synchronize()
    ro, rl = oracle.fwd(x["q"], x["k"], x["v"], x["w"], x["beta"], None, scale=scale)
    compare({"out": out, "lse": lse}, {"out": ro, "lse": rl}, "bf16in_f32out",
            f"scale={scale} d={d}")


# ---------------------------------------------------------------- degenerate cases
@pytest.mark.parametrize("dtype,d,L", [(torch.float32, 64, 300), (torch.bfloat16, 64, 333),
                                       (torch.bfloat16, 128, 200)])
def test_beta_zero_is_causal_softmax_attention(P, dtype, d, L):
    """beta = 0 makes every H the identity, so the kernels must compute causal softmax
    attention: out, dq, dk, dv against torch's SDPA and its autograd (fp64 on the CPU,
    a library routine rather than the oracle); dw is zero (H does not depend on w);
    dbeta against the oracle."""
    x = si.make_inputs(1, 2, L, d, dtype, seed=8, clip_beta=dtype == torch.bfloat16)
    x["beta"] = torch.zeros_like(x["beta"])
    q, k, v = (x[n].double().requires_grad_() for n in ("q", "k", "v"))
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True)
    ref.backward(x["dout"].double())
    od = torch.float32 if dtype == torch.bfloat16 else None
    out, lse, g = run_ours(P, x, True, out_dtype=od)
    rb = oracle.bwd(x["q"], x["k"], x["v"], x["w"], x["beta"], x["dout"], None)
    mode = "f32" if dtype == torch.float32 else "bf16in_f32out"
    compare({"out": out, "dq": g["dq"], "dk": g["dk"], "dv": g["dv"], "dbeta": g["dbeta"]},
            {"out": ref.detach().numpy(), "dq": q.grad.numpy(), "dk": k.grad.numpy(),
             "dv": v.grad.numpy(), "dbeta": rb["dbeta"]}, mode, f"beta=0 d={d} L={L}")
    assert float(g["dw"].abs().max()) <= 1e-6


def test_reflections_beta_two_fp32(P):
    """beta = 2 with unit w: every H is a reflection (orthogonal), so the transported keys
    keep their norms over the whole sequence and nothing decays: dw reaches |15| here. The
    bar is the absolute 1e-4 of every fp32 case (plain fp32 arithmetic of the key-cache
    recurrence stays near 8e-6 on this input)."""
    x = si.make_inputs(1, 2, 257, 64, torch.float32, seed=9, clip_beta=False)
    x["beta"] = torch.full_like(x["beta"], 2.0)
    ref = oracle_results(x, True)
    out, lse, g = run_ours(P, x, True)
    compare(ours_dict(out, lse, g), ref, "f32", "beta=2 reflections")


@pytest.mark.parametrize("dtype,mode", [(torch.float32, "f32"),
                                        (torch.bfloat16, "bf16in_f32out")])
def test_repeated_w_projector(P, dtype, mode):
    """One w at every position with beta = 1: H is (nearly) the same projector throughout
    and I + strictLower(D W W^T) is all ones below the diagonal."""
    x = si.make_inputs(1, 2, 300, 64, dtype, seed=10, clip_beta=dtype == torch.bfloat16)
    x["w"] = x["w"][:, :, :1].expand_as(x["w"]).contiguous()
    x["beta"] = torch.ones_like(x["beta"])
    check(P, x, True, [mode], f"repeated w {dtype}")
