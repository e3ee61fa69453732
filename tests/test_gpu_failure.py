"""Failure detection on the GPU without a fault: a bounded wait that runs out.

The library's test hook (path_test_withhold_kv_load) makes the tensor-core
forward's last query tile never receive one key/value block, and shortens
every wait of that kernel to 2 ms. The waiting warps then give up instead of
hanging: the tile's rows come back as NaN, path_attn_wait_status reports
PATH_ERR_TIMEOUT, every other tile is correct, and the next call on the same
CUDA context computes normally.
"""
import pytest
import torch

import oracle
import synthetic_inputs as si

from test_gpu_parity import check, compare, to_dev

pytestmark = pytest.mark.gpu

PATH_ERR_TIMEOUT = 5


@pytest.fixture(scope="module")
def P():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import softmax_attention_block_b200 as P

    P.lib()
    return P


@pytest.mark.parametrize("d", [64, 128])
def test_forward_wait_gives_up_reports_and_recovers(P, d):
    x = si.make_inputs(1, 2, 300, d, torch.bfloat16, seed=11)  # 3 query tiles
    dd = to_dev(x)
    B, H, L, D = dd["q"].shape
    ws = torch.full((P.path_attn_workspace_bytes(B, H, L, D, torch.bfloat16, True),), 0xFF,
                    dtype=torch.uint8, device="cuda")
    P.path_test_withhold_kv_load(True)
    try:
        out, lse = P.path_attn_fwd(dd["q"], dd["k"], dd["v"], dd["w"], dd["beta"], None,
                                   out_dtype=torch.float32, workspace=ws)
        torch.cuda.synchronize()
        status = P.lib().path_attn_wait_status(ws.data_ptr(), None)
    finally:
        P.path_test_withhold_kv_load(False)
    assert status == PATH_ERR_TIMEOUT
    last = slice(256, L)  # the last query tile could not finish: NaN, not stale values
    assert bool(torch.isnan(out[:, :, last]).all()) and bool(torch.isnan(lse[:, :, last]).all())
    # the other tiles completed and are correct
    ro, rl = oracle.fwd(x["q"], x["k"], x["v"], x["w"], x["beta"], None)
    compare({"out": out[:, :, :256], "lse": lse[:, :, :256]},
            {"out": ro[:, :, :256], "lse": rl[:, :, :256]}, "bf16in_f32out",
            f"tiles before the one that gave up, d={d}")
    # the context is still usable: the same forward and a backward pass parity
    check(P, x, True, ["bf16in_f32out"], f"after a wait gave up, d={d}")


PATH_ERR_WORKSPACE = 3


@pytest.mark.parametrize("d", [64, 128])
def test_reuse_after_a_forward_that_saved_nothing(P, d):
    """At bf16, head dims 64 and 128, a reusing backward reads per-block quantities that the
    forward leaves only when its workspace_bytes covers the backward size. A forward
    told less (C ABI, on the same backward-sized buffer) leaves none: the backward then
    writes no gradient and reports PATH_ERR_WORKSPACE, and the next forward given the
    whole buffer makes a reusing backward correct again."""
    x = si.make_inputs(1, 2, 200, d, torch.bfloat16, seed=12)
    dd = to_dev(x)
    B, H, L, D = dd["q"].shape
    nb_bwd = P.path_attn_workspace_bytes(B, H, L, D, torch.bfloat16, True)
    nb_fwd = P.path_attn_workspace_bytes(B, H, L, D, torch.bfloat16, False)
    assert nb_fwd < nb_bwd
    ws = torch.full((nb_bwd,), 0xFF, dtype=torch.uint8, device="cuda")
    out = torch.empty_like(dd["q"])
    lse = torch.empty((B, H, L), dtype=torch.float32, device="cuda")
    ptr = lambda t: t.data_ptr()
    st = P.lib().path_attn_fwd(ptr(dd["q"]), ptr(dd["k"]), ptr(dd["v"]), ptr(dd["w"]),
                               ptr(dd["beta"]), None, D ** -0.5, B, H, L, D, 1, ptr(out),
                               ptr(lse), ptr(ws), nb_fwd, None)
    assert st == 0
    grads = {n: torch.full_like(dd["q"], float("nan")) for n in ("dq", "dk", "dv", "dw")}
    grads["dbeta"] = torch.full_like(dd["beta"], float("nan"))
    P.path_attn_bwd(dd["q"], dd["k"], dd["v"], dd["w"], dd["beta"], out, lse, dd["dout"], None,
                    grads=grads, workspace=ws, reuse_fwd_workspace=True)
    torch.cuda.synchronize()
    assert P.lib().path_attn_wait_status(ws.data_ptr(), None) == PATH_ERR_WORKSPACE
    for n in ("dq", "dk", "dw", "dbeta"):
        assert bool(torch.isnan(grads[n]).all()), n  # nothing written
    # the binding gives the forward the whole buffer: the reusing backward is right
    out, lse = P.path_attn_fwd(dd["q"], dd["k"], dd["v"], dd["w"], dd["beta"], None, workspace=ws)
    g = P.path_attn_bwd(dd["q"], dd["k"], dd["v"], dd["w"], dd["beta"], out, lse, dd["dout"], None,
                        workspace=ws, reuse_fwd_workspace=True)
    torch.cuda.synchronize()
    assert P.lib().path_attn_wait_status(ws.data_ptr(), None) == 0
    ref = oracle.bwd(x["q"], x["k"], x["v"], x["w"], x["beta"], x["dout"], None)
    ro, rl = oracle.fwd(x["q"], x["k"], x["v"], x["w"], x["beta"], None)
    ref.update(out=ro, lse=rl)
    got = {"out": out, "lse": lse, **g}
    compare({n: got[n] for n in ref}, ref, "bf16", "reusing backward after a saving forward")
