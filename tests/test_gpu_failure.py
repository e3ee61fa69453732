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
