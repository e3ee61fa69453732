"""The Python binding's argument checks (no GPU needed). The C library reads and
writes every buffer by the sizes it is given, so the binding must reject a tensor
whose shape or dtype disagrees with them before anything is launched; these
checks run before the device check, so CPU tensors exercise them."""
import pytest
import torch

import softmax_attention_block_b200 as P

B, H, L, D = 1, 2, 40, 64


def attn_inputs(dtype=torch.bfloat16, fox=False):
    t = lambda *s, dt=dtype: torch.zeros(*s, dtype=dt)
    return dict(q=t(B, H, L, D), k=t(B, H, L, D), v=t(B, H, L, D), w=t(B, H, L, D),
                beta=t(B, H, L, dt=torch.float32),
                log_f=t(B, H, L, dt=torch.float32) if fox else None)


def fwd(**over):
    x = attn_inputs()
    x.update(over)
    return P.path_attn_fwd(x["q"], x["k"], x["v"], x["w"], x["beta"], x["log_f"])


@pytest.mark.parametrize("name,bad,msg", [
    ("k", torch.zeros(B, H, L + 1, D, dtype=torch.bfloat16), "k: shape"),
    ("v", torch.zeros(B, H, L, D, dtype=torch.float32), "v: dtype"),
    ("w", torch.zeros(B, H, L, 32, dtype=torch.bfloat16), "w: shape"),
    ("beta", torch.zeros(B, H, L, dtype=torch.bfloat16), "beta: dtype"),
    ("beta", torch.zeros(B, H, L - 1), "beta: shape"),
    ("log_f", torch.zeros(B, H, 2 * L), "log_f: shape"),
    ("q", torch.zeros(B, H, L, D, dtype=torch.float16), "q: dtype"),
])
def test_forward_rejects_mismatched_inputs(name, bad, msg):
    with pytest.raises(ValueError, match=msg):
        fwd(**{name: bad})


def test_forward_reaches_the_device_check_when_consistent():
    with pytest.raises(ValueError, match="CUDA tensors"):
        fwd()
    with pytest.raises(ValueError, match="out: shape"):
        x = attn_inputs()
        P.path_attn_fwd(x["q"], x["k"], x["v"], x["w"], x["beta"],
                        out=torch.zeros(B, H, L, D + 1, dtype=torch.bfloat16))


def test_backward_checks_outputs_and_gradients():
    x = attn_inputs(fox=True)
    out = torch.zeros(B, H, L, D, dtype=torch.bfloat16)
    lse = torch.zeros(B, H, L)
    args = (x["q"], x["k"], x["v"], x["w"], x["beta"], out, lse)
    with pytest.raises(ValueError, match="dout"):
        P.path_attn_bwd(*args, torch.zeros(B, H, L, D), x["log_f"])
    with pytest.raises(ValueError, match="lse: shape"):
        P.path_attn_bwd(*args[:-1], torch.zeros(B, H, L + 1), out, x["log_f"])
    grads = {n: torch.zeros(B, H, L, D, dtype=torch.bfloat16) for n in ("dq", "dk", "dv", "dw")}
    grads["dbeta"] = torch.zeros(B, H, L)
    with pytest.raises(ValueError, match="dlog_f"):
        P.path_attn_bwd(*args, out.clone(), x["log_f"], grads=grads)
    grads["dlog_f"] = torch.zeros(B, H, L)
    grads["dw"] = torch.zeros(B, H, L, D)
    with pytest.raises(ValueError, match="dw: dtype"):
        P.path_attn_bwd(*args, out.clone(), x["log_f"], grads=grads)


def test_decode_checks_step_tensors_and_caches():
    cap = 50
    kc = torch.zeros(B, H, cap, D, dtype=torch.bfloat16)
    vc = torch.zeros_like(kc)
    s = {n: torch.zeros(B, H, D, dtype=torch.bfloat16) for n in ("q", "k_new", "v_new", "w")}
    beta = torch.zeros(B, H)

    def dec(**over):
        a = dict(s, beta=beta, k_cache=kc, v_cache=vc, log_f=None, g_cache=None)
        a.update(over)
        return P.path_decode_step(a["q"], a["k_new"], a["v_new"], a["w"], a["beta"],
                                  a["k_cache"], a["v_cache"], 10, log_f=a["log_f"],
                                  g_cache=a["g_cache"])

    with pytest.raises(ValueError, match="q: shape"):
        dec(q=torch.zeros(B, H, D + 8, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="v_cache: shape"):
        dec(v_cache=torch.zeros(B, H, cap - 1, D, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="beta: shape"):
        dec(beta=torch.zeros(B, H + 1))
    with pytest.raises(ValueError, match="go together"):
        dec(g_cache=torch.zeros(B, H, cap))
    with pytest.raises(ValueError, match="g_cache: shape"):
        dec(log_f=torch.zeros(B, H), g_cache=torch.zeros(B, H, cap + 1))
    with pytest.raises(ValueError, match="CUDA tensors"):
        dec(log_f=torch.zeros(B, H), g_cache=torch.zeros(B, H, cap))


def test_prefill_checks_caches():
    x = attn_inputs(fox=True)
    args = (x["q"], x["k"], x["v"], x["w"], x["beta"], 64, x["log_f"])
    with pytest.raises(ValueError, match="k_cache: shape"):
        P.path_attn_prefill(*args, k_cache=torch.zeros(B, H, 63, D, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="v_cache: dtype"):
        P.path_attn_prefill(*args, v_cache=torch.zeros(B, H, 64, D))
    with pytest.raises(ValueError, match="g_cache: shape"):
        P.path_attn_prefill(*args, g_cache=torch.zeros(B, H, 65))
    with pytest.raises(ValueError, match="CUDA tensors"):
        P.path_attn_prefill(*args)


def test_wrappers_of_the_remaining_entry_points():
    cap = 50
    kc = torch.zeros(B, H, cap, D, dtype=torch.bfloat16)
    vc = torch.zeros_like(kc)
    s = [torch.zeros(B, H, D, dtype=torch.bfloat16) for _ in range(4)]
    beta = torch.zeros(B, H)
    with pytest.raises(ValueError, match="needs log_f and g_cache"):
        P.path_decode_step_gated(*s, beta, None, kc, vc, None, 10)
    with pytest.raises(ValueError, match="g_cache: dtype"):
        P.path_decode_step_gated(*s, beta, torch.zeros(B, H), kc, vc,
                                 torch.zeros(B, H, cap, dtype=torch.float64), 10)
    with pytest.raises(ValueError, match="w: shape"):
        P.path_decode_step_noalloc(*s[:3], torch.zeros(B, H, 2 * D, dtype=torch.bfloat16), beta,
                                   kc, vc, 10)
    with pytest.raises(ValueError, match="CUDA tensors"):
        P.path_decode_step_noalloc(*s, beta, kc, vc, 10)
    with pytest.raises(ValueError, match="CUDA tensors"):
        P.path_attn_wait_status(torch.zeros(64, dtype=torch.uint8))
    assert P.path_kernel_launch_count() >= 0
    prev = P.path_profile_enable(True)
    assert P.path_profile_enable(prev) is True
    assert P.path_profile_read() == {}


class _OnDevice:
    """Stands in for a contiguous CUDA tensor on device `index` (no GPU needed)."""
    is_cuda = True

    def __init__(self, index):
        self.device = torch.device("cuda", index)

    def is_contiguous(self):
        return True


def test_tensors_must_be_on_the_current_device(monkeypatch):
    """The library launches on the current device: tensors elsewhere are refused."""
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 1)
    with pytest.raises(ValueError, match="current CUDA device"):
        P._check_dev(_OnDevice(0), _OnDevice(0))
    with pytest.raises(ValueError, match="one device"):
        P._check_dev(_OnDevice(1), _OnDevice(0))
    P._check_dev(_OnDevice(1), None, _OnDevice(1))
