"""The allocation-free decode entry point against the regular one.

path_decode_step_noalloc serves callers that cannot call cudaMalloc (their
device memory belongs to another allocator, or an allocation's latency or
failure is unacceptable mid-decode). It keeps its chunk partials in a fixed
device array inside the library instead of a caller workspace. This test
calls it through the C ABI and checks, on two consecutive decode steps, that
it produces the same outputs as path_decode_step (within the decode tests'
tolerances: 2e-2 for bf16, 1e-4 for fp32) and bit-identical updated caches, for
every chunk size the fixed array leads it to and for both element types. The file is named to
be collected last, so a failure here does not hide any other test.
"""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu

PATH_BF16 = 1


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import softmax_attention_block_b200 as P

    L = P.lib()
    vp, fp, i, f = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    L.path_decode_step_noalloc.argtypes = [vp, vp, vp, vp, fp, f, i, i, i, i, i, i, vp, vp, vp, vp]
    L.path_decode_step_noalloc.restype = i
    return L


# Rows per chunk grow (256, 1024, 4096, 16384) until B*H*ceil(n/chunk)*(d+2) partials fit
# in the 2^20-float array; the cases cover each size and both element types.
@pytest.mark.parametrize("B,H,d,n0,dtype", [
    (2, 3, 64, 700, torch.bfloat16),       # 256-row chunks
    (2, 3, 64, 700, torch.float32),        # 256-row chunks, fp32 caches
    (8, 16, 128, 20000, torch.bfloat16),   # 1024-row chunks
    (32, 32, 128, 16384, torch.bfloat16),  # 4096-row chunks
    (64, 128, 64, 4097, torch.bfloat16),   # 16384-row chunks
])
def test_noalloc_matches_workspace_decode(lib, B, H, d, n0, dtype):
    import softmax_attention_block_b200 as P

    g = torch.Generator(device="cuda").manual_seed(7)
    cap = n0 + 2
    kc = torch.randn((B, H, cap, d), device="cuda", generator=g).to(dtype)
    vc = torch.randn((B, H, cap, d), device="cuda", generator=g).to(dtype)
    k_ref, v_ref = kc.clone(), vc.clone()
    mode = PATH_BF16 if dtype == torch.bfloat16 else 0
    tol = 2e-2 if dtype == torch.bfloat16 else 1e-4
    for step in range(2):
        q, kn, vn, w = (torch.randn((B, H, d), device="cuda", generator=g).to(dtype)
                        for _ in range(4))
        w = (w.float() / w.float().norm(dim=-1, keepdim=True)).to(dtype)
        beta = (2 * torch.sigmoid(torch.randn((B, H), device="cuda", generator=g))).clamp(0, 1.99)
        n = n0 + step
        out_ref = P.path_decode_step(q, kn, vn, w, beta, k_ref, v_ref, n)
        out = torch.empty_like(out_ref)
        st = lib.path_decode_step_noalloc(
            q.data_ptr(), kn.data_ptr(), vn.data_ptr(), w.data_ptr(), beta.data_ptr(),
            d ** -0.5, B, H, d, n, cap, mode, kc.data_ptr(), vc.data_ptr(), out.data_ptr(),
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == 0, P.path_status_string(st)
        torch.cuda.synchronize()
        err = (out.float() - out_ref.float()).abs().max().item()
        assert err <= tol, f"step {step}: outputs differ by {err}"
        assert torch.equal(kc[:, :, : n + 1], k_ref[:, :, : n + 1]), f"step {step}: key caches differ"
        assert torch.equal(vc[:, :, : n + 1], v_ref[:, :, : n + 1])


def test_noalloc_rejects_sizes_beyond_its_scratch(lib):
    # B*H*ceil(n/16384)*(d+2) > 2^20 floats: refused before any launch
    st = lib.path_decode_step_noalloc(16, 16, 16, 16, 16, 0.1, 64, 128, 128, 20000, 20001,
                                      PATH_BF16, 16, 16, 16, None)
    assert st == 3  # PATH_ERR_WORKSPACE
