"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function the header declares, sizes workspaces, and rejects invalid
arguments with the documented status before launching anything."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "path_attn.h")

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3
F32, BF16 = 0, 1


@pytest.fixture(scope="module")
def lib():
    import softmax_attention_block_b200 as P

    if not os.path.exists(P.LIB_PATH):
        from softmax_attention_block_b200 import build

        build.build()
    return P.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(path_[a-z_]+)\s*\(", text)))


def test_header_symbols_exported(lib):
    names = declared_functions()
    assert "path_attn_fwd" in names and "path_decode_step" in names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in the header but not exported"


def test_status_strings(lib):
    for s in range(6):
        assert lib.path_status_string(s)
    assert lib.path_status_string(99) == b"unknown status"


def test_workspace_sizes(lib):
    f = lib.path_attn_workspace_bytes
    assert f(1, 1, 64, 16, F32, 0) > 0
    assert f(8, 24, 4096, 64, BF16, 1) > f(8, 24, 4096, 64, BF16, 0) > 0
    assert f(1, 1, 64, 48, BF16, 0) == 0  # unsupported head dim
    assert f(0, 1, 64, 64, BF16, 0) == 0
    assert f(1, 1, 0, 64, BF16, 0) == 0
    assert f(1, 1, 64, 64, 7, 0) == 0
    assert lib.path_decode_workspace_bytes(32, 32, 16448, 128, BF16) > 0
    assert lib.path_decode_workspace_bytes(1, 1, 10, 96, BF16) == 0
    assert f(1, 1, 64, 64, BF16, 0) % 256 == 0


FAKE = 0x1000  # never dereferenced: every call below fails validation first


def fwd(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, w=FAKE, beta=FAKE, log_f=None, scale=0.125, B=1, H=1,
             L=64, d=64, dt=BF16, out=FAKE, lse=FAKE, ws=FAKE, wsb=1 << 40)
    a.update(kw)
    return lib.path_attn_fwd(a["q"], a["k"], a["v"], a["w"], a["beta"], a["log_f"], a["scale"],
                             a["B"], a["H"], a["L"], a["d"], a["dt"], a["out"], a["lse"], a["ws"],
                             a["wsb"], None)


def _ws_formula(nh, L, d, bwd):
    """path_attn_workspace_bytes at bf16, restated from the header's size formula."""
    nblk = -(-L // 128)
    Lp, npairs = 128 * nblk, nblk * (nblk - 1) // 2
    khat = nh * npairs * 128 * d * 2
    lin = nh * (Lp * (1044 + 12 * d) + L * 4 * d) if bwd else nh * (Lp * (516 + 4 * d) + L * 2 * d)
    prods = nh * nblk * d * d * (6 if bwd else 2)
    scratch = 0
    if d in (64, 128):  # the UT quantities the forward leaves for the adjoint
        scratch = nh * nblk * (98304 if d == 64 else 245760) if bwd else 0
    else:
        scratch = nh * nblk * ((14 * 128 * 128 + 3 * 128 * d) if bwd else (7 * 128 * 128 + 128 * d)) * 4
    return khat + lin + prods + scratch


@pytest.mark.parametrize("nh,L,d", [(24, 4096, 64), (3, 300, 64), (24, 65536, 64), (12, 4096, 128),
                                    (5, 700, 32)])
def test_workspace_follows_the_stated_formula(lib, nh, L, d):
    for bwd in (0, 1):
        got = lib.path_attn_workspace_bytes(1, nh, L, d, BF16, bwd)
        ref = _ws_formula(nh, L, d, bwd)
        # within the 256-byte rounding of each of the (at most 24) buffers
        assert ref <= got <= ref + 24 * 256, (nh, L, d, bwd, got, ref)
    if (nh, L) == (24, 65536):
        assert 52.9e9 < lib.path_attn_workspace_bytes(1, 24, 65536, 64, BF16, 0) < 53.1e9


def test_fwd_rejects_bad_arguments(lib):
    assert fwd(lib, q=None) == INVALID
    assert fwd(lib, lse=None) == INVALID
    assert fwd(lib, L=0) == INVALID
    assert fwd(lib, B=-1) == INVALID
    assert fwd(lib, scale=float("nan")) == INVALID
    assert fwd(lib, d=48) == UNSUPPORTED
    assert fwd(lib, dt=5) == UNSUPPORTED
    assert fwd(lib, ws=None) == WORKSPACE
    assert fwd(lib, wsb=100) == WORKSPACE


def test_fwd_rejects_unaligned_tma_inputs(lib):
    # bf16 at head dims 64 and 128 loads q, k, w by TMA: 16-byte aligned bases only
    assert fwd(lib, q=FAKE + 2) == INVALID
    assert fwd(lib, w=FAKE + 8) == INVALID
    assert fwd(lib, k=FAKE + 4, d=128) == INVALID
    # other head dims have no such rule: validation goes on to the (missing) workspace
    assert fwd(lib, k=FAKE + 2, d=32, ws=None) == WORKSPACE


def test_withhold_hook_arguments(lib):
    assert lib.path_test_withhold_kv_load(2) == INVALID
    assert lib.path_test_withhold_kv_load(-1) == INVALID
    assert lib.path_test_withhold_kv_load(0) == 0


def test_grid_limits_unsupported(lib):
    # heads and 128-row blocks index launch grid dimensions (at most 65535)
    assert fwd(lib, B=256, H=256) == UNSUPPORTED
    assert fwd(lib, L=65536 * 128 + 1, d=16) == UNSUPPORTED
    f = lib.path_attn_workspace_bytes
    assert f(256, 256, 64, 64, BF16, 1) == 0
    assert f(1, 1, 65536 * 128 + 1, 16, BF16, 0) == 0
    assert f(255, 257, 64, 64, BF16, 1) > 0  # 65535 heads
    assert lib.path_decode_workspace_bytes(256, 256, 100, 128, BF16) == 0
    st = lib.path_decode_step(FAKE, FAKE, FAKE, FAKE, FAKE, 0.1, 256, 256, 128, 10, 11, BF16,
                              FAKE, FAKE, FAKE, FAKE, 1 << 40, None)
    assert st == UNSUPPORTED


def test_bwd_rejects_bad_arguments(lib):
    def bwd(**kw):
        a = dict(log_f=None, dlog_f=None, dq=FAKE, L=64, d=64, wsb=1 << 40)
        a.update(kw)
        return lib.path_attn_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, a["log_f"], 0.125, 1, 1, a["L"],
                                 a["d"], BF16, FAKE, FAKE, FAKE, a["dq"], FAKE, FAKE, FAKE, FAKE,
                                 a["dlog_f"], a.get("flags", 0), FAKE, a["wsb"], None)

    assert bwd(dq=None) == INVALID
    assert bwd(log_f=FAKE) == INVALID  # dlog_f must be given with log_f
    assert bwd(dlog_f=FAKE) == INVALID
    assert bwd(d=24) == UNSUPPORTED
    assert bwd(flags=2) == INVALID  # unknown flag bits
    assert bwd(wsb=10) == WORKSPACE


def test_decode_rejects_bad_arguments(lib):
    def dec(**kw):
        a = dict(q=FAKE, n=10, cap=11, d=128, wsb=1 << 40, kc=FAKE)
        a.update(kw)
        return lib.path_decode_step(a["q"], FAKE, FAKE, FAKE, FAKE, 0.1, 2, 2, a["d"], a["n"],
                                    a["cap"], BF16, a["kc"], FAKE, FAKE, FAKE, a["wsb"], None)

    assert dec(n=11) == INVALID           # n_cached + 1 > capacity
    assert dec(n=-1) == INVALID
    assert dec(q=None) == INVALID
    assert dec(kc=FAKE + 8) == INVALID     # caches must be 16-byte aligned
    assert dec(d=32) == UNSUPPORTED
    assert dec(wsb=4) == WORKSPACE


def test_profile_toggle(lib):
    prev = lib.path_profile_enable(1)
    assert lib.path_profile_enable(prev) == 1


def test_gated_decode_rejects_bad_arguments(lib):
    def dec(**kw):
        a = dict(log_f=FAKE, g=FAKE, n=10, cap=11, d=128, wsb=1 << 40)
        a.update(kw)
        return lib.path_decode_step_gated(FAKE, FAKE, FAKE, FAKE, FAKE, a["log_f"], 0.1, 2, 2,
                                          a["d"], a["n"], a["cap"], BF16, FAKE, FAKE, a["g"],
                                          FAKE, FAKE, a["wsb"], None)

    assert dec(log_f=None) == INVALID
    assert dec(g=None) == INVALID
    assert dec(n=11) == INVALID
    assert dec(d=16) == UNSUPPORTED
    assert dec(wsb=4) == WORKSPACE


def test_prefill_rejects_bad_arguments(lib):
    def pre(**kw):
        a = dict(q=FAKE, v=FAKE, log_f=None, g=None, L=64, d=64, cap=64, kc=FAKE, ws=FAKE,
                 wsb=1 << 40)
        a.update(kw)
        return lib.path_attn_prefill(a["q"], FAKE, a["v"], FAKE, FAKE, a["log_f"], 0.125, 1, 1,
                                     a["L"], a["d"], BF16, FAKE, FAKE, a["kc"], FAKE, a["g"],
                                     a["cap"], a["ws"], a["wsb"], None)

    assert pre(q=None) == INVALID
    assert pre(kc=None) == INVALID
    assert pre(log_f=FAKE) == INVALID       # g_cache must come with log_f
    assert pre(g=FAKE) == INVALID
    assert pre(cap=63) == INVALID           # L > capacity
    assert pre(kc=FAKE + 8) == INVALID      # caches must be 16-byte aligned
    assert pre(v=FAKE + 4) == INVALID
    assert pre(d=32) == UNSUPPORTED         # decode head dims only
    assert pre(ws=None) == WORKSPACE
    assert pre(wsb=100) == WORKSPACE


def test_header_is_c99_and_links(lib, tmp_path):
    """The header is a C header: a C99 translation unit that takes the address of every
    declared entry point compiles warning-free and links against the library."""
    import subprocess

    import softmax_attention_block_b200 as P

    names = declared_functions()
    src = tmp_path / "use_header.c"
    src.write_text(
        '#include "path_attn.h"\n#include <stdio.h>\n'
        "typedef void (*any_fn)(void);\n"
        "int main(void) {\n    any_fn fns[] = {\n"
        + "".join(f"        (any_fn)&{n},\n" for n in names)
        + "    };\n    size_t n = sizeof fns / sizeof fns[0];\n"
        '    printf("%zu %s\\n", n, path_status_string(PATH_OK));\n    return 0;\n}\n')
    exe = tmp_path / "use_header"
    libdir = os.path.dirname(P.LIB_PATH)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
           "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
           "-L", libdir, "-l:libpath_attn.so", "-Wl,--allow-shlib-undefined",
           f"-Wl,-rpath,{libdir}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
