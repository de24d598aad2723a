"""C-ABI checks that need no GPU: the library loads, exports every entry point
the header declares, and rejects bad arguments before touching CUDA."""
import ctypes
import os
import re

import pytest

from long_context_bidirectional_b200 import build as B

HEADER = os.path.join(B.ROOT, "include", "b200attn.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    import long_context_bidirectional_b200 as m
    return m.lib


def declared_functions():
    text = open(HEADER).read()
    names = re.findall(r"B2A_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)
    assert len(names) >= 11
    return names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert isinstance(getattr(lib, name), ctypes._CFuncPtr)


def test_debug_build_exports_the_same_entry_points():
    path = B.build(debug=True)
    dbg = ctypes.CDLL(path)
    for name in declared_functions():
        assert hasattr(dbg, name), name
    dbg.b2a_debug_build.restype = ctypes.c_int
    assert dbg.b2a_debug_build() == 1


def test_version_and_status_strings(lib):
    assert lib.b2a_version() == 104
    assert lib.b2a_debug_build() == 0
    assert lib.b2a_status_string(0) == b"ok"
    assert lib.b2a_status_string(1) == b"invalid argument"
    assert lib.b2a_status_string(4) == b"device-side wait timed out"
    assert lib.b2a_status_string(5) == b"device-side bounds check failed (debug build)"
    assert lib.b2a_status_string(99) == b"unknown status"


FAKE = 0x10000  # aligned, never dereferenced: validation rejects first


def _attn(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, out=FAKE, lse=None, S=256, H=2, d=64, scale=0.125,
             ld_q=128, ld_k=128, ld_v=128, ld_o=128)
    a.update(kw)
    return lib.attn_fwd(a["q"], a["k"], a["v"], a["out"], a["lse"], a["S"], a["H"], a["d"],
                        a["scale"], a["ld_q"], a["ld_k"], a["ld_v"], a["ld_o"], None)


@pytest.mark.parametrize("kw", [
    dict(q=None), dict(k=None), dict(out=None), dict(q=FAKE + 2), dict(out=FAKE + 8),
    dict(lse=FAKE + 2), dict(S=0), dict(S=-5), dict(H=0), dict(d=96), dict(d=256),
    dict(scale=0.0), dict(scale=-1.0), dict(scale=float("inf")), dict(scale=float("nan")),
    dict(ld_q=127), dict(ld_q=120), dict(ld_k=64), dict(ld_o=100),
])
def test_attn_fwd_rejects(lib, kw):
    assert _attn(lib, **kw) == 1


def test_attn_fwd_valid_args_reach_the_device_check(lib):
    # Valid arguments get past validation; without a usable sm_100 device the
    # call must fail with a CUDA or unsupported status, never crash.
    import torch
    st = _attn(lib)
    if not torch.cuda.is_available():
        assert st in (2, 3)


def test_partial_and_merge_reject(lib):
    p = lib.attn_fwd_partial
    assert p(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 4, 2, 64, 0.1, 128, 128, None) == 1   # Sq = 0
    assert p(FAKE, FAKE, FAKE, FAKE, FAKE, 4, -1, 2, 64, 0.1, 128, 128, None) == 1  # Skv < 0
    assert p(FAKE, FAKE, FAKE, None, FAKE, 4, 4, 2, 64, 0.1, 128, 128, None) == 1   # o_part
    assert p(FAKE, FAKE, FAKE, FAKE + 4, FAKE, 4, 4, 2, 64, 0.1, 128, 128, None) == 1
    m = lib.attn_merge
    assert m(FAKE, FAKE, 0, FAKE, None, 16, 2, 64, None) == 1     # P = 0
    assert m(FAKE, FAKE, 65, FAKE, None, 16, 2, 64, None) == 2    # P above the limit
    assert m(FAKE, FAKE, 2, FAKE, None, 16, 2, 80, None) == 1     # d
    assert m(FAKE + 4, FAKE, 2, FAKE, None, 16, 2, 64, None) == 1  # alignment
    assert m(None, FAKE, 2, FAKE, None, 16, 2, 64, None) == 1


def test_fp16_partial_and_merge_reject(lib):
    p = lib.attn_fwd_partial_f16
    assert p(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 4, 2, 64, 0.1, 128, 128, None) == 1   # Sq = 0
    assert p(FAKE, FAKE, FAKE, FAKE, FAKE, 4, -1, 2, 64, 0.1, 128, 128, None) == 1  # Skv < 0
    assert p(FAKE, FAKE, FAKE, None, FAKE, 4, 4, 2, 64, 0.1, 128, 128, None) == 1   # o_part
    assert p(FAKE, FAKE, FAKE, FAKE + 8, FAKE, 4, 4, 2, 64, 0.1, 128, 128, None) == 1
    assert p(FAKE, FAKE, FAKE, FAKE, FAKE + 2, 4, 4, 2, 64, 0.1, 128, 128, None) == 1  # lse_part
    assert p(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 4, 2, 96, 0.1, 128, 128, None) == 1   # d
    m = lib.attn_merge_f16
    assert m(FAKE, FAKE, 0, FAKE, None, 16, 2, 64, None) == 1     # P = 0
    assert m(FAKE, FAKE, 65, FAKE, None, 16, 2, 64, None) == 2    # P above the limit
    assert m(FAKE, FAKE, 2, FAKE, None, 16, 2, 80, None) == 1     # d
    assert m(FAKE + 8, FAKE, 2, FAKE, None, 16, 2, 64, None) == 1  # alignment
    assert m(FAKE, FAKE, 2, FAKE + 2, None, 16, 2, 64, None) == 1
    assert m(None, FAKE, 2, FAKE, None, 16, 2, 64, None) == 1


def test_partials_reject(lib):
    for f in (lib.attn_fwd_partials, lib.attn_fwd_partials_f16):
        assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 4, 0, 2, 64, 0.1, 128, 128, None) == 1     # P = 0
        assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 4, 2, 2, 64, 0.1, 128, 128, None) == 1     # Sq = 0
        assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 4, -1, 2, 2, 64, 0.1, 128, 128, None) == 1    # Skv < 0
        assert f(FAKE, FAKE, FAKE, None, FAKE, 4, 4, 2, 2, 64, 0.1, 128, 128, None) == 1     # o_parts
        assert f(FAKE, FAKE, FAKE, FAKE + 8, FAKE, 4, 4, 2, 2, 64, 0.1, 128, 128, None) == 1
        assert f(FAKE, FAKE, FAKE, FAKE, FAKE + 2, 4, 4, 2, 2, 64, 0.1, 128, 128, None) == 1  # lse_parts
        assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 4, 2, 2, 96, 0.1, 128, 128, None) == 1     # d
        assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 4, 2, 2, 64, 0.1, 120, 128, None) == 1     # ld_q


def test_accumulate_rejects(lib):
    a = lib.attn_fwd_accumulate
    ok = (FAKE, FAKE, FAKE, FAKE, FAKE, None, 4, 4, 2, 64, 0.1, 128, 128, None)

    def call(**kw):
        names = ["q", "k", "v", "o", "lse", "out", "Sq", "Skv", "H", "d", "scale", "ld_q", "ld_kv", "s"]
        args = dict(zip(names, ok))
        args.update(kw)
        return a(*[args[n] for n in names])
    assert call(o=None) == 1
    assert call(lse=None) == 1
    assert call(o=FAKE + 4) == 1
    assert call(lse=FAKE + 2) == 1
    assert call(out=FAKE + 2) == 1
    assert call(Sq=0) == 1
    assert call(Skv=-1) == 1
    assert call(d=96) == 1
    assert call(scale=0.0) == 1
    assert call(ld_kv=100) == 1


def test_gathered_kv_and_batched_reject(lib):
    g = lib.attn_fwd_gathered_kv
    assert g(FAKE, FAKE, FAKE, FAKE, None, 4, 0, 2, 64, 0.1, 128, 128, 128, 128, None) == 1   # Skv = 0
    assert g(FAKE, FAKE, FAKE, FAKE, None, 0, 4, 2, 64, 0.1, 128, 128, 128, 128, None) == 1   # Sq = 0
    assert g(FAKE, FAKE, FAKE, FAKE, None, 4, 4, 2, 96, 0.1, 128, 128, 128, 128, None) == 1   # d
    assert g(FAKE, FAKE, FAKE, None, None, 4, 4, 2, 64, 0.1, 128, 128, 128, 128, None) == 1   # out
    b = lib.attn_fwd_batched
    assert b(FAKE, FAKE, FAKE, FAKE, None, 16, 0, 2, 64, 0.1, None) == 1    # B = 0
    assert b(FAKE, FAKE, FAKE, FAKE, None, 0, 2, 2, 64, 0.1, None) == 1     # S = 0
    assert b(FAKE, FAKE, FAKE, FAKE, None, 16, 2, 2, 80, 0.1, None) == 1    # d
    assert b(FAKE, FAKE, FAKE, FAKE, None, 16, 70000, 256, 128, 0.1, None) == 2  # B*H*d too wide


def test_qknorm_rejects(lib):
    f = lib.qkv_proj_qknorm
    f.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 4 + [ctypes.c_float, ctypes.c_void_p]
    assert f(FAKE, FAKE, None, FAKE, FAKE, 128, 2, 64, 128, 1e-6, None) == 1      # g_q
    assert f(FAKE, FAKE, FAKE, FAKE + 8, FAKE, 128, 2, 64, 128, 1e-6, None) == 1  # g_k alignment
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 128, 2, 96, 128, 1e-6, None) == 1      # d
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 128, 2, 64, 128, -1.0, None) == 1      # eps < 0
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 128, 2, 64, 128, float("nan"), None) == 1
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 128, 0, 64, 128, 1e-6, None) == 1      # H
    b = lib.attn_block_fwd_qknorm
    b.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_float] + [ctypes.c_void_p] * 4 + [ctypes.c_int] * 3 + \
        [ctypes.c_float, ctypes.c_void_p]
    assert b(FAKE, FAKE, FAKE, None, 1e-6, FAKE, FAKE, FAKE, FAKE, 16, 2, 64, 0.1, None) == 1  # one g only


def test_attn_kernel_choice(lib):
    assert lib.b2a_get_attn_kernel() == 0
    for c in (1, 2, 0):
        assert lib.b2a_set_attn_kernel(c) == 0
        assert lib.b2a_get_attn_kernel() == c
    assert lib.b2a_set_attn_kernel(3) == 1
    assert lib.b2a_set_attn_kernel(-1) == 1
    assert lib.b2a_get_attn_kernel() == 0


def test_gemm_rejects(lib):
    assert lib.qkv_proj(FAKE, FAKE, FAKE, 128, 100, 64, None) == 1   # N % 8
    assert lib.qkv_proj(FAKE, FAKE, FAKE, 128, 128, 60, None) == 1   # K % 8
    assert lib.qkv_proj(FAKE, FAKE, FAKE, 0, 128, 64, None) == 1
    assert lib.qkv_proj(None, FAKE, FAKE, 128, 128, 64, None) == 1
    assert lib.out_proj(FAKE, FAKE, FAKE + 2, FAKE, 128, 128, 64, None) == 1  # residual align


def test_host_workspace_layout(lib):
    def up(x):
        return (x + 255) // 256 * 256
    S, H, d = 1000, 3, 64
    n, nl = S * H * d, S * H
    base = 4 * up(n * 2) + up(nl * 4)
    assert lib.attn_fwd_host_workspace_bytes(S, H, d, 1) == base
    assert lib.attn_fwd_host_workspace_bytes(S, H, d, 3) == base + up(3 * n * 4) + up(3 * nl * 4)
    assert lib.attn_fwd_host_workspace_bytes(S, H, 80, 1) == 0
    assert lib.attn_fwd_host_workspace_bytes(S, H, d, 65) == 0
    small = lib.attn_fwd_host_workspace_bytes(S, H, d, 1)
    assert lib.attn_fwd_host(FAKE, FAKE, FAKE, FAKE, None, S, H, d, 0.1, 1, FAKE, small - 1, None) == 1
    assert lib.attn_fwd_host(FAKE, FAKE, FAKE, FAKE, None, S, H, d, 0.1, 1, FAKE + 16, small, None) == 1


def test_binding_chunk_bounds_partition_keys():
    import long_context_bidirectional_b200 as m
    for S, P in [(10, 3), (7, 7), (3, 5), (32768, 8)]:
        b = m.chunk_bounds(S, P)
        assert b[0][0] == 0 and b[-1][1] == S
        assert all(b[i][1] == b[i + 1][0] for i in range(P - 1))
