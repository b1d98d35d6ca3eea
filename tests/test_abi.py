"""The C-ABI library on the CPU: it loads, exports every symbol the header
declares, and rejects bad arguments on the host before touching a device.

No call here reaches CUDA: each either is host-only (version, path count,
workspace queries, status strings) or fails argument validation first.
"""
import ctypes
import os
import re

import pytest

from equivariant_graph_attention_b200 import egat

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from equivariant_graph_attention_b200.build import build
    build()
    return egat.load_library()


def _declared():
    with open(os.path.join(ROOT, "include", "egat.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"EGAT_API\s+[\w\s\*]+?\b(egat_\w+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert names == sorted(egat.EXPORTS)
    for n in names:
        assert hasattr(lib, n), n
    # nothing else is exported: the internal C++ symbols are hidden
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", egat._LIB_PATH], capture_output=True,
                         text=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert {n for n in exported if n.startswith("egat_")} == set(names)


def test_host_only_queries(lib):
    assert egat.egat_version() == 1
    assert [egat.egat_num_paths(l) for l in range(5)] == [1, 5, 15, 34, 0]
    assert lib.egat_strerror(0) == b"success"
    assert b"workspace" in lib.egat_strerror(egat.EGAT_ERR_WORKSPACE)
    assert egat.egat_graph_workspace_bytes(1000) > 0
    s = egat.Shape(n=32768, lmax=2, C=128, H=16, dk=16, K=256, dtype="bf16")
    # h' plus, for tensor-core shapes, the attention plan (2048 tiles: union
    # capacity 4096 ints, a 16 x 128-word mask and a target record of a
    # 4-word header + 16 x (1 id + 3 powers |r|^l + 35 Wigner-D entries) words
    # each, plus lengths and the attention kernel's tile-claim counter in a
    # 256-byte block of its own)
    plan = egat.egat_attention_plan_bytes(s)
    assert plan == 2048 * 4 + 2048 * 4096 * 4 + 2048 * 16 * 128 * 4 + 2048 * (4 + 16 * 39) * 4 + 256
    assert egat.egat_forward_workspace_bytes(s) == 32768 * 9 * 128 * 2 + plan
    f32 = egat.Shape(n=648, lmax=2, C=128, H=16, dk=16, K=64, dtype="f32")
    assert egat.egat_forward_workspace_bytes(f32) == 648 * 9 * 128 * 4


@pytest.mark.parametrize("field,value,code", [
    ("lmax", 4, egat.EGAT_ERR_UNSUPPORTED), ("lmax", 0, egat.EGAT_ERR_UNSUPPORTED),
    ("C", 96, egat.EGAT_ERR_UNSUPPORTED), ("H", 3, egat.EGAT_ERR_UNSUPPORTED),
    ("dk", 12, egat.EGAT_ERR_UNSUPPORTED), ("K", 0, egat.EGAT_ERR_ARG),
    ("K", 2000, egat.EGAT_ERR_ARG), ("n", -1, egat.EGAT_ERR_ARG), ("dtype", "f16", None)])
def test_shape_validation(lib, field, value, code):
    base = dict(n=10, lmax=2, C=128, H=16, dk=16, K=64, dtype="f32")
    base[field] = value
    if value == "f16":
        cs = egat.egat_shape(10, 2, 128, 16, 16, 64, 7, 0, 0)
        code = egat.EGAT_ERR_ARG
    else:
        cs = egat.Shape(**base).c()
    out = ctypes.c_size_t(0)
    assert lib.egat_forward_workspace_bytes(ctypes.byref(cs), ctypes.byref(out)) == code
    fake = ctypes.c_void_p(0x10000)
    rc = lib.egat_forward(ctypes.byref(cs), fake, fake, fake, fake, fake, fake, None, fake, fake,
                          fake, 1 << 30, fake, None)
    assert rc == code


def test_pointer_and_size_validation(lib):
    cs = egat.Shape(n=10, lmax=2, C=128, H=16, dk=16, K=64, dtype="bf16").c()
    ok = ctypes.c_void_p(0x10000)
    odd = ctypes.c_void_p(0x10008)     # not 16-byte aligned
    args = [ok, ok, ok, ok, ok, ok, None, ok, ok, ok, 1 << 30, ok, None]
    for slot in (0, 2, 3, 9, 11):      # h, q, k, workspace, out
        a = list(args)
        a[slot] = odd
        assert lib.egat_forward(ctypes.byref(cs), *a) == egat.EGAT_ERR_ARG
        b = list(args)
        b[slot] = None
        assert lib.egat_forward(ctypes.byref(cs), *b) == egat.EGAT_ERR_ARG
    small = list(args)
    small[10] = 100
    assert lib.egat_forward(ctypes.byref(cs), *small) == egat.EGAT_ERR_WORKSPACE
    assert lib.egat_forward(None, *args) == egat.EGAT_ERR_ARG
    # graph builder: bad cutoff, bad K, bad mode, missing overflow, key overflow
    g = lambda n, cut, K, mode, ovf: lib.egat_build_graph(ok, n, cut, K, mode, ok, ok, 0, None,
                                                          ovf, ok, 1 << 30, None)
    assert g(10, 0, 8, 0, ok) == egat.EGAT_ERR_ARG
    assert g(10, 100, 0, 0, ok) == egat.EGAT_ERR_ARG
    assert g(10, 100, 8, 5, ok) == egat.EGAT_ERR_ARG
    assert g(10, 100, 8, 0, None) == egat.EGAT_ERR_ARG
    assert g(1 << 30, 2 ** 31 - 1, 8, 0, ok) == egat.EGAT_ERR_UNSUPPORTED
    assert g(10, (1 << 26) + 1, 8, 0, ok) == egat.EGAT_ERR_UNSUPPORTED


def test_plan_and_status_entry_validation(lib):
    """Host-side checks of the plan, planned-coupling, tiled-attention and
    self-test entry points (no launch happens on these paths)."""
    cs = egat.Shape(n=10, lmax=2, C=128, H=16, dk=16, K=64, dtype="bf16").c()
    ok = ctypes.c_void_p(0x10000)
    odd = ctypes.c_void_p(0x10008)
    # plan: positions are required; the plan buffer must be 16-byte aligned and large enough
    assert lib.egat_build_attention_plan(ctypes.byref(cs), ok, ok, None, None, ok, 1 << 30,
                                         None) == egat.EGAT_ERR_ARG
    assert lib.egat_build_attention_plan(ctypes.byref(cs), ok, ok, None, ok, odd, 1 << 30,
                                         None) == egat.EGAT_ERR_ARG
    assert lib.egat_build_attention_plan(ctypes.byref(cs), ok, ok, None, ok, ok, 16,
                                         None) == egat.EGAT_ERR_WORKSPACE
    csr = egat.Shape(n=10, lmax=2, C=128, H=16, dk=16, K=64, dtype="bf16", graph_mode="csr",
                     n_edges=10).c()
    assert lib.egat_build_attention_plan(ctypes.byref(csr), ok, ok, None, ok, ok, 1 << 30,
                                         None) == egat.EGAT_ERR_UNSUPPORTED
    # planned coupling: every pointer required, storage 16-byte aligned
    assert lib.egat_eaas_couple_planned(ctypes.byref(cs), None, ok, ok, ok, None) == egat.EGAT_ERR_ARG
    assert lib.egat_eaas_couple_planned(ctypes.byref(cs), odd, ok, ok, ok, None) == egat.EGAT_ERR_ARG
    # tiled attention: w2 required when fused, not otherwise checked
    assert lib.egat_otf_attention_tiled(ctypes.byref(cs), ok, ok, ok, ok, None, ok, 1,
                                        None) == egat.EGAT_ERR_ARG
    f32 = egat.Shape(n=10, lmax=2, C=128, H=16, dk=16, K=64, dtype="f32").c()
    assert lib.egat_otf_attention_tiled(ctypes.byref(f32), ok, ok, ok, ok, ok, ok, 1,
                                        None) == egat.EGAT_ERR_UNSUPPORTED
    # self-test: poll count range
    assert lib.egat_selftest_wait_timeout(0, None) == egat.EGAT_ERR_ARG
    assert lib.egat_selftest_wait_timeout((1 << 20) + 1, None) == egat.EGAT_ERR_ARG
    assert lib.egat_strerror(egat.EGAT_ERR_TIMEOUT).startswith(b"a bounded device wait")


@pytest.mark.parametrize("n,K,supported", [
    (131072, 1024, True),     # bitmap builder: 32 KB of bitmaps + 32 KB mask + 64 KB of entries
    (131073, 512, True),      # hash builder past 131,072 atoms: shared memory set by K alone
    (1000000, 256, True),
    (131073, 1024, False),    # hash builder at K = 1024: 224 KiB, past the 200 KiB limit
])
def test_attention_plan_size_limits(lib, n, K, supported):
    """The documented limits of the attention plan: the bitmap builder up to
    131,072 atoms at every K, the hash builder beyond at K <= 512, whatever
    n is (its per-tile cost does not grow with n); the plan's size grows
    linearly in the tile count."""
    cs = egat.Shape(n=n, lmax=2, C=128, H=16, dk=16, K=K, dtype="bf16").c()
    out = ctypes.c_size_t(0)
    rc = lib.egat_attention_plan_bytes(ctypes.byref(cs), ctypes.byref(out))
    assert rc == (egat.EGAT_OK if supported else egat.EGAT_ERR_UNSUPPORTED)
    if supported:
        tiles = (n + 15) // 16
        cap = 32
        while cap < 16 * K:
            cap *= 2
        a256 = lambda x: (x + 255) // 256 * 256
        per_tile = 4 + cap * 4 + 16 * (cap // 32) * 4 + (4 + 16 * 39) * 4
        assert out.value == a256(tiles * 4) + a256(tiles * cap * 4) + a256(tiles * 16 * (cap // 32) * 4) \
            + a256(tiles * (4 + 16 * 39) * 4) + 256
        assert abs(out.value - tiles * per_tile) <= 4 * 256


def test_backward_entry_validation(lib):
    """egat_backward's host checks and workspace query (no launch on these paths)."""
    a256 = lambda x: (x + 255) // 256 * 256
    n, K, H, D, C = 32768, 256, 16, 9, 128
    s = egat.Shape(n=n, lmax=2, C=C, H=H, dk=16, K=K, dtype="bf16")
    tiles = n // 16
    ucap = n * K + 32 * tiles
    per_edge = (2 * a256(n * D * C * 4) + a256(n * 4) + a256((n + 1) * 4) + a256(n * 4)
                + 2 * a256(n * K * 4) + 2 * a256(n * H * 4))
    tiled = (2 * a256(n * D * C * 4) + a256(n * 2 * H * 4) + egat.egat_attention_plan_bytes(s)
             + 3 * a256((tiles + 1) * 4) + a256(ucap * 4) + a256(ucap // 2 * 4))
    # the tensor-core shape reserves the tiled passes' buffers (m, dL/dh', statistics, the forward
    # plan and the source plan at n*K + 32 per tile union entries) on top of the gather path's
    assert egat.egat_backward_workspace_bytes(s) == per_edge + a256(tiled)
    f32 = egat.Shape(n=648, lmax=2, C=C, H=H, dk=16, K=64, dtype="f32")
    assert egat.egat_backward_workspace_bytes(f32) == (
        2 * a256(648 * D * C * 4) + a256(648 * 4) + a256(649 * 4) + a256(648 * 4)
        + 2 * a256(648 * 64 * 4) + 2 * a256(648 * H * 4))

    cs = egat.Shape(n=10, lmax=2, C=C, H=H, dk=16, K=64, dtype="bf16").c()
    ok = ctypes.c_void_p(0x10000)
    odd4 = ctypes.c_void_p(0x10002)    # not 4-byte aligned
    odd16 = ctypes.c_void_p(0x10008)   # not 16-byte aligned
    # s, h, pos, q, k, nbr, cnt, order, w1, w2, grad_out, ws, ws_bytes, dh, dq, dk, dpos, stream
    args = [ok, ok, ok, ok, ok, ok, None, ok, ok, ok, ok, 1 << 30, ok, ok, ok, None, None]
    assert lib.egat_backward(ctypes.byref(cs), *args[:6], odd4, *args[7:]) == egat.EGAT_ERR_ARG
    for slot in (0, 2, 3, 9, 10, 12):   # h, q, k, grad_out, workspace, dh: 16-byte alignment
        a = list(args)
        a[slot] = odd16
        assert lib.egat_backward(ctypes.byref(cs), *a) == egat.EGAT_ERR_ARG
    for slot in (0, 1, 2, 3, 4, 7, 8, 9, 10, 12, 13, 14):   # required pointers
        a = list(args)
        a[slot] = None
        assert lib.egat_backward(ctypes.byref(cs), *a) == egat.EGAT_ERR_ARG
    small = list(args)
    small[11] = 64
    assert lib.egat_backward(ctypes.byref(cs), *small) == egat.EGAT_ERR_WORKSPACE
    csr = egat.Shape(n=10, lmax=2, C=C, H=H, dk=16, K=64, dtype="bf16", graph_mode="csr",
                     n_edges=10).c()
    assert lib.egat_backward(ctypes.byref(csr), *args) == egat.EGAT_ERR_UNSUPPORTED


def test_gather_rows_validation(lib):
    """egat_gather_rows' host checks; a zero count returns before any launch."""
    ok = ctypes.c_void_p(0x10000)
    odd = ctypes.c_void_p(0x10008)
    assert lib.egat_gather_rows(ok, 10, 64, ok, 0, ok, None) == egat.EGAT_OK
    assert lib.egat_gather_rows(ok, 10, 24, ok, 4, ok, None) == egat.EGAT_ERR_ARG     # row size
    assert lib.egat_gather_rows(ok, 10, 0, ok, 4, ok, None) == egat.EGAT_ERR_ARG
    assert lib.egat_gather_rows(ok, -1, 64, ok, 4, ok, None) == egat.EGAT_ERR_ARG
    assert lib.egat_gather_rows(ok, 10, 64, ok, -4, ok, None) == egat.EGAT_ERR_ARG
    assert lib.egat_gather_rows(ok, 10, 64, None, 4, ok, None) == egat.EGAT_ERR_ARG
    assert lib.egat_gather_rows(ok, 10, 64, ok, 4, None, None) == egat.EGAT_ERR_ARG
    assert lib.egat_gather_rows(ok, 10, 64, ok, 4, odd, None) == egat.EGAT_ERR_ARG
    assert lib.egat_gather_rows(odd, 10, 64, ok, 4, ok, None) == egat.EGAT_ERR_ARG
    assert lib.egat_gather_rows(None, 10, 64, ok, 4, ok, None) == egat.EGAT_ERR_ARG


def test_escn_weight_count_matches_the_oracle():
    """The library's SO(2) weight-row count (host code, no GPU work) equals the
    oracle's and the input generator's for every (lmax, mmax); out of range
    gives 0."""
    from equivariant_graph_attention_b200 import egat, synth
    from oracle.escn import num_weights
    lib = egat.load_library()
    for L in (1, 2, 3):
        for m in range(L + 1):
            assert lib.egat_escn_num_weights(L, m) == num_weights(L, m) == synth.escn_weight_count(L, m)
    assert lib.egat_escn_num_weights(0, 0) == 0 and lib.egat_escn_num_weights(2, 3) == 0
    assert lib.egat_escn_num_weights(4, 1) == 0 and lib.egat_escn_num_weights(2, -1) == 0
