"""Host-side checks of the C ABI that need no GPU: every symbol include/qi21.h
declares is exported by libqi21.so, and argument validation rejects bad calls
before anything is enqueued."""

import ctypes
import os
import re

import pytest

from diffusion_transformer_joint_axial_b200 import _binding as qb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qi21.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qi21_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(qb.LIB_PATH):
        pytest.skip("libqi21.so not built")
    return qb.load_library()


def test_header_declares_the_boundary():
    names = _declared_functions()
    for must in ("qi21_rope_positions", "qi21_attn_full", "qi21_attn_cached"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert names
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(qb.EXPORTED)


def test_status_strings(lib):
    for code, name in [(0, "QI21_OK"), (1, "QI21_ERR_INVALID_ARG"), (2, "QI21_ERR_UNSUPPORTED"),
                       (3, "QI21_ERR_CUDA"), (4, "QI21_ERR_TIMEOUT")]:
        assert lib.qi21_status_string(code).decode() == name


def test_workspace_sizes(lib):
    rnd = lambda x: (x + 255) // 256 * 256

    def split_region(B, H, rows):
        # tail-split scratch: arrival counters of up to 512 units, then up to
        # 512 piece slots of 64 KB (O / l) + 2 KB (row max, row sum)
        units = B * H * ((rows + 255) // 256)
        return rnd(min(units, 512) * 8 * 4) + min(4 * units, 512) * (65536 + 2048)

    def base(B, H, table_rows, k_rows):
        # header + cos/sin table (rows x 64 float2) + rotated keys of the rows
        # not stored in a cache (B x H x k_rows x 128 bf16)
        return rnd(rnd(256 + table_rows * 64 * 8) + B * H * k_rows * 128 * 2)

    full = lib.qi21_attn_full_workspace_size(1, 24, 4352, 256, qb.QI21_BF16)
    assert full == base(1, 24, 4352, 4096) + split_region(1, 24, 4352)
    assert full % 256 == 0
    no_cache = lib.qi21_attn_full_workspace_size(1, 24, 4352, 0, qb.QI21_BF16)
    assert no_cache == base(1, 24, 4352, 4352) + split_region(1, 24, 4352)
    f32 = lib.qi21_attn_full_workspace_size(1, 2, 300, 0, qb.QI21_F32)
    assert f32 == rnd(rnd(256 + 300 * 64 * 8) + 2 * 300 * 128 * 4)  # fp32: no split scratch
    assert lib.qi21_attn_full_workspace_size(1, 24, 4352, 4353, qb.QI21_BF16) == 0  # P > L
    cached = lib.qi21_attn_cached_workspace_size(1, 24, 256, 4096, qb.QI21_BF16)
    assert cached == base(1, 24, 4096, 4096) + split_region(1, 24, 4096)
    assert lib.qi21_attn_full_workspace_size(-1, 1, 1, 0, 0) == 0


def _segs(*items):
    arr = (qb.Segment * max(1, len(items)))()
    for i, it in enumerate(items):
        arr[i] = qb.Segment(*it)
    return arr


@pytest.mark.parametrize("segs,L", [
    (((0, 0, 0, 0, 0),), 0),          # text with n = 0
    (((1, 0, 0, 4, 0),), 0),          # image with H = 0
    (((7, 3, 0, 0, 0),), 3),          # unknown kind
    (((0, 3, 0, 0, 0),), 4),          # L does not match
])
def test_positions_rejects_bad_segments(lib, segs, L):
    arr = _segs(*segs)
    dummy = ctypes.c_void_p(16)
    st = lib.qi21_rope_positions(arr, len(segs), L, dummy, dummy, None)
    assert st == qb.QI21_ERR_INVALID_ARG
    assert lib.qi21_last_error().decode()


def test_positions_rejects_too_many_segments(lib):
    arr = _segs(*[(0, 1, 0, 0, 0)] * 129)
    st = lib.qi21_rope_positions(arr, 129, 129, ctypes.c_void_p(16), None, None)
    assert st == qb.QI21_ERR_INVALID_ARG


def test_positions_empty_is_noop(lib):
    assert lib.qi21_rope_positions(None, 0, 0, None, None, None) == qb.QI21_OK


def _full(lib, **kw):
    a = dict(B=1, H=2, L=32, P=16, dt=qb.QI21_F32, q=16, k=16, v=16, pos=16, kv=16, o=16,
             kc=None, vc=None, ws=256, wsb=1 << 30)
    a.update(kw)
    p = lambda x: ctypes.c_void_p(x) if x is not None else None
    return lib.qi21_attn_full(a["B"], a["H"], a["L"], a["P"], a["dt"], p(a["q"]), p(a["k"]), p(a["v"]),
                              p(a["pos"]), p(a["kv"]), p(a["o"]), p(a["kc"]), p(a["vc"]), p(a["ws"]),
                              a["wsb"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(P=33), qb.QI21_ERR_INVALID_ARG),            # P > L
    (dict(P=-1), qb.QI21_ERR_INVALID_ARG),
    (dict(B=-1), qb.QI21_ERR_INVALID_ARG),
    (dict(dt=5), qb.QI21_ERR_UNSUPPORTED),
    (dict(q=None), qb.QI21_ERR_INVALID_ARG),           # NULL input
    (dict(k=24), qb.QI21_ERR_INVALID_ARG),             # misaligned
    (dict(kc=16), qb.QI21_ERR_INVALID_ARG),            # k_cache without v_cache
    (dict(ws=272), qb.QI21_ERR_INVALID_ARG),           # workspace not 256-aligned
    (dict(wsb=100), qb.QI21_ERR_INVALID_ARG),          # workspace too small
])
def test_attn_full_rejects(lib, kw, code):
    assert _full(lib, **kw) == code


def test_attn_full_empty_is_noop(lib):
    assert _full(lib, L=0, P=0, q=None, k=None, v=None, o=None, ws=None) == qb.QI21_OK
    assert _full(lib, B=0, q=None, ws=None) == qb.QI21_OK
    assert _full(lib, H=0, q=None, ws=None) == qb.QI21_OK


def test_attn_cached_rejects(lib):
    p = ctypes.c_void_p
    ok = [p(16)] * 3
    args = lambda P, T, kc, ws, wsb: (1, 2, P, T, qb.QI21_BF16, *ok, p(16), kc, p(16), p(16), ws, wsb, None)
    assert lib.qi21_attn_cached(*args(-1, 4, p(16), p(256), 1 << 30)) == qb.QI21_ERR_INVALID_ARG
    assert lib.qi21_attn_cached(*args(4, 4, None, p(256), 1 << 30)) == qb.QI21_ERR_INVALID_ARG
    assert lib.qi21_attn_cached(*args(4, 4, p(16), p(256), 10)) == qb.QI21_ERR_INVALID_ARG
    assert lib.qi21_attn_cached(*args(4, 0, p(16), p(256), 10)) == qb.QI21_OK  # T = 0: nothing to do


def test_qknorm_rejects(lib):
    p = ctypes.c_void_p
    full = lambda nq, nk, eps: lib.qi21_attn_full_qknorm(
        1, 2, 32, 16, qb.QI21_BF16, p(16), p(16), p(16), p(16), p(16), p(16), None, None, nq, nk,
        ctypes.c_float(eps), p(256), 1 << 30, None)
    cached = lambda nq, nk, eps: lib.qi21_attn_cached_qknorm(
        1, 2, 16, 16, qb.QI21_BF16, p(16), p(16), p(16), p(16), p(16), p(16), p(16), nq, nk,
        ctypes.c_float(eps), p(256), 1 << 30, None)
    for fn in (full, cached):
        assert fn(None, p(16), 1e-6) == qb.QI21_ERR_INVALID_ARG      # weights missing
        assert fn(p(16), None, 1e-6) == qb.QI21_ERR_INVALID_ARG
        assert fn(p(16), p(20), 1e-6) == qb.QI21_ERR_INVALID_ARG     # misaligned weight
        assert fn(p(16), p(16), -1.0) == qb.QI21_ERR_INVALID_ARG     # negative eps
        assert fn(p(16), p(16), float("nan")) == qb.QI21_ERR_INVALID_ARG
        assert fn(p(16), p(16), float("inf")) == qb.QI21_ERR_INVALID_ARG
        assert "eps" in lib.qi21_last_error().decode()


def test_linear_rejects(lib):
    p = ctypes.c_void_p
    outs = (p * 4)(16, 16, 16, 16)
    lin = lambda M=64, N=96, K=64, x=16, w=16, b=None, out=outs, n=1, ws=256, wsb=256: lib.qi21_linear(
        M, N, K, p(x) if x else None, p(w) if w else None, p(b) if b else None, out, n,
        p(ws) if ws else None, wsb, None)
    bad = qb.QI21_ERR_INVALID_ARG
    assert lin(n=0) == bad and lin(n=5) == bad          # segment count
    assert lin(N=96, n=5) == bad                         # N not divisible
    assert lin(N=36, n=3) == bad                         # segment not a multiple of 8
    assert lin(K=60) == bad                              # K not a multiple of 8
    assert lin(K=0) == bad
    assert lin(M=-1) == bad
    assert lin(x=None) == bad and lin(w=24) == bad       # NULL / misaligned operand
    assert lin(b=40) == bad                              # misaligned bias
    assert lin(out=None) == bad
    assert lin(out=(p * 4)(16, 20, 16, 16), N=96, n=2) == bad  # misaligned second output
    assert lin(wsb=100) == bad                           # workspace smaller than its header
    assert lin(M=0, x=None, w=None, ws=None) == qb.QI21_OK  # nothing to do


def test_block_ops_reject(lib):
    p = ctypes.c_void_p
    bad = qb.QI21_ERR_INVALID_ARG
    lr = lambda residual=16, alpha=1.0, N=64: lib.qi21_linear_residual(
        32, N, 64, p(16), p(16), None, p(residual) if residual else None, ctypes.c_float(alpha), p(16),
        p(256), 256, None)
    assert lr(residual=None) == bad and lr(residual=24) == bad   # missing / misaligned residual
    assert lr(alpha=float("nan")) == bad and lr(alpha=float("inf")) == bad
    assert lr(N=60) == bad                                        # N not a multiple of 8
    rn = lambda M=4, D=64, eps=1e-6, x=16: lib.qi21_rmsnorm(M, D, p(x) if x else None, p(16), ctypes.c_float(eps),
                                                           p(16), None)
    assert rn(D=60) == bad and rn(D=0) == bad and rn(eps=-1.0) == bad and rn(x=None) == bad
    assert rn(M=0, x=None) == qb.QI21_OK
    ls = lambda N=512: lib.qi21_linear_swiglu(32, N, 64, p(16), p(16), None, p(16), p(256), 256, None)
    assert ls(N=384) == bad and ls(N=200) == bad                  # gate/up blocks of 128 need N % 256 == 0
    sw = lambda n=64, g=16: lib.qi21_swiglu(n, p(g) if g else None, p(16), p(16), None)
    assert sw(n=60) == bad and sw(n=-8) == bad and sw(g=None) == bad and sw(g=8) == bad
    assert sw(n=0, g=None) == qb.QI21_OK


def test_selftest_rejects_bad_limit(lib):
    assert lib.qi21_selftest_wait_timeout(ctypes.c_void_p(256), 0, None) == qb.QI21_ERR_INVALID_ARG


def test_binding_fails_loudly_without_cuda(monkeypatch):
    import torch
    monkeypatch.setattr(torch.cuda, "is_available", lambda: False)
    with pytest.raises(qb.QI21Error):
        qb.rope_positions([{"kind": "text", "n": 4}])


def test_rope_table_sizes_and_rejects(lib):
    """qi21_rope_table: n x 64 pairs as float2 then half2 (12 bytes a pair);
    bad sizes, pointers and short buffers are rejected before anything is
    enqueued, and so are the tabled cached step's."""
    p = ctypes.c_void_p
    bad = qb.QI21_ERR_INVALID_ARG
    for n in (0, 1, 77, 4096):
        assert lib.qi21_rope_table_size(n) == n * 64 * 12
    assert lib.qi21_rope_table_size(-1) == 0
    tab = lambda n=16, pos=16, t=256, tb=16 * 768: lib.qi21_rope_table(
        p(pos) if pos else None, n, p(t) if t else None, tb, None)
    assert tab(n=-1) == bad and tab(n=(1 << 30) + 1) == bad
    assert tab(pos=None) == bad and tab(pos=20) == bad       # NULL / misaligned positions
    assert tab(t=None) == bad and tab(t=24) == bad           # NULL / misaligned table
    assert tab(tb=16 * 768 - 16) == bad                      # table buffer too small
    assert tab(n=0, pos=None, t=None) == qb.QI21_OK          # nothing to do
    cached = lambda T=16, table=16: lib.qi21_attn_cached_tabled(
        1, 2, 16, T, qb.QI21_BF16, p(16), p(16), p(16), p(table) if table else None, p(16), p(16), p(16),
        p(256), 1 << 30, None)
    assert cached(T=-1) == bad
    assert cached(table=None) == bad and cached(table=24) == bad
