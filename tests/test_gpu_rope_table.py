"""The per-request rotation table (qi21_rope_table) and the cached step that
reads it (qi21_attn_cached_tabled): the table against the float64 oracle's
angles (one rounding to float32 and one to float16), and the tabled cached
step against the ordinary one, which must agree bit for bit since both
rotate with the same rounded values; also against the oracle directly, for
bf16 and fp32, an empty Prefix and a ragged target."""

import numpy as np
import pytest
import torch

import diffusion_transformer_joint_axial_b200 as qi
import oracle as O
from diffusion_transformer_joint_axial_b200 import workloads as W

from parity import assert_close, gpu_full

pytestmark = pytest.mark.gpu

T_, I_ = W.text, W.image


def _split_table(table, n):
    raw = table.cpu().numpy()
    t32 = raw[: n * 64 * 8].view(np.float32).reshape(n, 64, 2)
    t16 = raw[n * 64 * 8:].view(np.float16).reshape(n, 64, 2)
    return t32, t16


def test_table_matches_oracle_angles(cuda_device):
    segs = [T_(77), I_(20, 30, 1), I_(16, 24, 0)]
    pos, _ = qi.rope_positions(segs, cuda_device)
    n = pos.shape[0]
    table = qi.rope_table(pos)
    torch.cuda.synchronize()
    assert table.numel() == n * 64 * 12
    t32, t16 = _split_table(table, n)
    ang = O.rope_angles(pos.cpu().numpy())
    c, s = np.cos(ang), np.sin(ang)
    for got, ref, ulp in ((t32[..., 0], c, 2.0 ** -24), (t32[..., 1], s, 2.0 ** -24),
                          (t16[..., 0], c, 2.0 ** -11), (t16[..., 1], s, 2.0 ** -11)):
        # one rounding of the exact value (plus the float64 libraries' last bit)
        err = np.abs(got.astype(np.float64) - ref)
        bound = 2.0 * ulp * np.maximum(np.abs(ref), 2.0 ** -14)
        assert np.all(err <= bound), float((err / bound).max())


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_tabled_cached_step_is_bit_identical(cuda_device, dtype):
    segs, B, H = [T_(130), I_(16, 16, 1), I_(20, 24, 0)], 2, 3
    L = sum(W.seg_tokens(s) for s in segs)
    T = W.seg_tokens(segs[-1])
    P = L - T
    kind = "bf16" if dtype == torch.bfloat16 else "f32"
    q, k, v = W.draw_qkv(B, L, H, 71, kind)
    g = gpu_full(segs, q, k, v, P)
    pt = g["pos"][P:].clone().to(cuda_device)
    table = qi.rope_table(pt)
    qt, kt, vt = (x.to(cuda_device) for x in W.draw_qkv(B, T, H, 72, kind))
    ws = qi.new_workspace(qi.cached_workspace_size(B, H, P, T, dtype), cuda_device)
    plain = qi.attn_cached(qt, kt, vt, pt, g["kc"], g["vc"], workspace=ws)
    assert qi.workspace_status(ws) == 0
    tabled = qi.attn_cached(qt, kt, vt, None, g["kc"], g["vc"], workspace=ws, rope_table=table)
    assert qi.workspace_status(ws) == 0
    assert torch.equal(plain, tabled)
    pos, _ = O.positions(segs)
    okc, ovc = O.prefix_cache(W.as_f64(k), W.as_f64(v), pos, P)
    ref = O.attn_cached(W.as_f64(qt.cpu()), W.as_f64(kt.cpu()), W.as_f64(vt.cpu()), pos[P:], okc, ovc)
    assert_close(tabled.cpu(), ref, dtype, "tabled cached step")


def test_tabled_cached_step_empty_prefix(cuda_device):
    """P = 0 and a target of 1000 tokens (a partly filled last query tile)."""
    segs, B, H = [I_(25, 40, 0)], 1, 2
    T = W.seg_tokens(segs[-1])
    pt, _ = qi.rope_positions(segs, cuda_device)
    table = qi.rope_table(pt)
    kc = vc = torch.zeros((B, H, 0, 128), dtype=torch.bfloat16, device=cuda_device)
    qt, kt, vt = (x.to(cuda_device) for x in W.draw_qkv(B, T, H, 73, "bf16"))
    ws = qi.new_workspace(qi.cached_workspace_size(B, H, 0, T, torch.bfloat16), cuda_device)
    plain = qi.attn_cached(qt, kt, vt, pt, kc, vc, workspace=ws)
    tabled = qi.attn_cached(qt, kt, vt, None, kc, vc, workspace=ws, rope_table=table)
    assert qi.workspace_status(ws) == 0
    assert torch.equal(plain, tabled)


def test_table_argument_errors(cuda_device):
    pos = torch.zeros((10, 3), dtype=torch.int32, device=cuda_device)
    lib = qi.load_library()
    short = torch.empty(10 * 64 * 12 - 16, dtype=torch.uint8, device=cuda_device)
    st = lib.qi21_rope_table(qi._binding._ptr(pos), 10, qi._binding._ptr(short), short.numel(), None)
    assert st == 1  # QI21_ERR_INVALID_ARG: nothing enqueued
    assert lib.qi21_rope_table(qi._binding._ptr(pos), -1, qi._binding._ptr(short), short.numel(), None) == 1
