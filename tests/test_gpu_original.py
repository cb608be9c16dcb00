"""The earlier Qwen-Image model's layout as a second workload of the same
attention kernels: position table with text after the images (bit-exact),
no mask, [text | target | reference] order; against the float64 oracle."""

import numpy as np
import pytest
import torch

import diffusion_transformer_joint_axial_b200 as qi
import oracle as O
from diffusion_transformer_joint_axial_b200 import workloads as W

from parity import assert_close, check_status, sample_rows

pytestmark = pytest.mark.gpu

T_, I_ = W.text, W.image
LAYOUTS = {
    "edit_small": [T_(40), I_(8, 10, 0), I_(6, 6, 1)],
    "odd": [T_(7), I_(5, 3, 0), I_(9, 1, 1), I_(3, 7, 2)],
    "text_only": [T_(50)],
    "orig": W.WORKLOADS["orig"]["segments"],
}


@pytest.mark.parametrize("name", sorted(LAYOUTS))
def test_original_positions_bit_exact(cuda_device, name):
    segs = LAYOUTS[name]
    pos, kv_end = qi.rope_positions(segs, cuda_device, original=True)
    opos, okv = O.positions_original(segs)
    assert np.array_equal(pos.cpu().numpy(), opos)
    assert np.array_equal(kv_end.cpu().numpy(), okv)


def _full(segs, q, k, v, dev):
    B, L, H, _ = q.shape
    pos, kv_end = qi.rope_positions(segs, dev, original=True)
    ws = qi.new_workspace(qi.full_workspace_size(B, H, L, 0, q.dtype), dev)
    o = qi.attn_full(q.to(dev), k.to(dev), v.to(dev), pos, kv_end, 0, workspace=ws)
    check_status(ws)
    torch.cuda.synchronize()
    return o.cpu()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
@pytest.mark.parametrize("name", ["edit_small", "odd", "text_only"])
def test_original_small_layouts(cuda_device, name, dtype):
    segs = LAYOUTS[name]
    L = sum(W.seg_tokens(s) for s in segs)
    q, k, v = W.draw_qkv(2, L, 3, 23, "bf16" if dtype == torch.bfloat16 else "f32")
    got = _full(segs, q, k, v, cuda_device)
    opos, okv = O.positions_original(segs)
    ref = O.attn_full(W.as_f64(q), W.as_f64(k), W.as_f64(v), opos, okv)
    assert_close(got, ref, dtype, "original " + name)


def test_original_workload_full_size_sampled(cuda_device):
    name = "orig"
    cfg = W.WORKLOADS[name]
    L = sum(W.seg_tokens(s) for s in cfg["segments"])
    q, k, v = W.full_inputs(name)
    got = _full(cfg["segments"], q, k, v, cuda_device)
    opos, okv = O.positions_original(cfg["segments"])
    rows = sample_rows(L, 256, okv, np.random.default_rng(7))
    hs = [0, 12, 23]
    ref = O.attn_full(*(W.as_f64(x[:, :, hs]) for x in (q, k, v)), opos, okv, rows=rows)
    assert_close(got[:, rows][:, :, hs], ref, torch.bfloat16, "orig full (sampled)")


def _full_unmasked(segs, q, k, v, dev):
    """The same call with kv_end = NULL (no mask): the launcher may split the
    last wave of units into key-range pieces."""
    B, L, H, _ = q.shape
    pos, _ = qi.rope_positions(segs, dev, original=True)
    ws = qi.new_workspace(qi.full_workspace_size(B, H, L, 0, q.dtype), dev)
    o = qi.attn_full(q.to(dev), k.to(dev), v.to(dev), pos, None, 0, workspace=ws)
    check_status(ws)
    torch.cuda.synchronize()
    return o.cpu()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
@pytest.mark.parametrize("name", ["edit_small", "odd", "split_4"])
def test_original_without_kv_end(cuda_device, name, dtype):
    """kv_end NULL means every key is visible: the oracle's unmasked result.
    split_4 (32 units of 16 key tiles) is split into 4 pieces per unit."""
    segs = LAYOUTS[name] if name in LAYOUTS else [T_(256), I_(32, 32, 0), I_(24, 32, 1)]
    L = sum(W.seg_tokens(s) for s in segs)
    B, H = (1, 4) if name == "split_4" else (2, 3)
    q, k, v = W.draw_qkv(B, L, H, 29, "bf16" if dtype == torch.bfloat16 else "f32")
    got = _full_unmasked(segs, q, k, v, cuda_device)
    opos, okv = O.positions_original(segs)
    ref = O.attn_full(W.as_f64(q), W.as_f64(k), W.as_f64(v), opos, okv)
    assert_close(got, ref, dtype, "original without kv_end " + name)


def test_original_workload_full_size_without_kv_end(cuda_device):
    """The earlier model's full workload with kv_end NULL (its last wave is
    split into 3 pieces per unit on a 148-SM B200), sampled rows including the
    rows of the split units (rows 0-255 of every head)."""
    name = "orig"
    cfg = W.WORKLOADS[name]
    L = sum(W.seg_tokens(s) for s in cfg["segments"])
    q, k, v = W.full_inputs(name)
    got = _full_unmasked(cfg["segments"], q, k, v, cuda_device)
    opos, okv = O.positions_original(cfg["segments"])
    rows = sample_rows(L, 256, okv, np.random.default_rng(8))
    hs = [0, 12, 23]
    ref = O.attn_full(*(W.as_f64(x[:, :, hs]) for x in (q, k, v)), opos, okv, rows=rows)
    assert_close(got[:, rows][:, :, hs], ref, torch.bfloat16, "orig full without kv_end (sampled)")
