"""GPU edge cases: empty inputs, the bounded-wait machinery, launch counting."""

import pytest
import torch

import diffusion_transformer_joint_axial_b200 as qi
from diffusion_transformer_joint_axial_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
def test_empty_batch_and_heads(cuda_device, dtype):
    segs = [W.text(4), W.image(2, 2, 0)]
    pos, kv_end = qi.rope_positions(segs, cuda_device)
    for B, H in ((0, 2), (1, 0)):
        q = torch.zeros((B, 8, H, 128), dtype=dtype, device=cuda_device)
        o = qi.attn_full(q, q, q, pos, kv_end, 4)
        assert o.shape == q.shape
        qt = torch.zeros((B, 4, H, 128), dtype=dtype, device=cuda_device)
        kc = torch.zeros((B, H, 4, 128), dtype=dtype, device=cuda_device)
        oc = qi.attn_cached(qt, qt, qt, pos[4:].contiguous(), kc, kc)
        assert oc.shape == qt.shape


def test_cached_with_empty_prefix(cuda_device):
    """P = 0: the cached step is plain attention over the target alone."""
    import numpy as np
    import oracle as O
    from parity import assert_close
    segs = [W.image(9, 15, 0)]
    q, k, v = W.draw_qkv(1, 135, 2, 1, "bf16")
    pos, _ = qi.rope_positions(segs, cuda_device)
    kc = torch.zeros((1, 2, 0, 128), dtype=torch.bfloat16, device=cuda_device)
    o = qi.attn_cached(q.to(cuda_device), k.to(cuda_device), v.to(cuda_device), pos, kc, kc)
    opos, okv = O.positions(segs)
    ref = O.attn_full(W.as_f64(q), W.as_f64(k), W.as_f64(v), opos, okv)
    assert_close(o, ref, torch.bfloat16, "P=0")


def test_bounded_wait_times_out_and_context_survives(cuda_device):
    ws = qi.new_workspace(256, cuda_device)
    qi.selftest_wait_timeout(ws, 2_000_000)  # 2 ms on a barrier nobody arrives at
    assert qi.workspace_status(ws) == qi._binding.QI21_ERR_TIMEOUT
    assert qi.workspace_status(ws) == 0  # read-and-clear
    # the context is still usable
    pos, kv_end = qi.rope_positions([W.text(3)], cuda_device)
    assert pos.cpu().tolist() == [[0, 0, 0], [1, 1, 1], [2, 2, 2]]


def test_launch_count(cuda_device):
    segs = [W.text(16), W.image(4, 4, 0)]
    c0 = qi.launch_count()
    pos, kv_end = qi.rope_positions(segs, cuda_device)
    assert qi.launch_count() == c0 + 1
    q = torch.randn((1, 32, 2, 128), device=cuda_device).to(torch.bfloat16)
    qi.attn_full(q, q, q, pos, kv_end, 16)
    assert qi.launch_count() == c0 + 3  # rotation pre-pass + attention


def test_bad_shapes_rejected_by_binding(cuda_device):
    q = torch.zeros((1, 8, 2, 64), dtype=torch.bfloat16, device=cuda_device)
    pos, kv_end = qi.rope_positions([W.text(8)], cuda_device)
    with pytest.raises(qi.QI21Error):
        qi.attn_full(q, q, q, pos, kv_end, 8)
