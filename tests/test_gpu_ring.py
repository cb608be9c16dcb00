"""The key/value ring across work items: slot t holds key tile t and value
tile t - 1 of a CTA's whole sequence of items, and a unit's last slot (whose
key tile is the next unit's first) is released only after the next unit's
first S MMAs.  Units with one or two key tiles, several hundred of them (each
CTA runs a chain of short items back to back), in the full and the cached
step, compared with the float64 oracle on every head."""

import pytest
import torch

import diffusion_transformer_joint_axial_b200 as qi
import oracle as O
from diffusion_transformer_joint_axial_b200 import workloads as W

from parity import assert_close, gpu_full

pytestmark = pytest.mark.gpu

T_, I_ = W.text, W.image

# name: (segments, B, H); every unit has one or two key tiles
CASES = {
    # cached: T = 128, P = 0 -> one key tile per unit; 384 units
    "one_tile_units": ([I_(8, 16, 0)], 4, 96),
    # cached: T = 256, P = 0 -> two key tiles per unit; 288 units
    "two_tile_units": ([I_(16, 16, 0)], 3, 96),
    # full: text 64 + target 8 x 8 (L = 128, one key tile), cached: 64 target rows over 2 tiles' keys
    "tiny_prefix": ([T_(64), I_(8, 8, 0)], 4, 80),
}


def _run(name, cuda_device):
    segs, B, H = CASES[name]
    L = sum(W.seg_tokens(s) for s in segs)
    T = W.seg_tokens(segs[-1])
    P = L - T
    q, k, v = W.draw_qkv(B, L, H, 81, "bf16")
    pos, kv_end = O.positions(segs)
    if P > 0:
        g = gpu_full(segs, q, k, v, P)
        ref = O.attn_full(W.as_f64(q), W.as_f64(k), W.as_f64(v), pos, kv_end)
        assert_close(g["o"], ref, torch.bfloat16, "%s full step" % name)
        kc, vc, pt = g["kc"], g["vc"], g["pos"][P:].clone().to(cuda_device)
    else:
        kc = vc = torch.zeros((B, H, 0, 128), dtype=torch.bfloat16, device=cuda_device)
        pt, _ = qi.rope_positions(segs, cuda_device)
    okc, ovc = O.prefix_cache(W.as_f64(k), W.as_f64(v), pos, P)
    qt, kt, vt = W.draw_qkv(B, T, H, 82, "bf16")
    ws = qi.new_workspace(qi.cached_workspace_size(B, H, P, T, torch.bfloat16), cuda_device)
    for _ in range(2):  # a second call on the same workspace
        oc = qi.attn_cached(qt.to(cuda_device), kt.to(cuda_device), vt.to(cuda_device), pt, kc, vc,
                            workspace=ws)
        assert qi.workspace_status(ws) == 0
    ref = O.attn_cached(W.as_f64(qt), W.as_f64(kt), W.as_f64(vt), pos[P:], okc, ovc)
    assert_close(oc.cpu(), ref, torch.bfloat16, "%s cached step" % name)


@pytest.mark.parametrize("name", sorted(CASES))
def test_ring_across_short_units(cuda_device, name):
    _run(name, cuda_device)
