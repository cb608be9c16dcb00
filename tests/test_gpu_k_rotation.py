"""The key-rotation placement ablation (QI21_K_ROTATION=attention): the keys
that do not go to the Prefix cache reach the attention kernel unrotated, and
its epilogue warps turn each of their tiles in shared memory from the query
table before the tile's S MMAs; the pre-pass then rotates only the Prefix
keys (into the cache).  Full and cached steps are compared with the float64
oracle on layouts with several key tiles, ragged last tiles, an empty Prefix
and two batches, and the cache the full step writes is checked as well."""

import pytest
import torch

import diffusion_transformer_joint_axial_b200 as qi
import oracle as O
from diffusion_transformer_joint_axial_b200 import workloads as W

from parity import assert_close, check_cache, gpu_full

pytestmark = pytest.mark.gpu

T_, I_ = W.text, W.image

# name: (segments, B, H); the target is the last segment
CASES = {
    # Prefix of 2 key tiles, target of 8: several tiles, no ragged edge
    "text_256_image_32x32": ([T_(256), I_(32, 32, 0)], 1, 6),
    # ragged Prefix (77 tokens) and ragged target (600 tokens)
    "ragged": ([T_(77), I_(20, 30, 0)], 1, 4),
    # two batches, a reference image in the Prefix, ragged target
    "two_batches_edit": ([T_(130), I_(16, 16, 1), I_(20, 24, 0)], 2, 3),
}


@pytest.fixture
def rotate_in_attention(monkeypatch):
    monkeypatch.setenv("QI21_K_ROTATION", "attention")


def _sizes(segs):
    L = sum(W.seg_tokens(s) for s in segs)
    T = W.seg_tokens(segs[-1])
    return L, L - T, T


@pytest.mark.parametrize("name", sorted(CASES))
def test_keys_rotated_in_attention_match_oracle(cuda_device, rotate_in_attention, name):
    segs, B, H = CASES[name]
    L, P, T = _sizes(segs)
    q, k, v = W.draw_qkv(B, L, H, 61, "bf16")
    pos, kv_end = O.positions(segs)
    g = gpu_full(segs, q, k, v, P)
    ref = O.attn_full(W.as_f64(q), W.as_f64(k), W.as_f64(v), pos, kv_end)
    assert_close(g["o"], ref, torch.bfloat16, "%s full step" % name)
    check_cache(g["kc"], g["vc"], k, v, pos, P)
    okc, ovc = O.prefix_cache(W.as_f64(k), W.as_f64(v), pos, P)
    qt, kt, vt = W.draw_qkv(B, T, H, 62, "bf16")
    ws = qi.new_workspace(qi.cached_workspace_size(B, H, P, T, torch.bfloat16), cuda_device)
    oc = qi.attn_cached(qt.to(cuda_device), kt.to(cuda_device), vt.to(cuda_device),
                        g["pos"][P:].contiguous().to(cuda_device), g["kc"], g["vc"], workspace=ws)
    assert qi.workspace_status(ws) == 0
    refc = O.attn_cached(W.as_f64(qt), W.as_f64(kt), W.as_f64(vt), pos[P:], okc, ovc)
    assert_close(oc.cpu(), refc, torch.bfloat16, "%s cached step" % name)


def test_keys_rotated_in_attention_empty_prefix(cuda_device, rotate_in_attention):
    """P = 0: every key of the cached step is the target's own and unrotated."""
    segs, B, H = [I_(24, 40, 0)], 1, 3
    T = W.seg_tokens(segs[-1])
    pos, _ = O.positions(segs)
    pt, _ = qi.rope_positions(segs, cuda_device)
    kc = vc = torch.zeros((B, H, 0, 128), dtype=torch.bfloat16, device=cuda_device)
    qt, kt, vt = W.draw_qkv(B, T, H, 63, "bf16")
    ws = qi.new_workspace(qi.cached_workspace_size(B, H, 0, T, torch.bfloat16), cuda_device)
    oc = qi.attn_cached(qt.to(cuda_device), kt.to(cuda_device), vt.to(cuda_device), pt, kc, vc,
                        workspace=ws)
    assert qi.workspace_status(ws) == 0
    okc, ovc = O.prefix_cache(W.as_f64(kt), W.as_f64(vt), pos, 0)
    ref = O.attn_cached(W.as_f64(qt), W.as_f64(kt), W.as_f64(vt), pos, okc, ovc)
    assert_close(oc.cpu(), ref, torch.bfloat16, "empty Prefix")


def test_both_placements_agree(cuda_device, monkeypatch):
    """The same cached step with the keys rotated by the pre-pass (default)
    and by the attention kernel: equal up to the rounding of the rotated keys
    (fp32 table and one bf16 rounding against the fp16 query table)."""
    segs, B, H = CASES["ragged"]
    L, P, T = _sizes(segs)
    q, k, v = W.draw_qkv(B, L, H, 64, "bf16")
    g = gpu_full(segs, q, k, v, P)
    qt, kt, vt = (x.to(cuda_device) for x in W.draw_qkv(B, T, H, 65, "bf16"))
    pt = g["pos"][P:].contiguous().to(cuda_device)
    outs = []
    for mode in (None, "attention"):
        if mode is None:
            monkeypatch.delenv("QI21_K_ROTATION", raising=False)
        else:
            monkeypatch.setenv("QI21_K_ROTATION", mode)
        ws = qi.new_workspace(qi.cached_workspace_size(B, H, P, T, torch.bfloat16), cuda_device)
        outs.append(qi.attn_cached(qt, kt, vt, pt, g["kc"], g["vc"], workspace=ws).float().cpu())
        assert qi.workspace_status(ws) == 0
    assert (outs[0] - outs[1]).abs().max().item() < 2e-2
