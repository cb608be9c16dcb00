"""Cached steps whose last, partial wave of units is split into key-range
pieces (each piece's O / l and row max / row sum go to the workspace; the
last piece of a unit to finish merges them).  Shapes are chosen so that the
launcher's cost model splits into 2, 3 and 4 pieces on a 148-SM B200, with a
ragged last query-tile pair (its second tile empty, so its unit goes whole),
fewer units than SMs, and two batches.  Every target row of every head is
compared with the float64 oracle."""

import numpy as np
import pytest
import torch

import diffusion_transformer_joint_axial_b200 as qi
import oracle as O
from diffusion_transformer_joint_axial_b200 import workloads as W

from parity import assert_close, gpu_cached, gpu_full

pytestmark = pytest.mark.gpu

T_, I_ = W.text, W.image

# name: (segments, B, H); the target is the last segment
CASES = {
    # 72 units, 24 key tiles: 2 pieces each
    "k2_prefix_2304": ([T_(256), I_(32, 32, 1), I_(32, 32, 2), I_(24, 32, 0)], 1, 24),
    # 80 units, 48 key tiles: 3 pieces each
    "k3_prefix_5120": ([T_(256), I_(32, 32, 1), I_(32, 32, 2), I_(32, 32, 3), I_(32, 32, 4),
                        I_(24, 32, 5), I_(32, 32, 0)], 1, 20),
    # 8 units, 41 key tiles: 4 pieces each; the last pair's second tile is empty
    "k4_ragged_pair": ([T_(224), I_(64, 64, 1), I_(25, 32, 0)], 1, 2),
    # two batches, 18 units, 40 key tiles: 4 pieces each, ragged last pair
    "k4_two_batches": ([T_(300), I_(64, 64, 1), I_(20, 32, 0)], 2, 3),
}


def split_pieces(U, N, sms=148, slots=512):
    """The launcher's choice, restated: the r = U mod sms units of the last
    wave go out as k pieces when ceil(r k / sms) (N / k + 3.5) + 9 < N + 3.5
    (key tiles; 3.5 per item start, 9 for the merge left at the end and the
    slowdown beside it)."""
    r = U % sms
    best, k_best = float(N) + 3.5, 1
    for k in range(2, 5):
        if N < k or r * k > min(slots, 4 * U):
            break
        cost = -(-r * k // sms) * (N / k + 3.5) + 9.0
        if cost < best:
            best, k_best = cost, k
    return k_best


@pytest.mark.parametrize("name", sorted(CASES))
def test_tail_split_cached_matches_oracle(cuda_device, name):
    segs, B, H = CASES[name]
    L = sum(W.seg_tokens(s) for s in segs)
    T = W.seg_tokens(segs[-1])
    P = L - T
    U = B * H * (-(-T // 256))
    N = -(-P // 128) + -(-T // 128)
    expect = int(name[1])
    if torch.cuda.get_device_properties(cuda_device).multi_processor_count == 148:
        assert split_pieces(U, N) == expect
    q, k, v = W.draw_qkv(B, L, H, 40 + expect, "bf16")
    g = gpu_full(segs, q, k, v, P)
    pos, kv_end = O.positions(segs)
    okc, ovc = O.prefix_cache(W.as_f64(k), W.as_f64(v), pos, P)
    for seed in (7, 8):
        qt, kt, vt = W.draw_qkv(B, T, H, seed, "bf16")
        oc = gpu_cached(qt, kt, vt, g["pos"][P:].contiguous(), g["kc"], g["vc"])
        ref = O.attn_cached(W.as_f64(qt), W.as_f64(kt), W.as_f64(vt), pos[P:], okc, ovc)
        assert_close(oc, ref, torch.bfloat16, "%s cached, inputs %d" % (name, seed))


def test_tail_split_repeated_calls_on_one_workspace(cuda_device):
    """The arrival counters live in the workspace and are reset by each call's
    pre-pass: three calls in a row on one workspace give the same output."""
    segs, B, H = CASES["k3_prefix_5120"]
    L = sum(W.seg_tokens(s) for s in segs)
    T = W.seg_tokens(segs[-1])
    P = L - T
    q, k, v = W.draw_qkv(B, L, H, 3, "bf16")
    g = gpu_full(segs, q, k, v, P)
    qt, kt, vt = (x.to(cuda_device) for x in W.draw_qkv(B, T, H, 9, "bf16"))
    pt = g["pos"][P:].contiguous().to(cuda_device)
    ws = qi.new_workspace(qi.cached_workspace_size(B, H, P, T, torch.bfloat16), cuda_device)
    outs = [qi.attn_cached(qt, kt, vt, pt, g["kc"], g["vc"], workspace=ws).cpu() for _ in range(3)]
    assert qi.workspace_status(ws) == 0
    for o in outs[1:]:
        assert torch.equal(o, outs[0])
    pos, _ = O.positions(segs)
    okc, ovc = O.prefix_cache(W.as_f64(k), W.as_f64(v), pos, P)
    ref = O.attn_cached(W.as_f64(qt.cpu()), W.as_f64(kt.cpu()), W.as_f64(vt.cpu()), pos[P:], okc, ovc)
    assert_close(outs[0], ref, torch.bfloat16, "repeated calls")
    assert np.isfinite(outs[0].float().numpy()).all()


def _cached_vs_oracle(cuda_device, segs, B, H, seed, ws_bytes=None):
    L = sum(W.seg_tokens(s) for s in segs)
    T = W.seg_tokens(segs[-1])
    P = L - T
    q, k, v = W.draw_qkv(B, L, H, seed, "bf16")
    pos, _ = O.positions(segs)
    if P > 0:
        g = gpu_full(segs, q, k, v, P)
        kc, vc, pt = g["kc"], g["vc"], g["pos"][P:].contiguous()
    else:
        kc = vc = torch.zeros((B, H, 0, 128), dtype=torch.bfloat16, device=cuda_device)
        pt, _ = qi.rope_positions(segs, cuda_device)
    okc, ovc = O.prefix_cache(W.as_f64(k), W.as_f64(v), pos, P)
    qt, kt, vt = W.draw_qkv(B, T, H, seed + 1, "bf16")
    need = qi.cached_workspace_size(B, H, P, T, torch.bfloat16) if ws_bytes is None else ws_bytes
    ws = qi.new_workspace(need, cuda_device)
    oc = qi.attn_cached(qt.to(cuda_device), kt.to(cuda_device), vt.to(cuda_device), pt.to(cuda_device), kc, vc,
                        workspace=ws)
    assert qi.workspace_status(ws) == 0
    ref = O.attn_cached(W.as_f64(qt), W.as_f64(kt), W.as_f64(vt), pos[P:], okc, ovc)
    assert_close(oc.cpu(), ref, torch.bfloat16, "cached")
    return oc.cpu()


def test_tail_split_empty_prefix(cuda_device):
    """P = 0: the keys are the target's own (48 units of 24 key tiles: 3 pieces)."""
    assert split_pieces(48, 24) == 3
    _cached_vs_oracle(cuda_device, [I_(48, 64, 0)], 1, 4, 51)


def test_tail_split_partial_last_tile(cuda_device):
    """T = 1000: the last query-tile pair has a full first tile and a second
    tile of 104 rows; its unit is split like the others (12 units of 24 key
    tiles: 4 pieces), and the padding rows are never stored."""
    assert split_pieces(12, 24) == 4
    _cached_vs_oracle(cuda_device, [T_(2000), I_(25, 40, 0)], 1, 3, 53)


def test_tail_split_needs_no_scratch(cuda_device):
    """A workspace holding only the position table and the rotated keys (no
    split scratch) still runs, unsplit, with the same result up to rounding."""
    segs = CASES["k3_prefix_5120"][0]
    B, H = 1, 20
    T = W.seg_tokens(segs[-1])
    rnd = lambda x: (x + 255) // 256 * 256
    minimum = rnd(rnd(256 + T * 64 * 8) + B * H * T * 128 * 2)
    assert minimum < qi.cached_workspace_size(B, H, 5120, T, torch.bfloat16)
    small = _cached_vs_oracle(cuda_device, segs, B, H, 55, ws_bytes=minimum)
    split = _cached_vs_oracle(cuda_device, segs, B, H, 55)
    assert (small.float() - split.float()).abs().max().item() < 2e-2
