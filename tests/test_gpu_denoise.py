"""The denoising loop around the attention (blocks of RMSNorm -> attention ->
residual, RMSNorm -> SwiGLU -> residual; velocity head; Euler steps), run on
libqi21's kernels: the cached loop against the float64 oracle, the cached
loop against the full recomputation on the GPU (the cache-reuse check of the
overview's lab), and a CUDA-graph replay against the eager run."""

import numpy as np
import pytest
import torch

import diffusion_transformer_joint_axial_b200 as qi
import oracle as O
from diffusion_transformer_joint_axial_b200 import workloads as W

pytestmark = pytest.mark.gpu

SEGS = [W.text(40), W.image(6, 6, 1), W.image(8, 8, 0)]
HEADS, CH, BLOCKS, STEPS = 2, 16, 2, 3


def _model(cuda_device, cached):
    sig = W.denoise_sigmas(STEPS)
    params, draw = W.denoise_model(HEADS, CH, BLOCKS, STEPS, seed=31)
    L = sum(W.seg_tokens(s) for s in SEGS)
    T = W.seg_tokens(SEGS[-1])
    x0, ph = draw(1, L - T, T, 32)
    m = qi.denoise.DenoiseModel(SEGS, HEADS, CH, BLOCKS, STEPS, sig, device=cuda_device, cached=cached)
    m.load(params, x0, ph)
    return m, params, x0, ph, sig


def _f64(params):
    conv = lambda v: W.as_f64(v) if isinstance(v, torch.Tensor) else v
    out = {k: conv(v) for k, v in params.items() if k != "blocks"}
    out["blocks"] = [{k: conv(v) for k, v in b.items()} for b in params["blocks"]]
    return out


def test_denoise_cached_against_oracle_and_full(cuda_device):
    m, params, x0, ph, sig = _model(cuda_device, cached=True)
    m.run()
    m.check()
    got = W.as_f64(m.x.cpu())
    ref = O.denoise(W.as_f64(x0), W.as_f64(ph), _f64(params), SEGS, sig, cached=True)
    moved = np.abs(ref - W.as_f64(x0)).mean()
    err = np.abs(got - ref)
    print("denoise vs oracle: max %.3g mean %.3g (latents moved %.3g on average)" % (err.max(), err.mean(), moved))
    # bf16 storage between every kernel (about 30 roundings along a path) on
    # O(1) values: a relative error of a few 2^-9 per rounding, random in sign
    assert err.max() <= 6e-2 and err.mean() <= 1e-2

    full, *_ = _model(cuda_device, cached=False)
    full.run()
    full.check()
    diff = np.abs(W.as_f64(full.x.cpu()) - got)
    print("cached vs full recomputation on the GPU: max %.3g mean %.3g" % (diff.max(), diff.mean()))
    # the same bound: the two runs round in different places (key tiles split
    # at the prefix/target boundary in the cached steps, one sequence in the
    # full ones), so they differ by the same bf16 noise as each does from the
    # oracle; in float64 the oracle's two forms agree to 1e-12 (its pins)
    assert diff.max() <= 6e-2 and diff.mean() <= 1e-2


def test_denoise_graph_replay_bit_identical(cuda_device):
    m, *_ = _model(cuda_device, cached=True)
    x0 = m.x.clone()
    m.run()
    m.check()
    eager = m.x.clone()
    m.x.copy_(x0)
    m.capture()
    m.x.copy_(x0)
    m.replay()
    m.check()
    assert torch.equal(m.x, eager)


def test_denoise_cache_reuse_bit_exact_on_tile_aligned_prefix(cuda_device):
    """With a Prefix of whole 128-key tiles the cached steps sum the same key
    tiles in the same order as the full recomputation, and every other kernel
    works row by row: the cached loop equals the recomputation bit for bit
    (the GPU counterpart of the lab's 1e-16)."""
    segs = [W.text(64), W.image(8, 8, 1), W.image(8, 12, 0)]  # P = 128
    sig = W.denoise_sigmas(STEPS)
    params, draw = W.denoise_model(HEADS, CH, BLOCKS, STEPS, seed=33)
    x0, ph = draw(1, 128, 96, 34)
    out = []
    for cached in (True, False):
        m = qi.denoise.DenoiseModel(segs, HEADS, CH, BLOCKS, STEPS, sig, device=cuda_device, cached=cached)
        m.load(params, x0, ph)
        m.run()
        m.check()
        out.append(m.x.cpu())
    assert torch.equal(out[0], out[1])
    assert (out[0].float() - x0.float()).abs().mean() > 0.1


def test_denoise_tail_split_against_oracle(cuda_device):
    """The loop on a layout whose cached steps split their work units into 4
    key-range pieces (2 heads x 3 query-tile pairs of 16 key tiles): against
    the float64 oracle with the bounds above."""
    segs = [W.text(256), W.image(32, 32, 1), W.image(24, 32, 0)]
    sig = W.denoise_sigmas(STEPS)
    params, draw = W.denoise_model(HEADS, CH, BLOCKS, STEPS, seed=41)
    L = sum(W.seg_tokens(s) for s in segs)
    T = W.seg_tokens(segs[-1])
    x0, ph = draw(1, L - T, T, 42)
    m = qi.denoise.DenoiseModel(segs, HEADS, CH, BLOCKS, STEPS, sig, device=cuda_device, cached=True)
    m.load(params, x0, ph)
    m.run()
    m.check()
    got = W.as_f64(m.x.cpu())
    ref = O.denoise(W.as_f64(x0), W.as_f64(ph), _f64(params), segs, sig, cached=True)
    err = np.abs(got - ref)
    print("split layout, denoise vs oracle: max %.3g mean %.3g" % (err.max(), err.mean()))
    assert err.max() <= 6e-2 and err.mean() <= 1e-2
