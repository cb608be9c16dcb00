"""Seeded synthetic workloads shared by the tests, the bench and the smoke run.

This module holds data only: the five segment layouts (text length, image
grids and frame indices, heads, batch, dtype) and a seeded generator of the
Q/K/V inputs.  It contains none of the method's arithmetic, so both the CUDA
path and the float64 oracle may take their inputs from it.

Recipe (the same host arrays feed the oracle and the GPU):

* generator ``numpy.random.default_rng(seed)`` (PCG64);
* draw order Q, then K, then V, each ``standard_normal((B, L, H, 128))`` in
  float64, cast to float32, then to bf16 (round-to-nearest-even, via torch)
  for the bf16 workloads;
* seeds: tiny 0, t2i 1, edit3 2, maxref 3, hires 4; the max-reference loop's
  cached steps s = 2..8 draw fresh target Q/K/V with seed 3000 + s;
* the cached step of the other workloads reuses the target rows of the full
  step's Q/K/V, so its output must equal the full step's target rows.
"""

import numpy as np
import torch

HEAD_DIM = 128


def text(n):
    return {"kind": "text", "n": int(n)}


def image(H, W, frame):
    return {"kind": "image", "H": int(H), "W": int(W), "frame": int(frame)}


# Segment layouts of the five workloads: prompt text first, reference images
# next (frames 1..N), the target image (frame 0) last.
WORKLOADS = {
    "tiny": dict(dtype="f32", B=1, H=2, seed=0,
                 segments=[text(16), image(4, 4, 0)]),
    "t2i": dict(dtype="bf16", B=1, H=24, seed=1,
                segments=[text(256), image(64, 64, 0)]),
    "edit3": dict(dtype="bf16", B=1, H=24, seed=2,
                  segments=[text(512), image(64, 64, 1), image(64, 64, 2),
                            image(64, 64, 3), image(64, 64, 0)]),
    "maxref": dict(dtype="bf16", B=1, H=24, seed=3, cached_steps=7,
                   segments=[text(1024)] + [image(48, 48, f) for f in range(1, 11)]
                   + [image(64, 64, 0)]),
    "hires": dict(dtype="bf16", B=2, H=24, seed=4,
                  segments=[text(512), image(64, 64, 1), image(128, 128, 0)]),
    # the earlier Qwen-Image model's edit layout: [text | target | reference],
    # text positions after the images, no mask (full step only: nothing is
    # cacheable when the text attends the target)
    "orig": dict(dtype="bf16", B=1, H=24, seed=5, original=True,
                 segments=[text(256), image(64, 64, 0), image(64, 64, 1)]),
}

DESCRIPTIONS = {
    "tiny": "tiny fp32: B=1, 2 heads, text 16 + target 4x4 (L=32)",
    "t2i": "text-to-image 1024^2: B=1, 24 heads, text 256 + target 64x64 (L=4352)",
    "edit3": "edit with 3 references: B=1, 24 heads, text 512 + 3x(64x64) + target 64x64 (L=16896)",
    "maxref": "max-reference 8-step loop: B=1, 24 heads, text 1024 + 10x(48x48) + target 64x64 (L=28160)",
    "hires": "high-res 2048^2: B=2, 24 heads, text 512 + ref 64x64 + target 128x128 (L=20992)",
    "orig": "earlier-model edit: B=1, 24 heads, text 256 + target 64x64 + ref 64x64, no mask (L=8448)",
}


def seg_tokens(seg):
    return seg["n"] if seg["kind"] == "text" else seg["H"] * seg["W"]


def sizes(name_or_cfg):
    """(L, P, T): total tokens, prefix tokens, target tokens (target = last segment)."""
    cfg = WORKLOADS[name_or_cfg] if isinstance(name_or_cfg, str) else name_or_cfg
    counts = [seg_tokens(s) for s in cfg["segments"]]
    L = sum(counts)
    T = counts[-1]
    return L, L - T, T


def draw_qkv(B, L, H, seed, dtype):
    """Q, K, V as CPU torch tensors of ``dtype`` ("bf16" or "f32"), [B, L, H, 128]."""
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(3):
        x = rng.standard_normal((B, L, H, HEAD_DIM)).astype(np.float32)
        t = torch.from_numpy(x)
        out.append(t.to(torch.bfloat16) if dtype == "bf16" else t)
    return tuple(out)


def full_inputs(name):
    cfg = WORKLOADS[name]
    L, _, _ = sizes(name)
    return draw_qkv(cfg["B"], L, cfg["H"], cfg["seed"], cfg["dtype"])


def cached_inputs(name, step=2):
    """Target Q/K/V of a cached step.

    The max-reference loop draws them fresh per step (seed 3000 + step); the
    other workloads reuse the target rows of the full step's inputs.
    """
    cfg = WORKLOADS[name]
    L, P, T = sizes(name)
    if name == "maxref":
        return draw_qkv(cfg["B"], T, cfg["H"], 3000 + step, cfg["dtype"])
    q, k, v = full_inputs(name)
    return tuple(x[:, P:].contiguous() for x in (q, k, v))


# QK-RMSNorm inputs.  The pages publish no trained weights, so the two
# per-dimension weight vectors (queries, keys) are seeded synthetic values
# around 1; eps is the 1e-6 the pages print for the model's other RMSNorms.
QK_NORM_EPS = 1e-6


def qk_norm_weights(seed=7):
    """(w_q, w_k): float32 CPU tensors of 128 weights each, 1 + 0.25 * N(0, 1)."""
    rng = np.random.default_rng(seed)
    return tuple(torch.from_numpy((1.0 + 0.25 * rng.standard_normal(HEAD_DIM)).astype(np.float32))
                 for _ in range(2))


# The denoising loop's synthetic model (the pages publish no trained
# weights).  Widths: D = 128 * heads, a 3x wider SwiGLU hidden layer, C latent
# channels.  Weights N(0, 1/fan_in), norm weights 1 + 0.1 N(0, 1), biases
# 0.02 N(0, 1), the per-step embedding biases (the target's conditioning)
# 0.5 N(0, 1); latents and Prefix hidden states N(0, 1).  Sigmas
# linspace(1, 1/S, S) followed by 0.


def denoise_sigmas(steps):
    return [1.0 - i * (1.0 - 1.0 / steps) / max(1, steps - 1) for i in range(steps)] + [0.0]


def denoise_model(heads, channels, blocks, steps, seed, dtype="bf16"):
    """(params, draw) for the denoising loop: ``params`` as the oracle's
    ``denoise`` takes them (CPU torch tensors of ``dtype``); ``draw(B, P, T,
    seed)`` gives (x0 [B, T, C], prefix_h [B, P, D])."""
    rng = np.random.default_rng(seed)
    D, F, C = heads * HEAD_DIM, 3 * heads * HEAD_DIM, channels

    def t(a):
        x = torch.from_numpy(np.asarray(a, dtype=np.float32))
        return x.to(torch.bfloat16) if dtype == "bf16" else x

    def w(n, k):
        return t(rng.standard_normal((n, k)) / np.sqrt(k))

    def b(n, scale=0.02):
        return t(scale * rng.standard_normal(n))

    blk = []
    for _ in range(blocks):
        blk.append(dict(norm1=t(1 + 0.1 * rng.standard_normal(D)), w_qkv=w(3 * D, D), b_qkv=b(3 * D),
                        w_o=w(D, D), b_o=b(D), norm2=t(1 + 0.1 * rng.standard_normal(D)),
                        w_gu=w(2 * F, D), b_gu=b(2 * F), w_down=w(D, F), b_down=b(D)))
    params = dict(w_in=w(D, C), b_in=t(0.5 * rng.standard_normal((steps, D))), blocks=blk,
                  norm_out=t(1 + 0.1 * rng.standard_normal(D)), w_v=w(C, D), b_v=b(C))

    def draw(B, P, T, seed2):
        r = np.random.default_rng(seed2)
        return t(r.standard_normal((B, T, C))), t(r.standard_normal((B, P, D)))

    return params, draw


def as_f64(t):
    """float64 numpy copy of a (CPU) torch tensor, for the oracle."""
    return t.detach().to("cpu").to(torch.float64).numpy()
