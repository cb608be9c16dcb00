"""Pins of the float64 oracle against what the pages and the mathematics fix.

Each ``check_*`` takes the oracle module (or a stand-in with one function
replaced) so that ``test_mutants_are_caught`` can plant a plausible mistake in
the oracle and show that at least one pin fails.  Nothing here calls the CUDA
library.
"""

import math
import os
import types

import numpy as np
import pytest
import torch

import oracle as ORACLE
from oracle import qi21_oracle as OM
from diffusion_transformer_joint_axial_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


def _img_rows(O, H, Wd, frame=0, text_before=0):
    segs = ([W.text(text_before)] if text_before else []) + [W.image(H, Wd, frame)]
    pos, _ = O.positions(segs)
    return pos[text_before:].reshape(H, Wd, 3)


# ---------------------------------------------------------------- positions --

def check_page_example_h4(O):
    """3A section 1: H = 4 gives height indices (-2, -1, 0, 1)."""
    (row,) = _golden_lines("centring_h4.txt")
    H = int(row[0])
    expect = [int(x) for x in row[1:]]
    for Wd in (1, 4, 7):
        grid = _img_rows(O, H, Wd)
        assert list(grid[:, 0, 1]) == expect
        # the same rule numbers the width axis
        gridT = _img_rows(O, Wd, H)
        assert list(gridT[0, :, 2]) == expect


def check_centring_neg_pos_tables(O):
    """Close reading 7.3: the centred axis is the last H - H//2 entries of the
    negative table [-N..-1] followed by the first H//2 entries of [0..N-1]."""
    N = 64
    neg = -np.arange(N)[::-1] - 1  # -N, ..., -1
    posv = np.arange(N)
    for H in range(1, 10):
        for Wd in range(1, 10):
            grid = _img_rows(O, H, Wd, frame=3)
            exp_h = np.concatenate([neg[N - (H - H // 2):], posv[:H // 2]])
            exp_w = np.concatenate([neg[N - (Wd - Wd // 2):], posv[:Wd // 2]])
            # row-major, width fastest: broadcast the axes like view/expand and flatten
            hh = np.broadcast_to(exp_h[:, None], (H, Wd))
            ww = np.broadcast_to(exp_w[None, :], (H, Wd))
            assert np.array_equal(grid[:, :, 1], hh)
            assert np.array_equal(grid[:, :, 2], ww)
            assert np.all(grid[:, :, 0] == 3)


def check_text_and_frames(O):
    """3A section 1: text advances all three axes by +1 from 0; an image's
    frame is frozen at its own index over the whole image."""
    segs = [W.text(10), W.image(3, 5, 2), W.image(2, 2, 0)]
    pos, kv_end = O.positions(segs)
    assert pos.shape == (10 + 15 + 4, 3)
    assert np.array_equal(pos[:10], np.repeat(np.arange(10)[:, None], 3, axis=1))
    assert np.all(pos[10:25, 0] == 2) and np.all(pos[25:, 0] == 0)


def check_prompt_length_invariance(O):
    """3A section 4: the same image behind 10 or 30 text tokens gets the same
    coordinates."""
    a = _img_rows(O, 6, 8, frame=0, text_before=10)
    b = _img_rows(O, 6, 8, frame=0, text_before=30)
    assert np.array_equal(a, b)


def check_block_causal_rule(O):
    """Overview card 3C + learning goals, restated at segment level: a text
    token reads itself and what precedes it; an image token reads every earlier
    segment and its own image, never a later segment."""
    segs = [W.text(3), W.image(2, 2, 1), W.text(2), W.image(2, 3, 0)]
    sizes = [W.seg_tokens(s) for s in segs]
    seg_of = np.concatenate([np.full(n, i) for i, n in enumerate(sizes)])
    L = len(seg_of)
    brute = np.zeros((L, L), dtype=bool)
    for i in range(L):
        for j in range(L):
            si, sj = seg_of[i], seg_of[j]
            if segs[si]["kind"] == "text":
                brute[i, j] = j <= i
            else:
                brute[i, j] = sj <= si
    _, kv_end = O.positions(segs)
    assert np.array_equal(O.allowed_matrix(kv_end, L), brute)


def check_prefix_never_sees_target(O):
    """Learning goals of the overview: the Prefix never attends the target;
    the target (appended last) attends everything."""
    for name in ("t2i", "edit3", "maxref", "hires"):
        pos, kv_end = O.positions(W.WORKLOADS[name]["segments"])
        L, P, T = W.sizes(name)
        assert len(kv_end) == L
        assert kv_end[:P].max() <= P
        assert np.all(kv_end[P:] == L)


# --------------------------------------------------------------------- rope --

def check_bands(O):
    rows = {r[0]: [int(x) for x in r[1:]] for r in _golden_lines("bands.txt")}
    assert tuple(O.AXES_DIM) == tuple(rows["bands"])
    assert sum(O.AXES_DIM) == rows["head_dim"][0] == O.HEAD_DIM
    assert [d // 2 for d in O.AXES_DIM] == rows["pairs"]


def check_rope_vs_polar(O):
    """Close reading 7.1: per-axis tables polar(1, outer(index, 1/theta^(2i/dim)))
    concatenated over the axes, applied as a complex product to adjacent pairs."""
    rng = np.random.default_rng(11)
    L = 37
    pos = np.stack([rng.integers(-20, 20, L), rng.integers(-70, 70, L),
                    rng.integers(-300, 300, L)], axis=1)
    x = rng.standard_normal((L, 128))
    factors = []
    for axis, dim in enumerate((16, 56, 56)):
        inv = 1.0 / torch.pow(torch.tensor(10000.0, dtype=torch.float64),
                              torch.arange(0, dim, 2, dtype=torch.float64) / dim)
        ang = torch.outer(torch.tensor(pos[:, axis], dtype=torch.float64), inv)
        factors.append(torch.polar(torch.ones_like(ang), ang))
    f = torch.cat(factors, dim=1)  # (L, 64) complex
    xc = torch.view_as_complex(torch.tensor(x).reshape(L, 64, 2))
    ref = torch.view_as_real(xc * f).reshape(L, 128).numpy()
    got = O.rope(x, pos)
    assert np.max(np.abs(got - ref)) < 1e-12


def check_rope_invariants(O):
    """3A section 1: rotation, and the product of two rotated vectors depends
    only on the difference of positions (per axis)."""
    rng = np.random.default_rng(5)
    L = 24
    pos = rng.integers(-50, 50, (L, 3))
    q = rng.standard_normal((L, 128))
    k = rng.standard_normal((L, 128))
    # norm preservation
    assert np.allclose(np.linalg.norm(O.rope(q, pos), axis=1), np.linalg.norm(q, axis=1), atol=1e-12)
    # identity at position 0
    assert np.array_equal(O.rope(q, np.zeros_like(pos)), q)
    # composition rot(rot(x, p), p') = rot(x, p + p')
    pos2 = rng.integers(-50, 50, (L, 3))
    assert np.allclose(O.rope(O.rope(q, pos), pos2), O.rope(q, pos + pos2), atol=1e-10)
    # relative position: <rot(q,p+c), rot(k,p'+c)> = <rot(q,p), rot(k,p')>
    posk = rng.integers(-50, 50, (L, 3))
    c = np.array([7, -13, 29])
    lhs = O.rope(q, pos + c) @ O.rope(k, posk + c).T
    rhs = O.rope(q, pos) @ O.rope(k, posk).T
    assert np.allclose(lhs, rhs, atol=1e-9)


# ---------------------------------------------------------------- attention --

def _tiny_problem(seed=3):
    segs = [W.text(4), W.image(2, 3, 1), W.image(2, 2, 0)]
    rng = np.random.default_rng(seed)
    L = 14
    q, k, v = (rng.standard_normal((1, L, 2, 128)) for _ in range(3))
    return segs, q, k, v


def check_attention_brute_force(O):
    """Explicit loops over (i, j) with math.exp on a 14-token sequence."""
    segs, q, k, v = _tiny_problem()
    pos, kv_end = O.positions(segs)
    got = O.attn_full(q, k, v, pos, kv_end)
    L = q.shape[1]
    for h in range(2):
        qr = O.rope(q[0, :, h], pos)
        kr = O.rope(k[0, :, h], pos)
        for i in range(L):
            logits = [sum(qr[i, d] * kr[j, d] for d in range(128)) / math.sqrt(128)
                      for j in range(int(kv_end[i]))]
            mx = max(logits)
            w = [math.exp(s - mx) for s in logits]
            tot = sum(w)
            o = [sum(w[j] * v[0, j, h, d] for j in range(len(w))) / tot for d in range(128)]
            assert np.max(np.abs(np.array(o) - got[0, i, h])) < 1e-12


def check_attention_closed_forms(O):
    segs, q, k, v = _tiny_problem()
    pos, kv_end = O.positions(segs)
    # Q = 0: every logit is 0, so O_i is the mean of the allowed V_j
    got = O.attn_full(np.zeros_like(q), k, v, pos, kv_end)
    for i in range(q.shape[1]):
        assert np.allclose(got[0, i], v[0, :kv_end[i]].mean(axis=0), atol=1e-13)
    # constant V along keys: O = V
    vc = np.broadcast_to(v[:, :1], v.shape).copy()
    assert np.allclose(O.attn_full(q, k, vc, pos, kv_end), vc, atol=1e-13)
    # the first text token sees only itself: O_0 = V_0 exactly
    assert np.array_equal(O.attn_full(q, k, v, pos, kv_end)[0, 0], v[0, 0])


def check_attention_vs_sdpa(O):
    """With no mask and every position 0 the method is plain softmax attention:
    torch's scaled_dot_product_attention in float64 must agree."""
    rng = np.random.default_rng(9)
    L = 40
    q, k, v = (rng.standard_normal((1, L, 3, 128)) for _ in range(3))
    pos = np.zeros((L, 3), dtype=np.int64)
    kv_end = np.full(L, L)
    got = O.attn_full(q, k, v, pos, kv_end)
    tq, tk, tv = (torch.tensor(x).permute(0, 2, 1, 3) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv).permute(0, 2, 1, 3).numpy()
    assert np.max(np.abs(got - ref)) < 1e-12
    # and with the block-causal mask handed to SDPA as a boolean mask
    segs, q2, k2, v2 = _tiny_problem(4)
    pos2, kv2 = O.positions(segs)
    got2 = O.attn_full(q2, k2, v2, np.zeros_like(pos2), kv2)
    allowed = torch.tensor(O.allowed_matrix(kv2, q2.shape[1]))
    tq, tk, tv = (torch.tensor(x).permute(0, 2, 1, 3) for x in (q2, k2, v2))
    ref2 = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=allowed)
    assert np.max(np.abs(got2 - ref2.permute(0, 2, 1, 3).numpy())) < 1e-12


def check_prefix_invariance(O):
    """Learning goals: the Prefix never attends the target, so perturbing the
    target's Q/K/V leaves every prefix output unchanged."""
    segs, q, k, v = _tiny_problem()
    pos, kv_end = O.positions(segs)
    P = 10
    base = O.attn_full(q, k, v, pos, kv_end)
    rng = np.random.default_rng(1)
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    for x in (q2, k2, v2):
        x[:, P:] += rng.standard_normal(x[:, P:].shape)
    pert = O.attn_full(q2, k2, v2, pos, kv_end)
    assert np.array_equal(base[:, :P], pert[:, :P])
    assert not np.allclose(base[:, P:], pert[:, P:])


def check_cached_equals_full(O):
    """Overview (lab note): reusing the Prefix K/V reproduces the full
    recomputation to float64 rounding."""
    segs, q, k, v = _tiny_problem()
    pos, kv_end = O.positions(segs)
    P = 10
    full = O.attn_full(q, k, v, pos, kv_end)
    kc, vc = O.prefix_cache(k, v, pos, P)
    assert np.array_equal(vc, np.transpose(v[:, :P], (0, 2, 1, 3)))
    cached = O.attn_cached(q[:, P:], k[:, P:], v[:, P:], pos[P:], kc, vc)
    assert np.max(np.abs(cached - full[:, P:])) < 1e-13


# ----------------------------------------------------------------- QK-norm --

def check_rms_norm_vs_torch(O):
    """Card 4A / close reading 6: norm_q and norm_k are RMSNorm(128) with a
    weight; against torch's own rms_norm in float64."""
    rng = np.random.default_rng(11)
    x = rng.standard_normal((3, 5, 128)) * rng.uniform(0.05, 20.0, (3, 5, 1))
    w = 1.0 + 0.25 * rng.standard_normal(128)
    for eps in (1e-6, 0.5):
        ref = torch.nn.functional.rms_norm(torch.tensor(x), (128,), torch.tensor(w), eps).numpy()
        assert np.max(np.abs(O.rms_norm(x, w, eps) - ref)) < 1e-12


def check_rms_norm_closed_forms(O):
    """Constant rows, unit mean square, scale invariance, per-dimension weight."""
    ones = np.ones(128)
    for c in (3.0, -0.25):
        y = O.rms_norm(np.full((1, 128), c), ones, 1e-6)
        assert np.allclose(y, c / math.sqrt(c * c + 1e-6), rtol=1e-15, atol=0)
    rng = np.random.default_rng(12)
    x = rng.standard_normal((6, 128)) * 4.0
    y = O.rms_norm(x, ones, 0.0)
    assert np.allclose(np.mean(y * y, axis=-1), 1.0, rtol=1e-14, atol=0)
    assert np.allclose(O.rms_norm(7.5 * x, ones, 0.0), y, rtol=1e-14, atol=1e-15)
    w = rng.uniform(0.5, 2.0, 128)
    assert np.allclose(O.rms_norm(x, w, 1e-6), O.rms_norm(x, ones, 1e-6) * w, rtol=1e-15, atol=0)


# ------------------------------------------------- earlier model's positions --

def check_original_text_offset(O):
    """Close reading 7.2: the earlier model's text continues after the images,
    from max over images of max(H//2, W//2), +1 per text token on all axes;
    images keep the centred grid of 7.3; no mask (section 6)."""
    segs = [W.text(3), W.image(4, 6, 0), W.image(10, 2, 1)]  # max(2, 3, 5, 1) = 5
    pos, kv = O.positions_original(segs)
    assert [tuple(int(x) for x in p) for p in pos[:3]] == [(5, 5, 5), (6, 6, 6), (7, 7, 7)]
    assert np.array_equal(pos[3:], O.positions(segs)[0][3:])
    assert np.all(np.asarray(kv) == len(pos))
    img = np.asarray(pos[3:])
    assert pos[0][1] > img[:, 1].max() and pos[0][2] > img[:, 2].max()
    # the earlier model's edit layout: [text | target 64x64 | reference 64x64] -> text from 32
    pos2, _ = O.positions_original([W.text(2), W.image(64, 64, 0), W.image(64, 64, 1)])
    assert [tuple(int(x) for x in p) for p in pos2[:2]] == [(32, 32, 32), (33, 33, 33)]


# ------------------------------------------------------------- projections --

def check_linear_brute_force(O):
    """Y[i, n] = sum_k X[i, k] W[n, k] + b[n], by explicit loops on a tiny case."""
    rng = np.random.default_rng(13)
    x, w, b = rng.standard_normal((3, 5)), rng.standard_normal((4, 5)), rng.standard_normal(4)
    want = np.array([[sum(x[i, k] * w[n, k] for k in range(5)) + b[n] for n in range(4)] for i in range(3)])
    assert np.max(np.abs(O.linear(x, w, b) - want)) < 1e-13
    assert np.max(np.abs(O.linear(x, w) - (want - b))) < 1e-13


def check_linear_special_cases(O):
    """Identity weights reproduce X; zero input gives the bias; batched rows."""
    rng = np.random.default_rng(14)
    x = rng.standard_normal((2, 6, 8))
    assert np.array_equal(O.linear(x, np.eye(8)), x)
    b = rng.standard_normal(3)
    assert np.array_equal(O.linear(np.zeros((4, 8)), rng.standard_normal((3, 8)), b), np.tile(b, (4, 1)))


# ----------------------------------------------------------- denoising loop --

def _f64_params(params):
    conv = lambda v: W.as_f64(v) if isinstance(v, torch.Tensor) else v
    out = {k: conv(v) for k, v in params.items() if k != "blocks"}
    out["blocks"] = [{k: conv(v) for k, v in b.items()} for b in params["blocks"]]
    return out


def _tiny_denoise(steps=3):
    segs = [W.text(5), W.image(3, 3, 1), W.image(4, 4, 0)]
    params, draw = W.denoise_model(heads=1, channels=16, blocks=2, steps=steps, seed=21, dtype="f32")
    x0, ph = draw(1, 14, 16, 22)
    return segs, _f64_params(params), W.as_f64(x0), W.as_f64(ph), W.denoise_sigmas(steps)


def check_silu_vs_torch(O):
    x = np.linspace(-30, 30, 1001)
    ref = torch.nn.functional.silu(torch.tensor(x)).numpy()
    assert np.max(np.abs(O.silu(x) - ref)) < 1e-13


def check_denoise_cache_reuse(O):
    """Overview (lab note, card 6A): reusing the Prefix K/V over the Euler steps
    reproduces full recomputation to float64 rounding (the lab reports 1e-16)."""
    segs, params, x0, ph, sig = _tiny_denoise()
    xc = O.denoise(x0, ph, params, segs, sig, cached=True)
    xf = O.denoise(x0, ph, params, segs, sig, cached=False)
    assert np.max(np.abs(xc - xf)) < 1e-12
    assert np.max(np.abs(xc - x0)) > 0.1  # the steps did move the latents


def check_denoise_euler_closed_form(O):
    """Blocks with zero weights pass h through; a constant velocity c then
    gives x_S = x_0 + (sigma_S - sigma_0) c = x_0 - c (card 6B)."""
    segs, params, x0, ph, sig = _tiny_denoise()
    for blk in params["blocks"]:
        for k in blk:
            if not k.startswith("norm"):
                blk[k] = np.zeros_like(blk[k])
    params["w_v"] = np.zeros_like(params["w_v"])
    c = np.linspace(-1, 1, params["b_v"].shape[0])
    params["b_v"] = c
    x = O.denoise(x0, ph, params, segs, sig, cached=True)
    assert np.max(np.abs(x - (x0 - c))) < 1e-14


# Pins of the loop's stages, each against a closed form that fixes its
# composition (overview cards 4A, 5A, 6B): with identity-structured weights
# every stage reduces to a few scalar formulas, evaluated here with plain
# Python loops and math.exp / math.sqrt.

def _rms_scalar(row, w, eps):
    r = 1.0 / math.sqrt(sum(x * x for x in row) / len(row) + eps)
    return [x * r * wi for x, wi in zip(row, w)]


def _silu_scalar(x):
    return x / (1.0 + math.exp(-x))


def _single_key_block(D=128, seed=31):
    rng = np.random.default_rng(seed)
    h = rng.standard_normal((1, 1, D)) * 3.0 + 0.5
    blk = dict(norm1=1 + 0.1 * rng.standard_normal(D),
               w_qkv=np.concatenate([rng.standard_normal((2 * D, D)), np.eye(D)]),  # value third = I
               b_qkv=np.zeros(3 * D), w_o=np.eye(D), b_o=0.05 * rng.standard_normal(D),
               norm2=1 + 0.1 * rng.standard_normal(D),
               w_gu=np.concatenate([np.eye(D), 2.0 * np.eye(D)]),  # gate = a, up = 2a
               b_gu=np.zeros(2 * D), w_down=np.eye(D), b_down=0.05 * rng.standard_normal(D))
    return h, blk


def _attend_first_text_token(O):
    pos, kv = O.positions([W.text(1)])
    return lambda q, k, v: O.attn_full(q, k, v, pos, kv)


def _expect_attention_half(h, blk, eps=1e-6):
    """Token 0 of the text sees only itself (card 3C), so its attention
    weights are [1] and the output is its own V = RMSNorm(h; norm1);
    W_o = I: h + RMSNorm(h; norm1) + b_o."""
    a = _rms_scalar(h, blk["norm1"], eps)
    return [x + y + b for x, y, b in zip(h, a, blk["b_o"])]


def _expect_ffn_half(h, blk, eps=1e-6):
    """[g | u] = [a | 2a] with a = RMSNorm(h; norm2), W_down = I:
    h + silu(a) * 2a + b_down (card 5A: the gate passes through SiLU)."""
    a = _rms_scalar(h, blk["norm2"], eps)
    return [x + _silu_scalar(ai) * 2.0 * ai + b for x, ai, b in zip(h, a, blk["b_down"])]


def check_block_attention_single_key(O):
    h, blk = _single_key_block()
    got = O.block_attention(h, blk, 1e-6, _attend_first_text_token(O))
    exp = np.array(_expect_attention_half(list(h[0, 0]), blk))
    assert np.max(np.abs(got[0, 0] - exp)) < 1e-12


def check_block_ffn_closed_form(O):
    h, blk = _single_key_block(seed=32)
    got = O.block_ffn(h, blk, 1e-6)
    exp = np.array(_expect_ffn_half(list(h[0, 0]), blk))
    assert np.max(np.abs(got[0, 0] - exp)) < 1e-12


def check_block_order(O):
    """A block is the attention half, then the feed-forward half on its
    result (cards 4A then 5A)."""
    h, blk = _single_key_block(seed=33)
    got = O.block(h, blk, 1e-6, _attend_first_text_token(O))
    exp = np.array(_expect_ffn_half(_expect_attention_half(list(h[0, 0]), blk), blk))
    assert np.max(np.abs(got[0, 0] - exp)) < 1e-12


def check_velocity_closed_form(O):
    """Card 6B: the velocity is the RMS-normalised target state through W_v.
    A row of constant c normalises to c / sqrt(c^2 + eps) in every dim; with
    W_v = I the velocity is that times norm_out, plus b_v."""
    rng = np.random.default_rng(34)
    D, eps = 128, 1e-6
    c = np.array([0.5, -3.0, 7.0])
    h = np.repeat(c[None, :, None], D, axis=2)
    params = dict(norm_out=1 + 0.1 * rng.standard_normal(D), w_v=np.eye(D), b_v=0.1 * rng.standard_normal(D))
    got = O.velocity(h, params, eps)
    for t, ct in enumerate(c):
        exp = [ct / math.sqrt(ct * ct + eps) * w + b for w, b in zip(params["norm_out"], params["b_v"])]
        assert np.max(np.abs(got[0, t] - np.array(exp))) < 1e-13


def check_denoise_explicit_one_step(O):
    """One Euler step of a one-block model over a text token and a 1x1
    target, every stage written as explicit scalar loops: embedding (card
    1A), RMSNorm -> Q/K/V -> block-causal softmax attention -> W_o ->
    residual (card 4A; text token 0 sees itself, the target sees both),
    RMSNorm -> SwiGLU -> W_down -> residual (card 5A), velocity from the
    RMS-normalised target state and x1 = x0 + (sigma1 - sigma0) v (card
    6B).  The rotation uses the oracle's own rope (pinned above by the
    close reading's polar construction)."""
    rng = np.random.default_rng(35)
    D, C, F, eps = 128, 4, 384, 1e-6
    r = lambda *s, sc=1.0: sc * rng.standard_normal(s)
    blk = dict(norm1=1 + 0.1 * r(D), w_qkv=r(3 * D, D, sc=D ** -0.5), b_qkv=r(3 * D, sc=0.1),
               w_o=r(D, D, sc=D ** -0.5), b_o=r(D, sc=0.1), norm2=1 + 0.1 * r(D),
               w_gu=r(2 * F, D, sc=D ** -0.5), b_gu=r(2 * F, sc=0.1), w_down=r(D, F, sc=F ** -0.5),
               b_down=r(D, sc=0.1))
    params = dict(w_in=r(D, C, sc=C ** -0.5), b_in=r(1, D, sc=0.5), blocks=[blk], norm_out=1 + 0.1 * r(D),
                  w_v=r(C, D, sc=D ** -0.5), b_v=r(C, sc=0.1))
    x0, ph = r(1, 1, C), r(1, 1, D)
    segs = [W.text(1), W.image(1, 1, 0)]
    sig = [1.0, 0.4]
    got = O.denoise(x0, ph, params, segs, sig, cached=True, eps=eps)

    mv = lambda w, x, b: [sum(w[n][kk] * x[kk] for kk in range(len(x))) + b[n] for n in range(len(w))]
    h = [list(ph[0, 0]), mv(params["w_in"], list(x0[0, 0]), params["b_in"][0])]
    qkv = [mv(blk["w_qkv"], _rms_scalar(row, blk["norm1"], eps), blk["b_qkv"]) for row in h]
    pos = np.array([[0, 0, 0], [0, -1, -1]])  # text 0; 1x1 image centred at -(1 - 0) = -1
    q = O.rope(np.array([t[:D] for t in qkv]), pos)
    k = O.rope(np.array([t[D:2 * D] for t in qkv]), pos)
    v = [t[2 * D:] for t in qkv]
    h1 = []
    for i in range(2):
        s = [sum(q[i][d] * k[j][d] for d in range(D)) / math.sqrt(D) for j in range(i + 1)]
        m = max(s)
        e = [math.exp(x - m) for x in s]
        o = [sum(e[j] * v[j][d] for j in range(i + 1)) / sum(e) for d in range(D)]
        h1.append([a + b for a, b in zip(h[i], mv(blk["w_o"], o, blk["b_o"]))])
    h2 = []
    for row in h1:
        gu = mv(blk["w_gu"], _rms_scalar(row, blk["norm2"], eps), blk["b_gu"])
        mid = [_silu_scalar(gu[f]) * gu[F + f] for f in range(F)]
        h2.append([a + b for a, b in zip(row, mv(blk["w_down"], mid, blk["b_down"]))])
    vel = mv(params["w_v"], _rms_scalar(h2[1], params["norm_out"], eps), params["b_v"])
    exp = [x + (sig[1] - sig[0]) * vv for x, vv in zip(x0[0, 0], vel)]
    assert np.max(np.abs(got[0, 0] - np.array(exp))) < 1e-11


CHECKS = [check_page_example_h4, check_centring_neg_pos_tables, check_text_and_frames,
          check_prompt_length_invariance, check_block_causal_rule, check_prefix_never_sees_target,
          check_bands, check_rope_vs_polar, check_rope_invariants, check_attention_brute_force,
          check_attention_closed_forms, check_attention_vs_sdpa, check_prefix_invariance,
          check_cached_equals_full, check_rms_norm_vs_torch, check_rms_norm_closed_forms,
          check_linear_brute_force, check_linear_special_cases, check_original_text_offset,
          check_silu_vs_torch, check_denoise_cache_reuse, check_denoise_euler_closed_form,
          check_block_attention_single_key, check_block_ffn_closed_form, check_block_order,
          check_velocity_closed_form, check_denoise_explicit_one_step]


@pytest.mark.parametrize("check", CHECKS, ids=lambda f: f.__name__)
def test_oracle_pin(check):
    check(ORACLE)


# ------------------------------------------------------------------ mutants --

def _mutant(**repl):
    ns = types.SimpleNamespace(**{k: getattr(OM, k) for k in dir(OM) if not k.startswith("_")})
    for k, fn in repl.items():
        setattr(ns, k, fn)
    # rebind the helpers that call each other so the mutation propagates
    def attn_full(q, k, v, pos, kv_end, heads=None, rows=None, batches=None):
        B, L, H, D = q.shape
        out = np.empty((B, L, H, D))
        for b in range(B):
            for h in range(H):
                out[b, :, h] = ns.attention_head(ns.rope(q[b, :, h], pos), ns.rope(k[b, :, h], pos),
                                                 v[b, :, h], kv_end)
        return out
    if "attn_full" not in repl:
        ns.attn_full = attn_full
    return ns


def _rope_sign_flipped(x, pos):
    out = OM.rope(x, pos)
    ref = np.asarray(x, dtype=np.float64)
    return 2 * ref * np.cos(OM.rope_angles(pos)).repeat(2, axis=1) - out


def _angles_global_denominator(pos):
    pos = np.asarray(pos)
    ang = np.empty((pos.shape[0], 64))
    m = 0
    for axis, d in enumerate(OM.AXES_DIM):
        for j in range(d // 2):
            ang[:, m] = pos[:, axis] * OM.THETA ** (-2.0 * j / 128)
            m += 1
    return ang


def _rope_with(angles_fn):
    def rope(x, pos):
        x = np.asarray(x, dtype=np.float64)
        a = angles_fn(pos)
        c, s = np.cos(a), np.sin(a)
        out = np.empty_like(x)
        out[:, 0::2] = x[:, 0::2] * c - x[:, 1::2] * s
        out[:, 1::2] = x[:, 0::2] * s + x[:, 1::2] * c
        return out
    return rope


def _positions_floor_centre(segs):
    pos, kv_end = OM.positions(segs)
    start = 0
    for s in segs:
        n = W.seg_tokens(s)
        if s["kind"] == "image":
            H, Wd = s["H"], s["W"]
            r = np.arange(n) // Wd
            c = np.arange(n) % Wd
            pos[start:start + n, 1] = r - H // 2
            pos[start:start + n, 2] = c - Wd // 2
        start += n
    return pos, kv_end


def _positions_text_exclusive(segs):
    pos, kv_end = OM.positions(segs)
    start = 0
    for s in segs:
        n = W.seg_tokens(s)
        if s["kind"] == "text":
            kv_end[start:start + n] -= 1
        start += n
    return pos, kv_end


def _head_no_scale(q_rot, k_rot, v, kv_end=None, chunk=512):
    return OM.attention_head(q_rot * math.sqrt(128), k_rot, v, kv_end, chunk)


def _head_v_transposed(q_rot, k_rot, v, kv_end=None, chunk=512):
    return OM.attention_head(q_rot, k_rot, v[::-1], kv_end, chunk)


def _rms_sum_not_mean(x, weight, eps):
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps) * weight


def _rms_eps_outside(x, weight, eps):
    x = np.asarray(x, dtype=np.float64)
    return x / (np.sqrt(np.mean(x * x, axis=-1, keepdims=True)) + eps) * weight


def _rms_no_weight(x, weight, eps):
    return OM.rms_norm(x, np.ones(128), eps)


def _linear_untransposed(x, w, bias=None):
    x, w = np.asarray(x, dtype=np.float64), np.asarray(w, dtype=np.float64)
    y = x @ w.reshape(w.shape[1], w.shape[0]) if w.shape[0] != w.shape[1] else x @ w
    return y if bias is None else y + bias


def _linear_no_bias(x, w, bias=None):
    return OM.linear(x, w)


def _original_offset_unhalved(segments):
    """Text offset max(H, W) (the earlier model's scale_rope=False branch)."""
    pos, kv = OM.positions_original(segments)
    imgs = [s for s in segments if s["kind"] == "image"]
    shift = max(max(s["H"], s["W"]) for s in imgs) - max(max(s["H"] // 2, s["W"] // 2) for s in imgs)
    start = 0
    for seg in segments:
        n = W.seg_tokens(seg)
        if seg["kind"] == "text":
            pos[start:start + n] += shift
        start += n
    return pos, kv


def _original_from_zero(segments):
    _, kv = OM.positions_original(segments)
    return OM.positions(segments)[0], kv


def _silu_as_sigmoid(x):
    return 1.0 / (1.0 + np.exp(-np.asarray(x, dtype=np.float64)))


def _denoise_step_sign(x0, prefix_h, params, segments, sigmas, cached=True, eps=1e-6):
    return OM.denoise(x0, prefix_h, params, segments, [-s for s in sigmas], cached, eps)


def _denoise_stale_target(x0, prefix_h, params, segments, sigmas, cached=True, eps=1e-6):
    """A cached loop that drifts from the full recomputation: its later steps
    only go half way."""
    if not cached:
        return OM.denoise(x0, prefix_h, params, segments, sigmas, False, eps)
    x = OM.denoise(x0, prefix_h, params, segments, sigmas[:2], True, eps)
    return x + (OM.denoise(x, prefix_h, params, segments, sigmas[1:], False, eps) - x) * 0.5


_ORIG_BLOCK_ATTENTION, _ORIG_BLOCK_FFN = OM.block_attention, OM.block_ffn


def _ffn_gate_up_swapped(h, blk, eps):
    a = OM.rms_norm(h, blk["norm2"], eps)
    g, u = OM._split(OM.linear(a, blk["w_gu"], blk["b_gu"]), 2)
    return h + OM.linear(OM.silu(u) * g, blk["w_down"], blk["b_down"])


def _ffn_norm2_dropped(h, blk, eps):
    g, u = OM._split(OM.linear(h, blk["w_gu"], blk["b_gu"]), 2)
    return h + OM.linear(OM.silu(g) * u, blk["w_down"], blk["b_down"])


def _attn_residual_dropped(h, blk, eps, attend):
    B, L, D = h.shape
    a = OM.rms_norm(h, blk["norm1"], eps)
    q, k, v = (t.reshape(B, L, D // 128, 128) for t in OM._split(OM.linear(a, blk["w_qkv"], blk["b_qkv"]), 3))
    return OM.linear(attend(q, k, v).reshape(B, L, D), blk["w_o"], blk["b_o"])


def _block_order_swapped(h, blk, eps, attend):
    return _ORIG_BLOCK_ATTENTION(_ORIG_BLOCK_FFN(h, blk, eps), blk, eps, attend)


def _velocity_norm_dropped(h_t, params, eps):
    return OM.linear(h_t, params["w_v"], params["b_v"])


def _embed_bias_dropped(x, params, step):
    return OM.linear(x, params["w_in"])


# Stages that ``denoise`` looks up in the oracle module at call time: these
# mutants are also planted in the module itself while the pins run, so that
# the loop uses them.
STAGE_MUTANTS = {"ffn_gate_up_swapped", "ffn_norm2_dropped", "attn_residual_dropped",
                 "block_order_swapped", "velocity_norm_dropped", "embed_bias_dropped"}

MUTANTS = {
    "rope_sign": dict(rope=_rope_sign_flipped),
    "band_denominator_128": dict(rope=_rope_with(_angles_global_denominator),
                                 rope_angles=_angles_global_denominator),
    "centre_floor": dict(positions=_positions_floor_centre),
    "text_mask_exclusive": dict(positions=_positions_text_exclusive),
    "missing_scale": dict(attention_head=_head_no_scale),
    "value_order": dict(attention_head=_head_v_transposed),
    "rms_sum_not_mean": dict(rms_norm=_rms_sum_not_mean),
    "rms_eps_outside_root": dict(rms_norm=_rms_eps_outside),
    "rms_weight_dropped": dict(rms_norm=_rms_no_weight),
    "linear_weight_untransposed": dict(linear=_linear_untransposed),
    "linear_bias_dropped": dict(linear=_linear_no_bias),
    "original_offset_unhalved": dict(positions_original=_original_offset_unhalved),
    "original_text_from_zero": dict(positions_original=_original_from_zero),
    "silu_as_sigmoid": dict(silu=_silu_as_sigmoid),
    "euler_step_sign": dict(denoise=_denoise_step_sign),
    "cache_not_reused_faithfully": dict(denoise=_denoise_stale_target),
    "ffn_gate_up_swapped": dict(block_ffn=_ffn_gate_up_swapped),
    "ffn_norm2_dropped": dict(block_ffn=_ffn_norm2_dropped),
    "attn_residual_dropped": dict(block_attention=_attn_residual_dropped),
    "block_order_swapped": dict(block=_block_order_swapped),
    "velocity_norm_dropped": dict(velocity=_velocity_norm_dropped),
    "embed_bias_dropped": dict(embed=_embed_bias_dropped),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutants_are_caught(name, monkeypatch):
    ns = _mutant(**MUTANTS[name])
    if name in STAGE_MUTANTS:
        for k, fn in MUTANTS[name].items():
            monkeypatch.setattr(OM, k, fn)
    failed = []
    for check in CHECKS:
        try:
            with np.errstate(all="ignore"):
                check(ns)
        except (AssertionError, ValueError, IndexError, FloatingPointError):
            failed.append(check.__name__)
    assert failed, "planted mistake %s passed every pin" % name
