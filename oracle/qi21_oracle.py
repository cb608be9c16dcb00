"""Float64 CPU oracle for the Qwen-Image-2.1 joint-attention hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg (and ``bench.py --impl reference``) may call it.  It shares no code with
the CUDA library: it is written from the pages' description of the method,
step by step, with no blocking, fusion or reordering beyond the plain
definitions.

What it computes (sources are the pages this build follows):

* ``positions`` -- the 3D axial position table and the block-causal visibility
  bound.  "3A - 3D Axial RoPE (16, 56, 56) & Zero-Centered Grid", section 1
  (Definition) and the glossary entry "zero-centred grid": text tokens advance
  frame/height/width together by +1; an image freezes its frame index and
  numbers rows and columns around (0, 0), height from -(H - H//2) to H//2 - 1
  (example H = 4 -> -2, -1, 0, 1), width likewise.  Token order inside an image
  is row-major with width fastest ("Qwen-Image-Edit close reading", section
  7.3, ``_compute_video_freqs``).  The mask: "Qwen-Image-2.1 architecture"
  overview, card 3C (text reads only what precedes it, tokens of one image see
  each other both ways) and the learning goals (the Prefix never attends the
  target); the target is appended last (card 2A).
* ``positions_original`` -- the earlier Qwen-Image model's table, a second
  workload for the same attention: images are numbered as above, text tokens
  continue after the images, f = h = w = max_vid_index + running text index
  with max_vid_index the largest max(H//2, W//2) over the images, and there
  is no mask (close reading, section 7.2: ``txt_freqs`` taken from
  ``max_vid_index`` on; section 6: ``is_causal=False``, text sees the images).
* ``rope_angles`` / ``rope`` -- axial rotary embedding: head_dim 128 split
  into bands (16, 56, 56) for (frame, height, width) (3A, section 1); per axis
  the angle of pair j is pos * theta^(-2j/d_axis) with theta = 10000 (close
  reading, section 7.1: per-axis ``outer(index, 1/theta^(2i/dim))`` turned into
  unit complex factors by ``torch.polar``), applied to adjacent pairs
  (2m, 2m+1) as a complex multiplication (close reading, section 6: RoPE on Q
  and K before attention).
* ``attention_head`` -- softmax(Q K^T / sqrt(128) + M) V with an explicit
  dense mask M (0 where key j < kv_end[i], -inf elsewhere); the scale is the
  SDPA default since the attention call passes none (close reading, section 6).
* ``prefix_cache`` / ``attn_cached`` -- the Prefix KV Cache: step 1 stores the
  rotated prefix K and the prefix V; later steps attend the target queries
  over [cached prefix K/V || fresh target K/V] with no mask, since the target
  sees everything (overview, card 6A and learning goals).

* ``rms_norm`` -- the QK-RMSNorm in front of RoPE: every head's 128-dim
  query and key vector of every token is divided by its root mean square (plus
  eps under the root) and multiplied by a learned per-dimension weight, one
  weight vector for queries and one for keys, before the rotation ("Qwen-Image-2.1"
  overview, card 4A; close reading, section 6: ``norm_q``/``norm_k`` are
  RMSNorm(head_dim = 128) applied before ``apply_rope``).  The pages print no eps
  for these two norms; callers pass it (the model's other RMSNorms use 1e-6).

* ``linear`` -- the projections around the attention: Y = X W^T + b with
  the nn.Linear weight layout W[N, K] (close reading, section 6: to_q, to_k,
  to_v make the joint Q, K, V from the hidden states and to_out maps the
  attention output back); in steps 2..N only the target tokens' rows are
  projected (overview, card 6A).

* ``silu`` / ``denoise`` -- the denoising loop around the attention: each
  step embeds the target latents, runs the stack of blocks (RMSNorm ->
  attention -> residual, RMSNorm -> SwiGLU with a 3x wider hidden layer ->
  residual; overview cards 4A and 5A), maps the target tokens to a velocity
  and takes the Euler step x <- x + (sigma_next - sigma) v (card 6B and the
  learning goals).  The Prefix tokens take no step-dependent input, so in
  the cached form step 1 runs every token and stores each block's Prefix
  K/V, and later steps run the target tokens only (card 6A); the full form
  recomputes everything at every step.  The pages' lab finds both equal to
  about 1e-16.

Inputs are arrays already cast to the GPU dtype (bf16 or fp32) by the seeded
input module; every function promotes them to float64 first.

Pins: every function here is pinned by ``tests/test_oracle_pins.py`` against
the pages' worked example, closed forms, invariants and library routines.
No function is "parity unpinned".
"""

import math

import numpy as np

HEAD_DIM = 128
AXES_DIM = (16, 56, 56)  # frame, height, width bands of one head (3A, section 1)
THETA = 10000.0


# ----------------------------------------------------------------------------
# a1: position table and visibility bound
# ----------------------------------------------------------------------------

def positions(segments):
    """Position table ``pos[L, 3]`` = (frame, height, width) and ``kv_end[L]``.

    ``segments`` is the sequence in order; each item is a dict
    ``{"kind": "text", "n": n}`` or
    ``{"kind": "image", "H": H, "W": W, "frame": f}``.

    Text: the three coordinates advance together by +1 per text token; the
    counter starts at 0 and counts text tokens only (3A, section 1).
    Image: the frame stays fixed over the whole image, the row r and column c
    (row-major, width fastest) map to h = r - (H - H//2), w = c - (W - W//2)
    (3A, section 1 and glossary).

    ``kv_end[i]`` is one past the last key token i may attend (block-causal
    mask, overview card 3C): a text token sees itself and everything before
    it; an image token sees everything before its image and its whole image.
    """
    pos = []
    kv_end = []
    text_counter = 0
    start = 0
    for seg in segments:
        if seg["kind"] == "text":
            n = int(seg["n"])
            for t in range(n):
                pos.append((text_counter, text_counter, text_counter))
                kv_end.append(start + t + 1)
                text_counter += 1
            start += n
        elif seg["kind"] == "image":
            H, W, frame = int(seg["H"]), int(seg["W"]), int(seg["frame"])
            end = start + H * W
            for r in range(H):
                for c in range(W):
                    pos.append((frame, r - (H - H // 2), c - (W - W // 2)))
                    kv_end.append(end)
            start = end
        else:
            raise ValueError("unknown segment kind %r" % (seg["kind"],))
    return (np.array(pos, dtype=np.int64).reshape(-1, 3),
            np.array(kv_end, dtype=np.int64))


def allowed_matrix(kv_end, n_keys):
    """Dense boolean mask: allowed[i, j] = j < kv_end[i]."""
    kv_end = np.asarray(kv_end, dtype=np.int64)
    return np.arange(n_keys)[None, :] < kv_end[:, None]


def positions_original(segments):
    """The earlier model's position table and (absent) mask.

    Image tokens get the same (frame, h, w) as in ``positions`` (close
    reading, section 7.3: negative table tail then positive table head, frame
    = the image's index).  Text tokens get f = h = w = max_vid_index + j for
    the j-th text token, where max_vid_index = max over the images of
    max(H//2, W//2) (section 7.2, ``scale_rope``): text continues beyond the
    images.  No mask: every token sees all L keys (section 6).
    """
    pos, _ = positions(segments)
    max_vid_index = 0
    for seg in segments:
        if seg["kind"] == "image":
            max_vid_index = max(max_vid_index, int(seg["H"]) // 2, int(seg["W"]) // 2)
    start = 0
    text_counter = 0
    for seg in segments:
        n = int(seg["n"]) if seg["kind"] == "text" else int(seg["H"]) * int(seg["W"])
        if seg["kind"] == "text":
            for t in range(n):
                v = max_vid_index + text_counter
                pos[start + t] = (v, v, v)
                text_counter += 1
        start += n
    kv_end = np.full(start, start, dtype=np.int32)
    return pos, kv_end


# ----------------------------------------------------------------------------
# a2-a4: axial rotary embedding
# ----------------------------------------------------------------------------

def rope_angles(pos):
    """Angles ``[L, 64]`` in float64: pair m of the head belongs to one band.

    Pairs 0..7 use the frame axis, 8..35 the height axis, 36..63 the width
    axis; inside band a of width d_a, pair j turns by pos_a * theta^(-2j/d_a).
    """
    pos = np.asarray(pos, dtype=np.int64)
    L = pos.shape[0]
    ang = np.empty((L, HEAD_DIM // 2), dtype=np.float64)
    m = 0
    for axis, d in enumerate(AXES_DIM):
        for j in range(d // 2):
            omega = THETA ** (-2.0 * j / d)
            ang[:, m] = pos[:, axis].astype(np.float64) * omega
            m += 1
    assert m == HEAD_DIM // 2
    return ang


def rope(x, pos):
    """Rotate ``x[L, 128]`` (one head) by the axial angles of ``pos[L, 3]``.

    Dims (2m, 2m+1) form a complex number x0 + i*x1 that is multiplied by
    exp(i*phi_m): (x0 cos - x1 sin, x0 sin + x1 cos).
    """
    x = np.asarray(x, dtype=np.float64)
    ang = rope_angles(pos)
    c = np.cos(ang)
    s = np.sin(ang)
    x0 = x[:, 0::2]
    x1 = x[:, 1::2]
    out = np.empty_like(x)
    out[:, 0::2] = x0 * c - x1 * s
    out[:, 1::2] = x0 * s + x1 * c
    return out


# ----------------------------------------------------------------------------
# QK-RMSNorm (applied to Q and K before the rotation)
# ----------------------------------------------------------------------------

def rms_norm(x, weight, eps):
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) * weight (head_dim
    128 for the QK norm, the model width for the block norms)."""
    x = np.asarray(x, dtype=np.float64)
    weight = np.asarray(weight, dtype=np.float64)
    assert weight.shape == (x.shape[-1],)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * weight


# ----------------------------------------------------------------------------
# a5-a8: masked softmax attention
# ----------------------------------------------------------------------------

def attention_head(q_rot, k_rot, v, kv_end=None, chunk=512):
    """softmax(Q K^T / sqrt(128) + M) V for one (batch, head).

    ``q_rot[R,128]`` are the (already rotated) query rows to compute,
    ``k_rot[Lk,128]`` the rotated keys and ``v[Lk,128]`` the values.
    ``kv_end[R]`` gives the mask of those rows, M[i, j] = 0 if j < kv_end[i]
    else -inf; ``None`` means no mask.  The mask is built as an explicit dense
    matrix for each chunk of rows.
    """
    q_rot = np.asarray(q_rot, dtype=np.float64)
    k_rot = np.asarray(k_rot, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    R = q_rot.shape[0]
    Lk = k_rot.shape[0]
    scale = 1.0 / math.sqrt(HEAD_DIM)
    out = np.empty((R, HEAD_DIM), dtype=np.float64)
    for c0 in range(0, R, chunk):
        c1 = min(R, c0 + chunk)
        S = (q_rot[c0:c1] @ k_rot.T) * scale
        if kv_end is not None:
            kv = np.asarray(kv_end, dtype=np.int64)[c0:c1]
            M = np.where(np.arange(Lk)[None, :] < kv[:, None], 0.0, -np.inf)
            S = S + M
        S = S - S.max(axis=1, keepdims=True)
        E = np.exp(S)
        out[c0:c1] = (E @ v) / E.sum(axis=1, keepdims=True)
    return out


def attn_full(q, k, v, pos, kv_end, heads=None, rows=None, batches=None):
    """Full block-causal step for ``q, k, v[B, L, H, 128]``.

    Returns ``o[len(batches), len(rows), len(heads), 128]`` in float64
    (defaults: all batches, rows and heads).
    """
    B, L, H, D = q.shape
    assert D == HEAD_DIM
    heads = range(H) if heads is None else heads
    batches = range(B) if batches is None else batches
    rows = np.arange(L) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.empty((len(batches), rows.shape[0], len(heads), D), dtype=np.float64)
    for bi, b in enumerate(batches):
        for hi, h in enumerate(heads):
            k_rot = rope(k[b, :, h, :], pos)
            q_rot = rope(q[b, rows, h, :], np.asarray(pos)[rows])
            out[bi, :, hi, :] = attention_head(q_rot, k_rot, v[b, :, h, :],
                                               np.asarray(kv_end)[rows])
    return out


# ----------------------------------------------------------------------------
# a9: prefix KV cache and the target-only step
# ----------------------------------------------------------------------------

def prefix_cache(k, v, pos, P, heads=None, batches=None):
    """Step-1 store: rotated prefix K and prefix V, laid out ``[B, H, P, 128]``."""
    B, L, H, D = k.shape
    heads = range(H) if heads is None else heads
    batches = range(B) if batches is None else batches
    pos = np.asarray(pos)
    kc = np.empty((len(batches), len(heads), P, D), dtype=np.float64)
    vc = np.empty((len(batches), len(heads), P, D), dtype=np.float64)
    for bi, b in enumerate(batches):
        for hi, h in enumerate(heads):
            kc[bi, hi] = rope(k[b, :P, h, :], pos[:P])
            vc[bi, hi] = np.asarray(v[b, :P, h, :], dtype=np.float64)
    return kc, vc


def attn_cached(q_t, k_t, v_t, pos_t, k_cache, v_cache, heads=None, rows=None, batches=None):
    """Target-only step: target queries over [cached prefix || target] keys.

    ``q_t, k_t, v_t[B, T, H, 128]``; ``k_cache, v_cache[B, H, P, 128]`` (the
    cache holds rotated K); no mask.  ``heads``/``batches`` index both the
    target tensors and the cache (the cache must cover them).
    """
    B, T, H, D = q_t.shape
    heads = range(H) if heads is None else heads
    batches = range(B) if batches is None else batches
    rows = np.arange(T) if rows is None else np.asarray(rows, dtype=np.int64)
    pos_t = np.asarray(pos_t)
    out = np.empty((len(batches), rows.shape[0], len(heads), D), dtype=np.float64)
    for bi, b in enumerate(batches):
        for hi, h in enumerate(heads):
            keys = np.concatenate([np.asarray(k_cache[b, h], dtype=np.float64),
                                   rope(k_t[b, :, h, :], pos_t)], axis=0)
            vals = np.concatenate([np.asarray(v_cache[b, h], dtype=np.float64),
                                   np.asarray(v_t[b, :, h, :], dtype=np.float64)], axis=0)
            q_rot = rope(q_t[b, rows, h, :], pos_t[rows])
            out[bi, :, hi, :] = attention_head(q_rot, keys, vals, None)
    return out


# ----------------------------------------------------------------------------
# projections (Q/K/V in, attention output out)
# ----------------------------------------------------------------------------

def linear(x, w, bias=None):
    """Y = X W^T (+ b) for ``x[..., K]``, ``w[N, K]``, ``bias[N]``; float64."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    y = x @ w.T
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)
    return y


# ----------------------------------------------------------------------------
# the denoising loop: blocks of attention + SwiGLU, Euler steps
# ----------------------------------------------------------------------------

def silu(x):
    """x * sigmoid(x)."""
    x = np.asarray(x, dtype=np.float64)
    return x / (1.0 + np.exp(-x))


def _split(y, parts):
    n = y.shape[-1] // parts
    return [y[..., i * n:(i + 1) * n] for i in range(parts)]


def block_attention(h, blk, eps, attend):
    """Attention half of a block (overview card 4A): h + (attend(q, k, v) W_o^T + b_o),
    with q, k, v the three thirds of RMSNorm(h; norm1) W_qkv^T + b_qkv, each
    split into 128-wide heads."""
    B, L, D = h.shape
    a = rms_norm(h, blk["norm1"], eps)
    q, k, v = (t.reshape(B, L, D // HEAD_DIM, HEAD_DIM) for t in _split(linear(a, blk["w_qkv"], blk["b_qkv"]), 3))
    o = attend(q, k, v)
    return h + linear(o.reshape(B, L, D), blk["w_o"], blk["b_o"])


def block_ffn(h, blk, eps):
    """Feed-forward half of a block (card 5A, SwiGLU): h + (silu(g) * u) W_down^T
    + b_down, with the gate g first and the up branch u second in
    [g | u] = RMSNorm(h; norm2) W_gu^T + b_gu."""
    a = rms_norm(h, blk["norm2"], eps)
    g, u = _split(linear(a, blk["w_gu"], blk["b_gu"]), 2)
    return h + linear(silu(g) * u, blk["w_down"], blk["b_down"])


def block(h, blk, eps, attend):
    """One block: the attention half, then the feed-forward half (cards 4A, 5A)."""
    return block_ffn(block_attention(h, blk, eps, attend), blk, eps)


def embed(x, params, step):
    """Target latents to hidden states: x W_in^T + b_in[step] (card 1A: the
    latent patches enter the DiT through a linear map; the per-step bias
    stands for the step's conditioning of the target tokens)."""
    return linear(x, params["w_in"], params["b_in"][step])


def velocity(h_t, params, eps):
    """Velocity head (card 6B): RMSNorm(h_t; norm_out) W_v^T + b_v on the
    target tokens."""
    return linear(rms_norm(h_t, params["norm_out"], eps), params["w_v"], params["b_v"])


def denoise(x0, prefix_h, params, segments, sigmas, cached=True, eps=1e-6):
    """Euler denoising of the target latents ``x0[B, T, C]`` over
    ``len(sigmas) - 1`` steps.

    ``prefix_h[B, P, D]`` are the Prefix tokens' hidden states (fixed inputs);
    ``params`` holds ``w_in[D, C]``, ``b_in[S, D]`` (one embedding bias per step:
    the step's conditioning of the target tokens), ``blocks`` (list of dicts
    norm1, w_qkv, b_qkv, w_o, b_o, norm2, w_gu, b_gu, w_down, b_down),
    ``norm_out``, ``w_v[C, D]``, ``b_v``.  ``segments`` fix positions and the
    block-causal mask (target last).  Returns x after the last step.
    """
    pos, kv_end = positions(segments)
    pos = np.asarray(pos)
    P = prefix_h.shape[1]
    x = np.asarray(x0, dtype=np.float64)
    prefix_h = np.asarray(prefix_h, dtype=np.float64)
    caches = [None] * len(params["blocks"])
    for step in range(len(sigmas) - 1):
        h_t = embed(x, params, step)
        if step == 0 or not cached:
            h = np.concatenate([prefix_h, h_t], axis=1)
            for i, blk in enumerate(params["blocks"]):
                def attend(q, k, v, i=i):
                    if cached:
                        caches[i] = prefix_cache(k, v, pos, P)
                    return attn_full(q, k, v, pos, kv_end)
                h = block(h, blk, eps, attend)
            h_t = h[:, P:]
        else:
            h = h_t
            for i, blk in enumerate(params["blocks"]):
                attend = lambda q, k, v, i=i: attn_cached(q, k, v, pos[P:], caches[i][0], caches[i][1])
                h = block(h, blk, eps, attend)
            h_t = h
        x = x + (sigmas[step + 1] - sigmas[step]) * velocity(h_t, params, eps)
    return x


# ----------------------------------------------------------------------------
# measurement helper
# ----------------------------------------------------------------------------

def allowed_pairs(kv_end):
    """Number of allowed (query, key) pairs of the full step for one head."""
    return int(np.sum(np.asarray(kv_end, dtype=np.int64)))
