"""The tensor-core projection Y = X W^T (+ b) against the float64 oracle, and
one target-only attention layer of a cached step built from it: fused Q/K/V
projection of the target tokens -> cached attention -> output projection."""

import numpy as np
import pytest
import torch

import diffusion_transformer_joint_axial_b200 as qi
import oracle as O
from diffusion_transformer_joint_axial_b200 import workloads as W

from parity import assert_close, check_status

pytestmark = pytest.mark.gpu


def _draw(M, N, K, seed, bias=True):
    """Seeded bf16 inputs: X ~ N(0, 1), W ~ N(0, 1/K), b ~ N(0, 0.1^2)."""
    rng = np.random.default_rng(seed)
    bf = lambda a: torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16)
    x = bf(rng.standard_normal((M, K)))
    w = bf(rng.standard_normal((N, K)) / np.sqrt(K))
    b = bf(0.1 * rng.standard_normal(N)) if bias else None
    return x, w, b


def _check(got, x, w, b, rows=None, what=""):
    """|gpu - ref| <= 2^-8 |ref| + 2^-16 sum_k |x w|: one bf16 rounding of the
    result plus a generous bound on the fp32 accumulation order."""
    xf = W.as_f64(x) if rows is None else W.as_f64(x)[rows]
    wf, bf = W.as_f64(w), (None if b is None else W.as_f64(b))
    ref = O.linear(xf, wf, bf)
    g = got.to(torch.float64).cpu().numpy() if isinstance(got, torch.Tensor) else got
    if rows is not None:
        g = g[rows]
    bound = 2.0 ** -8 * np.abs(ref) + 2.0 ** -16 * (np.abs(xf) @ np.abs(wf).T)
    err = np.abs(g - ref)
    assert np.all(np.isfinite(g)), what
    assert np.all(err <= bound), "%s: worst excess %.3g" % (what, float(np.max(err - bound)))


@pytest.mark.parametrize("M,N,K,n_out,bias", [
    (1, 8, 8, 1, False),          # smallest
    (200, 408, 200, 3, True),     # ragged M, N (3 x 136) and K (not a multiple of 64)
    (256, 512, 128, 1, True),     # exact tiles
    (130, 264, 72, 1, False),     # one row and one column group past a tile
    (300, 1024, 512, 4, True),    # four segments
    (1000, 20480, 136, 2, True),  # many column tiles, ragged in M and K
])
def test_linear_shapes(cuda_device, M, N, K, n_out, bias):
    x, w, b = _draw(M, N, K, seed=M + N + K, bias=bias)
    ws = qi.new_workspace(256, cuda_device)
    outs = qi.linear(x.to(cuda_device), w.to(cuda_device), None if b is None else b.to(cuda_device),
                     n_out=n_out, workspace=ws)
    check_status(ws)
    got = torch.cat([o.cpu() for o in outs], dim=-1)
    _check(got, x, w, b, what="linear %dx%dx%d/%d" % (M, N, K, n_out))


@pytest.mark.parametrize("M,F,K", [(200, 384, 136), (4096, 1536, 512)])
def test_linear_swiglu(cuda_device, M, F, K):
    """silu(x W_g^T + b_g) * (x W_u^T + b_u) from one launch, weights given to
    the GPU in the alternating-block layout, against the float64 oracle with
    the plain [gate; up] layout."""
    x, w, b = _draw(M, 2 * F, K, seed=M + F)
    dev = cuda_device
    got = qi.linear_swiglu(x.to(dev), qi.interleave_gate_up(w).to(dev), qi.interleave_gate_up(b).to(dev)).cpu()
    xf, wf, bf = W.as_f64(x), W.as_f64(w), W.as_f64(b)
    gu = O.linear(xf, wf, bf)
    g, u = gu[:, :F], gu[:, F:]
    ref = O.silu(g) * u
    # one bf16 rounding of the result plus the fp32 accumulation of g and u
    # carried through silu(g) * u (|d silu / dg| <= 1.1)
    acc = 2.0 ** -16 * (np.abs(xf) @ np.abs(wf).T)
    bound = 2.0 ** -8 * np.abs(ref) + 1.1 * np.abs(u) * acc[:, :F] + np.abs(O.silu(g)) * acc[:, F:]
    err = np.abs(got.double().numpy() - ref)
    assert np.all(err <= bound + 1e-6), float(np.max(err - bound))


def test_linear_target_qkv_full_size_sampled(cuda_device):
    """The t2i cached step's fused Q/K/V projection: 4096 target tokens,
    hidden 3072 = 24 heads x 128, N = 3 x 3072; sampled rows against the oracle."""
    M, K, N = 4096, 3072, 3 * 3072
    x, w, b = _draw(M, N, K, seed=99)
    outs = qi.linear(x.to(cuda_device), w.to(cuda_device), b.to(cuda_device), n_out=3)
    torch.cuda.synchronize()
    got = torch.cat([o.cpu() for o in outs], dim=-1)
    rows = np.array(sorted(set([0, 1, 127, 128, M - 1] + list(np.random.default_rng(5).integers(0, M, 27)))))
    _check(got, x, w, b, rows=rows, what="t2i target Q/K/V projection")


def test_cached_layer_projection_attention_projection(cuda_device):
    """x_t -> [Q|K|V] = x_t W_qkv^T + b -> cached attention over the prefix
    cache -> O W_o^T + b_o, against the same chain in float64."""
    segs = [W.text(64), W.image(8, 8, 1), W.image(12, 12, 0)]
    L = sum(W.seg_tokens(s) for s in segs)
    T = W.seg_tokens(segs[-1])
    P = L - T
    B, H = 1, 2
    D = H * 128
    dev = cuda_device
    x, w_qkv, b_qkv = _draw(B * L, 3 * D, D, seed=41)
    _, w_o, b_o = _draw(1, D, D, seed=42)
    x = x.reshape(B, L, D)
    # step 1: project every token, full step with cache store
    q, k, v = (t.reshape(B, L, H, 128) for t in qi.linear(x.to(dev), w_qkv.to(dev), b_qkv.to(dev), n_out=3))
    pos, kv_end = qi.rope_positions(segs, dev)
    kc, vc = qi.alloc_cache(B, H, P, torch.bfloat16, dev)
    qi.attn_full(q, k, v, pos, kv_end, P, kc, vc)
    # a later step: only the target rows are projected
    xt = x[:, P:].contiguous()
    qt, kt, vt = (t.reshape(B, T, H, 128) for t in qi.linear(xt.to(dev), w_qkv.to(dev), b_qkv.to(dev), n_out=3))
    ot = qi.attn_cached(qt, kt, vt, pos[P:].clone(), kc, vc)
    (y,) = qi.linear(ot.reshape(B, T, D), w_o.to(dev), b_o.to(dev))
    torch.cuda.synchronize()

    xf = W.as_f64(x)
    qkv = O.linear(xf, W.as_f64(w_qkv), W.as_f64(b_qkv))
    qf, kf, vf = (qkv[..., i * D:(i + 1) * D].reshape(B, L, H, 128) for i in range(3))
    opos, okv = O.positions(segs)
    okc, ovc = O.prefix_cache(kf, vf, opos, P)
    ref_o = O.attn_cached(qf[:, P:], kf[:, P:], vf[:, P:], opos[P:], okc, ovc)
    assert_close(ot, ref_o, torch.bfloat16, "cached attention on projected inputs")
    ref_y = O.linear(ref_o.reshape(B, T, D), W.as_f64(w_o), W.as_f64(b_o))
    assert_close(y, ref_y, torch.bfloat16, "output projection of the cached step")
