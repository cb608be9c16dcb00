"""The denoising loop of one attention layer (step 1 full + cache store,
steps 2..N cached on fresh target Q/K/V), run eagerly and replayed as a CUDA
graph: every step against the float64 oracle, graph replays bit-identical to
the eager calls, and replays reading the buffers' current contents."""

import pytest
import torch

import diffusion_transformer_joint_axial_b200 as qi
import oracle as O
from diffusion_transformer_joint_axial_b200 import workloads as W

from parity import assert_close

SEGS = [W.text(64), W.image(8, 8, 1), W.image(16, 12, 0)]
B, H, STEPS = 1, 2, 4


def _inputs(seed):
    L, T = sum(W.seg_tokens(s) for s in SEGS), W.seg_tokens(SEGS[-1])
    full = W.draw_qkv(B, L, H, seed, "bf16")
    targets = [W.draw_qkv(B, T, H, seed * 100 + s, "bf16") for s in range(2, STEPS + 1)]
    return full, targets


def _outputs(loop):
    torch.cuda.synchronize()
    return [loop.out_full.cpu()] + [o.cpu() for o in loop.out_target]


def test_loop_without_cuda_fails_loudly():
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present")
    with pytest.raises(qi.QI21Error):
        qi.DenoiseLoop(SEGS, B, H, STEPS)


@pytest.mark.gpu
def test_loop_eager_matches_oracle_and_graph_replays_bit_identical(cuda_device):
    loop = qi.DenoiseLoop(SEGS, B, H, STEPS, device=cuda_device)
    (q, k, v), targets = _inputs(5)
    loop.load(q, k, v, targets)
    loop.run()
    loop.check()
    eager = _outputs(loop)

    opos, okv = O.positions(SEGS)
    P = loop.P
    qf, kf, vf = W.as_f64(q), W.as_f64(k), W.as_f64(v)
    assert_close(eager[0], O.attn_full(qf, kf, vf, opos, okv), torch.bfloat16, "loop step 1")
    okc, ovc = O.prefix_cache(kf, vf, opos, P)
    for s, (tq, tk, tv) in enumerate(targets, start=2):
        ref = O.attn_cached(W.as_f64(tq), W.as_f64(tk), W.as_f64(tv), opos[P:], okc, ovc)
        assert_close(eager[s - 1], ref, torch.bfloat16, "loop step %d" % s)

    loop.capture()
    for o in [loop.out_full] + loop.out_target:
        o.fill_(float("nan"))
    loop.replay()
    loop.check()
    for s, (a, b) in enumerate(zip(eager, _outputs(loop)), start=1):
        assert torch.equal(a, b), "graph replay differs from the eager call at step %d" % s

    # the graph reads the buffers at replay time: new inputs, new results
    (q2, k2, v2), targets2 = _inputs(6)
    loop.load(q2, k2, v2, targets2)
    loop.replay()
    loop.check()
    replayed = _outputs(loop)
    loop.run()
    loop.check()
    for s, (a, b) in enumerate(zip(replayed, _outputs(loop)), start=1):
        assert torch.equal(a, b), "replay on new inputs differs from the eager call at step %d" % s
    assert not torch.equal(replayed[0], eager[0])


def _layer_inputs(seed, L, T, D, steps):
    import numpy as np
    rng = np.random.default_rng(seed)
    bf = lambda a: torch.from_numpy(a.astype("float32")).to(torch.bfloat16)
    x = bf(rng.standard_normal((B, L, D)))
    xt = [bf(rng.standard_normal((B, T, D))) for _ in range(steps - 1)]
    w_qkv, b_qkv = bf(rng.standard_normal((3 * D, D)) / np.sqrt(D)), bf(0.1 * rng.standard_normal(3 * D))
    w_o, b_o = bf(rng.standard_normal((D, D)) / np.sqrt(D)), bf(0.1 * rng.standard_normal(D))
    return x, xt, w_qkv, b_qkv, w_o, b_o


@pytest.mark.gpu
def test_layer_loop_with_projections(cuda_device):
    """Each step projects its tokens' hidden states (step 1 all, later steps
    the target only), attends and projects the output; against the float64
    chain, and replayed as a graph bit-identically."""
    loop = qi.DenoiseLoop(SEGS, B, H, STEPS, device=cuda_device, projections=True)
    L, T, P, D = loop.L, loop.T, loop.P, H * 128
    x, xt, w_qkv, b_qkv, w_o, b_o = _layer_inputs(8, L, T, D, STEPS)
    loop.load_layer(x, xt, w_qkv, b_qkv, w_o, b_o)
    loop.run()
    loop.check()
    torch.cuda.synchronize()
    eager = [loop.y.cpu()] + [y.cpu() for y in loop.target_y]

    f = W.as_f64
    opos, okv = O.positions(SEGS)

    def qkv(h):
        z = O.linear(f(h), f(w_qkv), f(b_qkv))
        return [z[..., i * D:(i + 1) * D].reshape(z.shape[0], z.shape[1], H, 128) for i in range(3)]

    q, k, v = qkv(x)
    o = O.attn_full(q, k, v, opos, okv)
    assert_close(eager[0], O.linear(o.reshape(B, L, D), f(w_o), f(b_o)), torch.bfloat16, "layer step 1")
    okc, ovc = O.prefix_cache(k, v, opos, P)
    for s in range(2, STEPS + 1):
        qt, kt, vt = qkv(xt[s - 2])
        ot = O.attn_cached(qt, kt, vt, opos[P:], okc, ovc)
        assert_close(eager[s - 1], O.linear(ot.reshape(B, T, D), f(w_o), f(b_o)), torch.bfloat16,
                     "layer step %d" % s)

    loop.capture()
    for y in [loop.y] + loop.target_y:
        y.fill_(float("nan"))
    loop.replay()
    loop.check()
    torch.cuda.synchronize()
    for s, (a, b) in enumerate(zip(eager, [loop.y.cpu()] + [y.cpu() for y in loop.target_y]), start=1):
        assert torch.equal(a, b), "graph replay differs from the eager layer step %d" % s
