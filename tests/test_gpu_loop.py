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
