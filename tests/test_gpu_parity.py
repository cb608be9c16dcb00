"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle on
identical seeded inputs.  Positions bit-exact; attention within fp32 1e-4 /
bf16 3e-2 max & 3e-3 mean."""

import numpy as np
import pytest
import torch

import diffusion_transformer_joint_axial_b200 as qi
import oracle as O
from diffusion_transformer_joint_axial_b200 import workloads as W

from parity import assert_close, check_cache, gpu_cached, gpu_full, sample_rows

pytestmark = pytest.mark.gpu

T_, I_ = W.text, W.image

ODD_LAYOUTS = {
    "ragged3": [T_(100), I_(10, 13, 1), I_(12, 9, 0)],
    "diag300": [T_(300), I_(16, 16, 0)],
    "target_only": [I_(8, 8, 0)],
    "two_tokens": [T_(1), I_(1, 1, 0)],
    "text_after_image": [T_(200), I_(5, 7, 2), T_(50), I_(9, 9, 0)],
    "odd_grids": [T_(7), I_(5, 3, -1), I_(1, 9, 4), I_(7, 7, 0)],
}


# ---------------------------------------------------------------- positions --

@pytest.mark.parametrize("name", sorted(W.WORKLOADS))
def test_positions_bit_exact_workloads(cuda_device, name):
    segs = W.WORKLOADS[name]["segments"]
    pos, kv_end = qi.rope_positions(segs, cuda_device)
    opos, okv = O.positions(segs)
    assert np.array_equal(pos.cpu().numpy(), opos)
    assert np.array_equal(kv_end.cpu().numpy(), okv)


@pytest.mark.parametrize("name", sorted(ODD_LAYOUTS))
def test_positions_bit_exact_odd(cuda_device, name):
    segs = ODD_LAYOUTS[name]
    pos, kv_end = qi.rope_positions(segs, cuda_device)
    opos, okv = O.positions(segs)
    assert np.array_equal(pos.cpu().numpy(), opos)
    assert np.array_equal(kv_end.cpu().numpy(), okv)


def test_positions_many_segments(cuda_device):
    rng = np.random.default_rng(0)
    segs = []
    for i in range(128):
        if rng.random() < 0.4:
            segs.append(T_(int(rng.integers(1, 40))))
        else:
            segs.append(I_(int(rng.integers(1, 12)), int(rng.integers(1, 12)), int(rng.integers(-3, 20))))
    pos, kv_end = qi.rope_positions(segs, cuda_device)
    opos, okv = O.positions(segs)
    assert np.array_equal(pos.cpu().numpy(), opos)
    assert np.array_equal(kv_end.cpu().numpy(), okv)


# -------------------------------------------------------------- tiny (fp32) --

def test_tiny_fp32_full_cached(cuda_device):
    name = "tiny"
    cfg = W.WORKLOADS[name]
    L, P, T = W.sizes(name)
    q, k, v = W.full_inputs(name)
    g = gpu_full(cfg["segments"], q, k, v, P)
    pos, kv_end = O.positions(cfg["segments"])
    ref = O.attn_full(W.as_f64(q), W.as_f64(k), W.as_f64(v), pos, kv_end)
    assert_close(g["o"], ref, torch.float32, "tiny full")
    check_cache(g["kc"], g["vc"], k, v, pos, P)
    qt, kt, vt = W.cached_inputs(name)
    oc = gpu_cached(qt, kt, vt, g["pos"][P:].contiguous(), g["kc"], g["vc"])
    okc, ovc = O.prefix_cache(W.as_f64(k), W.as_f64(v), pos, P)
    refc = O.attn_cached(W.as_f64(qt), W.as_f64(kt), W.as_f64(vt), pos[P:], okc, ovc)
    assert_close(oc, refc, torch.float32, "tiny cached")
    assert_close(oc, ref[:, P:], torch.float32, "tiny cached vs full target rows")


# --------------------------------------------------- small layouts (bf16/f32) --

def _small(name, dtype, B=2, H=3, seed=7):
    segs = ODD_LAYOUTS[name]
    L = sum(W.seg_tokens(s) for s in segs)
    P = L - W.seg_tokens(segs[-1])
    q, k, v = W.draw_qkv(B, L, H, seed, "bf16" if dtype == torch.bfloat16 else "f32")
    return segs, L, P, q, k, v


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
@pytest.mark.parametrize("name", sorted(ODD_LAYOUTS))
def test_small_layouts_full_and_cached(cuda_device, name, dtype):
    segs, L, P, q, k, v = _small(name, dtype)
    g = gpu_full(segs, q, k, v, P)
    pos, kv_end = O.positions(segs)
    qf, kf, vf = W.as_f64(q), W.as_f64(k), W.as_f64(v)
    ref = O.attn_full(qf, kf, vf, pos, kv_end)
    assert_close(g["o"], ref, dtype, name + " full")
    check_cache(g["kc"], g["vc"], k, v, pos, P)
    # cached step on the same target rows must reproduce the full step's target rows
    qt, kt, vt = (x[:, P:].contiguous() for x in (q, k, v))
    oc = gpu_cached(qt, kt, vt, g["pos"][P:].contiguous(), g["kc"], g["vc"])
    okc, ovc = O.prefix_cache(kf, vf, pos, P)
    refc = O.attn_cached(W.as_f64(qt), W.as_f64(kt), W.as_f64(vt), pos[P:], okc, ovc)
    assert_close(oc, refc, dtype, name + " cached")
    assert_close(oc, ref[:, P:], dtype, name + " cached vs full")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
def test_full_without_cache(cuda_device, dtype):
    segs, L, P, q, k, v = _small("ragged3", dtype, B=1, H=2, seed=3)
    g = gpu_full(segs, q, k, v, P, cache=False)
    pos, kv_end = O.positions(segs)
    ref = O.attn_full(W.as_f64(q), W.as_f64(k), W.as_f64(v), pos, kv_end)
    assert_close(g["o"], ref, dtype, "no cache")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
def test_q_zero_is_mean_of_visible_values(cuda_device, dtype):
    """Q = 0 makes every logit 0: O_i is the mean of V over j < kv_end[i].
    Pins the mask and the tile skipping on the GPU independently of RoPE."""
    segs = [T_(300), I_(12, 12, 1), I_(16, 16, 0)]
    L = 300 + 144 + 256
    P = 444
    _, k, v = W.draw_qkv(1, L, 2, 5, "bf16" if dtype == torch.bfloat16 else "f32")
    q = torch.zeros_like(k)
    g = gpu_full(segs, q, k, v, P)
    _, kv_end = O.positions(segs)
    vf = W.as_f64(v)
    csum = np.cumsum(vf, axis=1)
    ref = csum[:, kv_end - 1] / kv_end[None, :, None, None]
    assert_close(g["o"], ref, dtype, "Q=0")


def test_prefix_outputs_ignore_target(cuda_device):
    """The Prefix never attends the target: changing the target's Q/K/V must
    leave every prefix output bit-identical on the GPU too."""
    segs, L, P, q, k, v = _small("diag300", torch.bfloat16, B=1, H=2, seed=11)
    a = gpu_full(segs, q, k, v, P)["o"]
    q2, k2, v2 = q.clone(), k.clone(), v.clone()
    for x in (q2, k2, v2):
        x[:, P:] = -x[:, P:] * 3
    b = gpu_full(segs, q2, k2, v2, P)["o"]
    assert torch.equal(a[:, :P], b[:, :P])
    assert not torch.equal(a[:, P:], b[:, P:])


def test_deterministic(cuda_device):
    segs, L, P, q, k, v = _small("ragged3", torch.bfloat16, B=1, H=2, seed=2)
    a = gpu_full(segs, q, k, v, P)["o"]
    b = gpu_full(segs, q, k, v, P)["o"]
    assert torch.equal(a, b)


# ----------------------------------------------------------- full-size runs --

@pytest.mark.parametrize("name", ["t2i", "edit3", "hires", "maxref"])
def test_workload_full_size(cuda_device, name):
    """Full sizes: the launch configuration the bench times; sampled rows and
    heads against the oracle, computed one by one."""
    cfg = W.WORKLOADS[name]
    L, P, T = W.sizes(name)
    q, k, v = W.full_inputs(name)
    g = gpu_full(cfg["segments"], q, k, v, P)
    pos, kv_end = O.positions(cfg["segments"])
    assert np.array_equal(g["pos"].numpy(), pos)
    rng = np.random.default_rng(123)
    rows = sample_rows(L, P, kv_end, rng)
    H = cfg["H"]
    hs = [0, H // 2, H - 1]
    qf, kf, vf = (W.as_f64(x[:, :, hs]) for x in (q, k, v))
    ref = O.attn_full(qf, kf, vf, pos, kv_end, rows=rows)
    got = g["o"][:, rows][:, :, hs]
    assert_close(got, ref, torch.bfloat16, name + " full (sampled)")
    check_cache(g["kc"][:, hs], g["vc"][:, hs], k[:, :, hs], v[:, :, hs], pos, P)
    okc, ovc = O.prefix_cache(kf, vf, pos, P)
    steps = range(2, 2 + cfg.get("cached_steps", 1))
    trows = np.array(sorted(set([0, 1, T - 1] + list(rng.integers(0, T, 24)))), dtype=np.int64)
    for s in steps:
        qt, kt, vt = W.cached_inputs(name, s)
        oc = gpu_cached(qt, kt, vt, g["pos"][P:].contiguous(), g["kc"], g["vc"])
        qts, kts, vts = (W.as_f64(x[:, :, hs]) for x in (qt, kt, vt))
        refc = O.attn_cached(qts, kts, vts, pos[P:], okc, ovc, rows=trows)
        gotc = oc[:, trows][:, :, hs]
        assert_close(gotc, refc, torch.bfloat16, "%s cached step %d (sampled)" % (name, s))
        if name != "maxref":
            full_t = g["o"][:, P + trows][:, :, hs].to(torch.float64).numpy()
            assert_close(gotc, full_t, torch.bfloat16, name + " cached vs full target rows")
