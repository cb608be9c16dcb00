"""The fused QK-RMSNorm (per-head RMSNorm(128) with weight on Q and K, then
RoPE) against the float64 oracle composed the same way: small ragged layouts
in bf16 and fp32 for the full step, the cache store and the cached step, and
the text-to-image workload at full size on sampled rows and heads."""

import numpy as np
import pytest
import torch

import diffusion_transformer_joint_axial_b200 as qi
import oracle as O
from diffusion_transformer_joint_axial_b200 import workloads as W

from parity import assert_close, check_cache, check_status, sample_rows

pytestmark = pytest.mark.gpu

T_, I_ = W.text, W.image
LAYOUTS = {
    "ragged3": [T_(100), I_(10, 13, 1), I_(12, 9, 0)],
    "diag300": [T_(300), I_(16, 16, 0)],
    "text_after_image": [T_(200), I_(5, 7, 2), T_(50), I_(9, 9, 0)],
    "two_tokens": [T_(1), I_(1, 1, 0)],
}
EPS = W.QK_NORM_EPS


def _run(segs, q, k, v, P, wq, wk, dev, qt=None, kt=None, vt=None):
    B, L, H, _ = q.shape
    pos, kv_end = qi.rope_positions(segs, dev)
    norm = (wq.to(dev), wk.to(dev), EPS)
    kc, vc = qi.alloc_cache(B, H, P, q.dtype, dev)
    ws = qi.new_workspace(qi.full_workspace_size(B, H, L, P, q.dtype), dev)
    o = qi.attn_full(q.to(dev), k.to(dev), v.to(dev), pos, kv_end, P, kc, vc, workspace=ws, qk_norm=norm)
    check_status(ws)
    out = dict(o=o.cpu(), kc=kc, vc=vc, pos=pos)
    if qt is not None:
        T = qt.shape[1]
        wsc = qi.new_workspace(qi.cached_workspace_size(B, H, P, T, q.dtype), dev)
        oc = qi.attn_cached(qt.to(dev), kt.to(dev), vt.to(dev), pos[P:].clone(), kc, vc, workspace=wsc,
                            qk_norm=norm)
        check_status(wsc)
        out["oc"] = oc.cpu()
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
@pytest.mark.parametrize("name", sorted(LAYOUTS))
def test_qknorm_small_layouts(cuda_device, name, dtype):
    segs = LAYOUTS[name]
    L = sum(W.seg_tokens(s) for s in segs)
    P = L - W.seg_tokens(segs[-1])
    B, H = 2, 3
    q, k, v = W.draw_qkv(B, L, H, 17, "bf16" if dtype == torch.bfloat16 else "f32")
    # inputs far from unit scale, so the norm has work to do
    q, k = (q.float() * 6.0).to(dtype), (k.float() * 0.2).to(dtype)
    wq, wk = W.qk_norm_weights()
    qt, kt, vt = W.draw_qkv(B, L - P, H, 18, "bf16" if dtype == torch.bfloat16 else "f32")
    g = _run(segs, q, k, v, P, wq, wk, cuda_device, qt, kt, vt)

    pos, kv_end = O.positions(segs)
    wq64, wk64 = W.as_f64(wq), W.as_f64(wk)
    qn, kn = O.rms_norm(W.as_f64(q), wq64, EPS), O.rms_norm(W.as_f64(k), wk64, EPS)
    vf = W.as_f64(v)
    ref = O.attn_full(qn, kn, vf, pos, kv_end)
    assert_close(g["o"], ref, dtype, name + " qk-norm full")
    check_cache(g["kc"], g["vc"], k, v, pos, P, k_f64=kn)
    okc, ovc = O.prefix_cache(kn, vf, pos, P)
    refc = O.attn_cached(O.rms_norm(W.as_f64(qt), wq64, EPS), O.rms_norm(W.as_f64(kt), wk64, EPS),
                         W.as_f64(vt), pos[P:], okc, ovc)
    assert_close(g["oc"], refc, dtype, name + " qk-norm cached")


def test_qknorm_changes_the_result(cuda_device):
    """The fused path is not the plain one: with non-unit weights and inputs
    away from unit scale the outputs differ by far more than the tolerance."""
    segs = LAYOUTS["ragged3"]
    L = sum(W.seg_tokens(s) for s in segs)
    P = L - W.seg_tokens(segs[-1])
    q, k, v = W.draw_qkv(1, L, 2, 19, "bf16")
    q = (q.float() * 6.0).to(torch.bfloat16)
    wq, wk = W.qk_norm_weights()
    g = _run(segs, q, k, v, P, wq, wk, cuda_device)
    pos, kv_end = qi.rope_positions(segs, cuda_device)
    plain = qi.attn_full(q.to(cuda_device), k.to(cuda_device), v.to(cuda_device), pos, kv_end, P).cpu()
    assert (g["o"].float() - plain.float()).abs().max().item() > 0.3


def test_qknorm_t2i_full_size_sampled(cuda_device):
    name = "t2i"
    cfg = W.WORKLOADS[name]
    L, P, T = W.sizes(name)
    q, k, v = W.full_inputs(name)
    wq, wk = W.qk_norm_weights()
    g = _run(cfg["segments"], q, k, v, P, wq, wk, cuda_device, *(x[:, P:].contiguous() for x in (q, k, v)))
    pos, kv_end = O.positions(cfg["segments"])
    rng = np.random.default_rng(321)
    rows = sample_rows(L, P, kv_end, rng)
    hs = [0, 11, 23]
    wq64, wk64 = W.as_f64(wq), W.as_f64(wk)
    qn = O.rms_norm(W.as_f64(q[:, :, hs]), wq64, EPS)
    kn = O.rms_norm(W.as_f64(k[:, :, hs]), wk64, EPS)
    vf = W.as_f64(v[:, :, hs])
    ref = O.attn_full(qn, kn, vf, pos, kv_end, rows=rows)
    assert_close(g["o"][:, rows][:, :, hs], ref, torch.bfloat16, "t2i qk-norm full (sampled)")
    check_cache(g["kc"][:, hs], g["vc"][:, hs], k[:, :, hs], v[:, :, hs], pos, P, k_f64=kn)
    trows = rows[rows >= P] - P
    assert_close(g["oc"][:, trows][:, :, hs], g["o"][:, P + trows][:, :, hs].to(torch.float64).numpy(),
                 torch.bfloat16, "t2i qk-norm cached vs full target rows")


def test_qknorm_cached_step_tail_split(cuda_device):
    """The fused norm on a cached step whose last wave is split into 3
    key-range pieces per unit (80 units of 48 key tiles on a 148-SM B200):
    every target row of every head against the float64 oracle."""
    segs = [T_(256), I_(32, 32, 1), I_(32, 32, 2), I_(32, 32, 3), I_(32, 32, 4), I_(24, 32, 5),
            I_(32, 32, 0)]
    L = sum(W.seg_tokens(s) for s in segs)
    T = W.seg_tokens(segs[-1])
    P = L - T
    B, H = 1, 20
    q, k, v = W.draw_qkv(B, L, H, 33, "bf16")
    q, k = (q.float() * 6.0).to(torch.bfloat16), (k.float() * 0.2).to(torch.bfloat16)
    wq, wk = W.qk_norm_weights()
    qt, kt, vt = W.draw_qkv(B, T, H, 34, "bf16")
    qt = (qt.float() * 3.0).to(torch.bfloat16)
    g = _run(segs, q, k, v, P, wq, wk, cuda_device, qt, kt, vt)
    pos, _ = O.positions(segs)
    wq64, wk64 = W.as_f64(wq), W.as_f64(wk)
    kn = O.rms_norm(W.as_f64(k), wk64, EPS)
    okc, ovc = O.prefix_cache(kn, W.as_f64(v), pos, P)
    refc = O.attn_cached(O.rms_norm(W.as_f64(qt), wq64, EPS), O.rms_norm(W.as_f64(kt), wk64, EPS),
                         W.as_f64(vt), pos[P:], okc, ovc)
    assert_close(g["oc"], refc, torch.bfloat16, "qk-norm cached step, tail split")
