"""Shared helpers of the GPU parity tests: run the CUDA path through the
binding, run the float64 oracle on the same seeded inputs, compare."""

import numpy as np
import torch

import diffusion_transformer_joint_axial_b200 as qi
import oracle as O
from diffusion_transformer_joint_axial_b200 import workloads as W

# Tolerances on unit-variance inputs: fp32 max |err| <= 1e-4; bf16 max |err|
# <= 3e-2 and mean |err| <= 3e-3 (both against the float64 oracle).
F32_MAX = 1e-4
BF16_MAX = 3e-2
BF16_MEAN = 3e-3


def assert_close(gpu, ref, dtype, what=""):
    g = gpu.detach().to("cpu").to(torch.float64).numpy() if isinstance(gpu, torch.Tensor) else gpu
    err = np.abs(g - ref)
    assert np.all(np.isfinite(g)), "%s: non-finite GPU output" % what
    if dtype == torch.float32:
        assert err.max() <= F32_MAX, "%s: max err %.3g > %g" % (what, err.max(), F32_MAX)
    else:
        assert err.max() <= BF16_MAX, "%s: max err %.3g > %g" % (what, err.max(), BF16_MAX)
        assert err.mean() <= BF16_MEAN, "%s: mean err %.3g > %g" % (what, err.mean(), BF16_MEAN)
    return float(err.max()), float(err.mean())


def check_status(ws):
    st = qi.workspace_status(ws)
    assert st == 0, "device status %d: %s" % (st, qi.load_library().qi21_last_error().decode())


def gpu_full(segments, q, k, v, P, cache=True, device="cuda"):
    """Runs positions + the full step on the GPU; returns CPU copies."""
    dev = torch.device(device)
    B, L, H, _ = q.shape
    pos, kv_end = qi.rope_positions(segments, dev)
    qd, kd, vd = (x.to(dev) for x in (q, k, v))
    kc = vc = None
    if cache:
        kc, vc = qi.alloc_cache(B, H, P, q.dtype, dev)
    ws = qi.new_workspace(qi.full_workspace_size(B, H, L, P if cache else 0, q.dtype), dev)
    o = qi.attn_full(qd, kd, vd, pos, kv_end, P, kc, vc, workspace=ws)
    check_status(ws)
    torch.cuda.synchronize()
    return dict(o=o.cpu(), pos=pos.cpu(), kv_end=kv_end.cpu(), kc=kc, vc=vc)


def gpu_cached(q_t, k_t, v_t, pos_t, kc, vc, device="cuda"):
    dev = torch.device(device)
    B, T, H, _ = q_t.shape
    P = kc.shape[2]
    ws = qi.new_workspace(qi.cached_workspace_size(B, H, P, T, q_t.dtype), dev)
    o = qi.attn_cached(q_t.to(dev), k_t.to(dev), v_t.to(dev), pos_t.to(dev), kc, vc, workspace=ws)
    check_status(ws)
    torch.cuda.synchronize()
    return o.cpu()


def check_cache(kc, vc, k, v, pos, P, heads=None, batches=None, k_f64=None):
    """GPU cache vs the oracle's step-1 store: V copied exactly, K rotated
    within one rounding of the storage type.  ``k_f64`` replaces the keys the
    oracle rotates (the QK-normalised keys, for the fused norm)."""
    if P == 0:
        return
    kf, vf = (W.as_f64(k) if k_f64 is None else k_f64), W.as_f64(v)
    ok, ov = O.prefix_cache(kf, vf, pos, P, heads=heads, batches=batches)
    heads = list(range(k.shape[2])) if heads is None else list(heads)
    batches = list(range(k.shape[0])) if batches is None else list(batches)
    gk = kc.detach().cpu().to(torch.float64).numpy()[batches][:, heads]
    gv = vc.detach().cpu().to(torch.float64).numpy()[batches][:, heads]
    assert np.array_equal(gv, ov), "V cache is not an exact copy of the prefix V"
    rel = 2.0 ** -8 if kc.dtype == torch.bfloat16 else 2.0 ** -20
    assert np.all(np.abs(gk - ok) <= rel * np.abs(ok) + 1e-5), "rotated K cache off"


def sample_rows(L, P, kv_end, rng, extra=24):
    """Query rows that exercise every tile class: text start, text-diagonal
    tile edges, segment boundaries, the prefix/target boundary, the end."""
    rows = {0, 1, 2, 127, 128, 129, 255, 256, L - 1, L - 2, P - 1, P, P + 1}
    kv = np.asarray(kv_end)
    bounds = np.nonzero(np.diff(kv) > 1)[0]  # ends of image segments
    for b in bounds[:16]:
        rows.update({int(b), int(b) + 1})
    rows.update(int(x) for x in rng.integers(0, L, extra))
    return np.array(sorted(r for r in rows if 0 <= r < L), dtype=np.int64)
