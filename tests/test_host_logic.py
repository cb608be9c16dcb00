"""Host-side logic the kernels rely on, checked on the CPU: the weight layout
the fused projection + SwiGLU launch reads, the denoising loop's sigma
schedule, and the seeded inputs (same seed, same data; different steps,
different data)."""

import numpy as np
import torch

from diffusion_transformer_joint_axial_b200 import _binding as qb
from diffusion_transformer_joint_axial_b200 import workloads as W


def test_interleave_gate_up_layout():
    """Rows 256j..256j+127 are gate rows 128j.., rows 256j+128.. the matching
    up rows (the layout qi21_linear_swiglu documents)."""
    F, K = 384, 5
    t = torch.arange(2 * F * K, dtype=torch.float32).reshape(2 * F, K)
    il = qb.interleave_gate_up(t)
    assert il.shape == t.shape and il.is_contiguous()
    for j in range(F // 128):
        assert torch.equal(il[256 * j:256 * j + 128], t[128 * j:128 * j + 128])
        assert torch.equal(il[256 * j + 128:256 * j + 256], t[F + 128 * j:F + 128 * j + 128])
    b = torch.arange(2 * F)
    assert torch.equal(qb.interleave_gate_up(b)[:256], torch.cat([b[:128], b[F:F + 128]]))
    # a permutation: every row appears once
    assert sorted(qb.interleave_gate_up(b).tolist()) == list(range(2 * F))


def test_denoise_sigmas():
    """linspace(1, 1/S, S) followed by 0 (close reading 8.3's schedule, Euler to sigma = 0)."""
    for S in (1, 3, 8):
        s = W.denoise_sigmas(S)
        assert len(s) == S + 1 and s[-1] == 0.0
        assert np.allclose(s[:-1], np.linspace(1.0, 1.0 / S, S), rtol=0, atol=1e-15)


def test_seeded_inputs_are_deterministic():
    a = W.draw_qkv(1, 33, 2, 7, "bf16")
    b = W.draw_qkv(1, 33, 2, 7, "bf16")
    assert all(torch.equal(x, y) for x, y in zip(a, b))
    c2, c3 = W.cached_inputs("maxref", 2), W.cached_inputs("maxref", 3)
    assert not torch.equal(c2[0], c3[0])
    p1, _ = W.denoise_model(1, 16, 1, 2, seed=5, dtype="f32")
    p2, _ = W.denoise_model(1, 16, 1, 2, seed=5, dtype="f32")
    assert torch.equal(p1["blocks"][0]["w_gu"], p2["blocks"][0]["w_gu"])


def test_fp16_rotation_table_error_bound():
    """The bf16 path rotates its queries with (cos, sin) rounded to fp16; over
    every position of every workload they stay within 2.4e-4 (2^-12) of the
    float64 values, a tenth of the bf16 rounding of a rotated query."""
    import oracle as O
    worst = 0.0
    for name, cfg in W.WORKLOADS.items():
        fn = O.positions_original if cfg.get("original") else O.positions
        pos, _ = fn(cfg["segments"])
        ang = O.rope_angles(pos)
        for f in (np.cos, np.sin):
            exact = f(ang)
            worst = max(worst, float(np.max(np.abs(exact.astype(np.float16).astype(np.float64) - exact))))
    assert worst <= 2.0 ** -12, worst
