"""The allocation-free cached step, qi21_attn_cached_noalloc.

It serves callers that must not allocate device memory while they run
attention (plugin hosts that only get a stream and tensors, servers that
reserve all memory up front, loops where cudaMalloc would synchronise the
device).  Its scratch is an array built into the library, so the test checks
two calls in a row -- the second one finding the first one's data still in
that array -- against the float64 oracle and against qi21_attn_cached with a
workspace, and that a device wait that runs out on the built-in scratch is
reported by qi21_workspace_status(NULL).  This file is collected last on
purpose.
"""

import ctypes

import pytest
import torch

import diffusion_transformer_joint_axial_b200 as qi
import oracle as O
from diffusion_transformer_joint_axial_b200 import _binding as qb
from diffusion_transformer_joint_axial_b200 import workloads as W

from parity import assert_close


def _noalloc(lib, q, k, v, pos_t, kc, vc, out):
    B, T, H, _ = q.shape
    P = kc.shape[2]
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream(q.device).cuda_stream)
    return lib.qi21_attn_cached_noalloc(B, H, P, T, qb.QI21_BF16, p(q), p(k), p(v), p(pos_t), p(kc), p(vc),
                                        p(out), stream)


@pytest.mark.gpu
def test_noalloc_matches_oracle_on_two_calls(cuda_device):
    lib = qi.load_library()
    segs = [W.text(200), W.image(16, 20, 1), W.image(32, 32, 0)]
    L, T = 200 + 320 + 1024, 1024
    P = L - T
    B, H = 1, 4
    q, k, v = W.draw_qkv(B, L, H, 21, "bf16")
    pos, kv_end = qi.rope_positions(segs, cuda_device)
    kc, vc = qi.alloc_cache(B, H, P, torch.bfloat16, cuda_device)
    qi.attn_full(q.to(cuda_device), k.to(cuda_device), v.to(cuda_device), pos, kv_end, P, kc, vc)
    pos_t = pos[P:].contiguous()
    opos, _ = O.positions(segs)
    okc, ovc = O.prefix_cache(W.as_f64(k), W.as_f64(v), opos, P)
    for call, seed in enumerate((31, 32)):
        qt, kt, vt = W.draw_qkv(B, T, H, seed, "bf16")
        dq, dk, dv = (x.to(cuda_device) for x in (qt, kt, vt))
        out = torch.full_like(dq, float("nan"))
        st = _noalloc(lib, dq, dk, dv, pos_t, kc, vc, out)
        assert st == 0, lib.qi21_last_error().decode()
        torch.cuda.synchronize()
        ref = O.attn_cached(W.as_f64(qt), W.as_f64(kt), W.as_f64(vt), opos[P:], okc, ovc)
        assert_close(out, ref, torch.bfloat16, "no-alloc call %d vs the oracle" % call)
        with_ws = qi.attn_cached(dq, dk, dv, pos_t, kc, vc)
        assert_close(out, with_ws.to(torch.float64).cpu().numpy(), torch.bfloat16,
                     "no-alloc call %d vs qi21_attn_cached" % call)
    assert qi.workspace_status(None) == 0


@pytest.mark.gpu
def test_noalloc_timeout_is_reported(cuda_device):
    """A bounded device wait that runs out on the built-in scratch stays
    recorded until qi21_workspace_status(NULL) reads and clears it; later
    calls still work."""
    lib = qi.load_library()
    qi.selftest_wait_timeout(None, 2_000_000)  # 2 ms on a barrier nobody arrives at
    assert qi.workspace_status(None) == qb.QI21_ERR_TIMEOUT
    assert qi.workspace_status(None) == 0
    segs = [W.text(40), W.image(8, 8, 0)]
    B, H, P, T = 1, 2, 40, 64
    q, k, v = (x.to(cuda_device) for x in W.draw_qkv(B, P + T, H, 5, "bf16"))
    pos, kv_end = qi.rope_positions(segs, cuda_device)
    kc, vc = qi.alloc_cache(B, H, P, torch.bfloat16, cuda_device)
    ref = qi.attn_full(q, k, v, pos, kv_end, P, kc, vc)
    out = torch.empty((B, T, H, 128), dtype=torch.bfloat16, device=cuda_device)
    st = _noalloc(lib, q[:, P:].contiguous(), k[:, P:].contiguous(), v[:, P:].contiguous(),
                  pos[P:].contiguous(), kc, vc, out)
    assert st == 0, lib.qi21_last_error().decode()
    torch.cuda.synchronize()
    assert qi.workspace_status(None) == 0
    assert_close(out, ref[:, P:].to(torch.float64).cpu().numpy(), torch.bfloat16, "after a timeout")


def test_noalloc_rejects_sizes_beyond_its_scratch():
    """Host-side check, no GPU: a cached step needing more than the built-in
    32 MiB is refused before anything is enqueued."""
    lib = qb.load_library()
    B, H, P, T = 2, 24, 4608, 16384  # the 2048^2 workload's cached step: ~200 MB of scratch
    assert lib.qi21_attn_cached_workspace_size(B, H, P, T, qb.QI21_BF16) > (32 << 20)
    p = ctypes.c_void_p(256)
    st = lib.qi21_attn_cached_noalloc(B, H, P, T, qb.QI21_BF16, p, p, p, p, p, p, p, None)
    assert st == qb.QI21_ERR_INVALID_ARG
    assert "built-in scratch" in lib.qi21_last_error().decode()
