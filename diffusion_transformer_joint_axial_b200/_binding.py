"""ctypes binding of libqi21 (argument marshalling only).

Every step of the path runs in the library's CUDA kernels; torch supplies
device memory and the current stream.  If ``libqi21.so`` is missing or no
CUDA device is present, every call raises ``QI21Error``: there is no fallback.
"""

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqi21.so")

QI21_OK = 0
QI21_ERR_INVALID_ARG = 1
QI21_ERR_UNSUPPORTED = 2
QI21_ERR_CUDA = 3
QI21_ERR_TIMEOUT = 4
QI21_BF16 = 0
QI21_F32 = 1
HEAD_DIM = 128
MAX_SEGMENTS = 128
WORKSPACE_HEADER_BYTES = 256

EXPORTED = (
    # positions and the attention steps
    "qi21_rope_positions", "qi21_rope_positions_original",
    "qi21_attn_full_workspace_size", "qi21_attn_full", "qi21_attn_full_qknorm",
    "qi21_attn_cached_workspace_size", "qi21_attn_cached", "qi21_attn_cached_qknorm",
    "qi21_attn_cached_noalloc",
    # the request's rotation table and the cached step that reads it
    "qi21_rope_table_size", "qi21_rope_table", "qi21_attn_cached_tabled",
    # projections and the rest of a block of the denoising loop
    "qi21_linear", "qi21_linear_residual", "qi21_linear_swiglu", "qi21_rmsnorm", "qi21_swiglu",
    # status, errors, counters, timing and self-tests
    "qi21_workspace_status", "qi21_status_string", "qi21_last_error", "qi21_launch_count",
    "qi21_selftest_wait_timeout",
)


class QI21Error(RuntimeError):
    def __init__(self, status, message):
        super().__init__(message)
        self.status = status


class Segment(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("n", ctypes.c_int32), ("H", ctypes.c_int32),
                ("W", ctypes.c_int32), ("frame", ctypes.c_int32)]


_lib = None
_vp = ctypes.c_void_p
_i32 = ctypes.c_int32
_i64 = ctypes.c_int64
_sz = ctypes.c_size_t


def load_library(path=LIB_PATH):
    """Loads libqi21.so and declares its C signatures (no CUDA needed)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise QI21Error(QI21_ERR_UNSUPPORTED,
                        "libqi21.so is not built (python -m diffusion_transformer_joint_axial_b200.build)")
    L = ctypes.CDLL(path)
    L.qi21_rope_positions.argtypes = [ctypes.POINTER(Segment), _i32, _i64, _vp, _vp, _vp]
    L.qi21_rope_positions_original.argtypes = [ctypes.POINTER(Segment), _i32, _i64, _vp, _vp, _vp]
    L.qi21_rope_positions_original.restype = _i32
    L.qi21_attn_full_workspace_size.argtypes = [_i32, _i32, _i64, _i64, _i32]
    L.qi21_attn_full_workspace_size.restype = _sz
    L.qi21_attn_full.argtypes = [_i32, _i32, _i64, _i64, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                 _vp, _vp, _sz, _vp]
    L.qi21_attn_cached_workspace_size.argtypes = [_i32, _i32, _i64, _i64, _i32]
    L.qi21_attn_cached_workspace_size.restype = _sz
    L.qi21_attn_cached.argtypes = [_i32, _i32, _i64, _i64, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                   _vp, _sz, _vp]
    L.qi21_attn_full_qknorm.argtypes = [_i32, _i32, _i64, _i64, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                        _vp, _vp, _vp, ctypes.c_float, _vp, _sz, _vp]
    L.qi21_attn_cached_qknorm.argtypes = [_i32, _i32, _i64, _i64, _i32, _vp, _vp, _vp, _vp, _vp, _vp,
                                          _vp, _vp, _vp, ctypes.c_float, _vp, _sz, _vp]
    L.qi21_linear.argtypes = [_i64, _i64, _i64, _vp, _vp, _vp, ctypes.POINTER(_vp), _i32, _vp, _sz, _vp]
    L.qi21_linear.restype = _i32
    L.qi21_linear_residual.argtypes = [_i64, _i64, _i64, _vp, _vp, _vp, _vp, ctypes.c_float, _vp, _vp, _sz, _vp]
    L.qi21_linear_residual.restype = _i32
    L.qi21_linear_swiglu.argtypes = [_i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
    L.qi21_linear_swiglu.restype = _i32
    L.qi21_rmsnorm.argtypes = [_i64, _i32, _vp, _vp, ctypes.c_float, _vp, _vp]
    L.qi21_rmsnorm.restype = _i32
    L.qi21_swiglu.argtypes = [_i64, _vp, _vp, _vp, _vp]
    L.qi21_swiglu.restype = _i32
    L.qi21_workspace_status.argtypes = [_vp, _vp]
    L.qi21_selftest_wait_timeout.argtypes = [_vp, _i64, _vp]
    L.qi21_status_string.argtypes = [_i32]
    L.qi21_status_string.restype = ctypes.c_char_p
    L.qi21_last_error.argtypes = []
    L.qi21_last_error.restype = ctypes.c_char_p
    L.qi21_launch_count.argtypes = []
    L.qi21_launch_count.restype = ctypes.c_uint64
    L.qi21_attn_cached_noalloc.argtypes = [_i32, _i32, _i64, _i64, _i32, _vp, _vp, _vp, _vp, _vp, _vp,
                                           _vp, _vp]
    L.qi21_attn_cached_noalloc.restype = _i32
    L.qi21_rope_table_size.argtypes = [_i64]
    L.qi21_rope_table_size.restype = _sz
    L.qi21_rope_table.argtypes = [_vp, _i64, _vp, _sz, _vp]
    L.qi21_rope_table.restype = _i32
    L.qi21_attn_cached_tabled.argtypes = [_i32, _i32, _i64, _i64, _i32, _vp, _vp, _vp, _vp, _vp, _vp,
                                          _vp, _vp, _sz, _vp]
    L.qi21_attn_cached_tabled.restype = _i32
    for name in ("qi21_rope_positions", "qi21_attn_full", "qi21_attn_cached", "qi21_attn_full_qknorm",
                 "qi21_attn_cached_qknorm", "qi21_workspace_status", "qi21_selftest_wait_timeout"):
        getattr(L, name).restype = _i32
    _lib = L
    return L


def _check(status):
    if status != QI21_OK:
        L = load_library()
        raise QI21Error(status, "%s: %s" % (L.qi21_status_string(status).decode(),
                                            L.qi21_last_error().decode()))


def _cuda_lib():
    if not torch.cuda.is_available():
        raise QI21Error(QI21_ERR_CUDA, "libqi21 needs a CUDA device; none is available")
    return load_library()


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return QI21_BF16
    if t.dtype == torch.float32:
        return QI21_F32
    raise QI21Error(QI21_ERR_UNSUPPORTED, "dtype %s is not supported (bf16 or fp32)" % t.dtype)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _need(t, name, shape, dtype, device):
    if not isinstance(t, torch.Tensor):
        raise QI21Error(QI21_ERR_INVALID_ARG, "%s must be a torch.Tensor" % name)
    if tuple(t.shape) != tuple(shape):
        raise QI21Error(QI21_ERR_INVALID_ARG, "%s has shape %s, expected %s" % (name, tuple(t.shape), tuple(shape)))
    if t.dtype != dtype or t.device != device or not t.is_contiguous():
        raise QI21Error(QI21_ERR_INVALID_ARG,
                        "%s must be a contiguous %s tensor on %s" % (name, dtype, device))


def to_segments(segments):
    """ctypes array from dicts {"kind": "text", "n"} / {"kind": "image", "H", "W", "frame"}."""
    arr = (Segment * max(1, len(segments)))()
    for i, s in enumerate(segments):
        if s["kind"] == "text":
            arr[i] = Segment(0, int(s["n"]), 0, 0, 0)
        elif s["kind"] == "image":
            arr[i] = Segment(1, 0, int(s["H"]), int(s["W"]), int(s["frame"]))
        else:
            raise QI21Error(QI21_ERR_INVALID_ARG, "unknown segment kind %r" % (s["kind"],))
    return arr


def rope_positions(segments, device="cuda", with_kv_end=True, original=False):
    """Position table ``pos[L, 3]`` (int32) and ``kv_end[L]`` on ``device``.

    ``original=True`` builds the earlier model's table (text after the
    images, no mask; ``qi21_rope_positions_original``)."""
    L_ = _cuda_lib()
    device = torch.device(device)
    if device.index is None:
        device = torch.device("cuda", torch.cuda.current_device())
    segs = to_segments(segments)
    n = sum(int(s["n"]) if s["kind"] == "text" else int(s["H"]) * int(s["W"]) for s in segments)
    pos = torch.empty((n, 3), dtype=torch.int32, device=device)
    kv_end = torch.empty((n,), dtype=torch.int32, device=device) if with_kv_end else None
    with torch.cuda.device(device):
        fn = L_.qi21_rope_positions_original if original else L_.qi21_rope_positions
        _check(fn(segs, len(segments), n, _ptr(pos), _ptr(kv_end), _stream(device)))
    return pos, kv_end


def full_workspace_size(B, H, L, P, dtype):
    code = QI21_BF16 if dtype == torch.bfloat16 else QI21_F32
    return int(load_library().qi21_attn_full_workspace_size(B, H, L, P, code))


def cached_workspace_size(B, H, P, T, dtype):
    code = QI21_BF16 if dtype == torch.bfloat16 else QI21_F32
    return int(load_library().qi21_attn_cached_workspace_size(B, H, P, T, code))


def new_workspace(nbytes, device):
    """Zeroed device workspace (the header must start at zero)."""
    return torch.zeros(max(int(nbytes), WORKSPACE_HEADER_BYTES), dtype=torch.uint8, device=device)


def alloc_cache(B, H, P, dtype, device):
    """Empty Prefix KV cache pair, [B, H, P, 128] each."""
    return (torch.empty((B, H, P, HEAD_DIM), dtype=dtype, device=device),
            torch.empty((B, H, P, HEAD_DIM), dtype=dtype, device=device))


def _norm_args(qk_norm, device):
    """(w_q, w_k, eps) -> pointers and eps for the *_qknorm entry points."""
    if qk_norm is None:
        return None
    w_q, w_k, eps = qk_norm
    _need(w_q, "w_q", (HEAD_DIM,), torch.float32, device)
    _need(w_k, "w_k", (HEAD_DIM,), torch.float32, device)
    return _ptr(w_q), _ptr(w_k), ctypes.c_float(float(eps))


def attn_full(q, k, v, pos, kv_end, prefix_len, k_cache=None, v_cache=None, out=None, workspace=None,
              qk_norm=None):
    """First step: block-causal joint attention; stores the prefix K/V cache if given.

    q, k, v: [B, L, H, 128] bf16 or fp32 on one CUDA device; pos [L, 3],
    kv_end [L] int32 from :func:`rope_positions`, or None for no mask (every
    query sees all L keys, as in the earlier model).  ``qk_norm = (w_q, w_k, eps)``
    (float32 [128] weights on the same device) fuses the QK-RMSNorm in front of
    the rotation.  Returns ``out``.
    """
    L_ = _cuda_lib()
    B, L, H, D = q.shape
    dev, dt = q.device, q.dtype
    code = _dtype_code(q)
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, (B, L, H, HEAD_DIM), dt, dev)
    _need(pos, "pos", (L, 3), torch.int32, dev)
    if kv_end is not None:
        _need(kv_end, "kv_end", (L,), torch.int32, dev)
    P = int(prefix_len)
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", (B, L, H, HEAD_DIM), dt, dev)
    if (k_cache is None) != (v_cache is None):
        raise QI21Error(QI21_ERR_INVALID_ARG, "give both k_cache and v_cache or neither")
    if k_cache is not None:
        _need(k_cache, "k_cache", (B, H, P, HEAD_DIM), dt, dev)
        _need(v_cache, "v_cache", (B, H, P, HEAD_DIM), dt, dev)
    need = full_workspace_size(B, H, L, P if k_cache is not None else 0, dt)
    if workspace is None:
        workspace = new_workspace(need, dev)
    norm = _norm_args(qk_norm, dev)
    with torch.cuda.device(dev):
        if norm is None:
            _check(L_.qi21_attn_full(B, H, L, P, code, _ptr(q), _ptr(k), _ptr(v), _ptr(pos), _ptr(kv_end),
                                     _ptr(out), _ptr(k_cache), _ptr(v_cache), _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _stream(dev)))
        else:
            _check(L_.qi21_attn_full_qknorm(B, H, L, P, code, _ptr(q), _ptr(k), _ptr(v), _ptr(pos),
                                            _ptr(kv_end), _ptr(out), _ptr(k_cache), _ptr(v_cache), *norm,
                                            _ptr(workspace), workspace.numel() * workspace.element_size(),
                                            _stream(dev)))
    return out


def rope_table_size(n):
    """Bytes of the rotation table of n tokens."""
    return int(load_library().qi21_rope_table_size(n))


def rope_table(pos, out=None):
    """The rotation table of the tokens whose positions are ``pos`` ([n, 3]
    int32 on the device): built once per request, read by every later step
    (``attn_cached(..., rope_table=t)``).  Returns a uint8 device tensor
    (``out``, if given: ``rope_table_size(n)`` bytes)."""
    L_ = _cuda_lib()
    dev = pos.device
    n = pos.shape[0]
    _need(pos, "pos", (n, 3), torch.int32, dev)
    table = out
    if table is None:
        table = torch.empty(int(L_.qi21_rope_table_size(n)), dtype=torch.uint8, device=dev)
    _need(table, "out", (int(L_.qi21_rope_table_size(n)),), torch.uint8, dev)
    with torch.cuda.device(dev):
        _check(L_.qi21_rope_table(_ptr(pos), n, _ptr(table), table.numel(), _stream(dev)))
    return table


def attn_cached(q, k, v, pos_tgt, k_cache, v_cache, out=None, workspace=None, qk_norm=None, rope_table=None):
    """Later step: target queries over [cached prefix K/V || fresh target K/V], no mask.

    q, k, v: [B, T, H, 128]; pos_tgt [T, 3]; k_cache, v_cache [B, H, P, 128].
    ``qk_norm`` as for :func:`attn_full` (the cache must come from a full step
    with the same norm).  ``rope_table``: the target's table from
    :func:`rope_table` (then ``pos_tgt`` may be None), read instead of
    computing the angles again; not with ``qk_norm``.
    """
    L_ = _cuda_lib()
    B, T, H, D = q.shape
    dev, dt = q.device, q.dtype
    code = _dtype_code(q)
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, (B, T, H, HEAD_DIM), dt, dev)
    if rope_table is None:
        _need(pos_tgt, "pos_tgt", (T, 3), torch.int32, dev)
    else:
        if qk_norm is not None:
            raise ValueError("rope_table is not taken together with qk_norm")
        _need(rope_table, "rope_table", (int(L_.qi21_rope_table_size(T)),), torch.uint8, dev)
    P = k_cache.shape[2]
    _need(k_cache, "k_cache", (B, H, P, HEAD_DIM), dt, dev)
    _need(v_cache, "v_cache", (B, H, P, HEAD_DIM), dt, dev)
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", (B, T, H, HEAD_DIM), dt, dev)
    need = cached_workspace_size(B, H, P, T, dt)
    if workspace is None:
        workspace = new_workspace(need, dev)
    norm = _norm_args(qk_norm, dev)
    with torch.cuda.device(dev):
        if rope_table is not None:
            _check(L_.qi21_attn_cached_tabled(B, H, P, T, code, _ptr(q), _ptr(k), _ptr(v), _ptr(rope_table),
                                              _ptr(k_cache), _ptr(v_cache), _ptr(out), _ptr(workspace),
                                              workspace.numel() * workspace.element_size(), _stream(dev)))
        elif norm is None:
            _check(L_.qi21_attn_cached(B, H, P, T, code, _ptr(q), _ptr(k), _ptr(v), _ptr(pos_tgt),
                                       _ptr(k_cache), _ptr(v_cache), _ptr(out), _ptr(workspace),
                                       workspace.numel() * workspace.element_size(), _stream(dev)))
        else:
            _check(L_.qi21_attn_cached_qknorm(B, H, P, T, code, _ptr(q), _ptr(k), _ptr(v), _ptr(pos_tgt),
                                              _ptr(k_cache), _ptr(v_cache), _ptr(out), *norm,
                                              _ptr(workspace), workspace.numel() * workspace.element_size(),
                                              _stream(dev)))
    return out


def linear(x, w, bias=None, n_out=1, out=None, workspace=None):
    """Y = X W^T (+ b) on the tensor cores, bf16 with fp32 accumulation.

    x: [..., K], w: [N, K] (nn.Linear layout), bias: [N] or None, all bf16 on
    one CUDA device.  The N output columns are cut into ``n_out`` equal
    segments; returns the list of ``n_out`` tensors [..., N / n_out] (or fills
    ``out``, a list of such tensors).
    """
    L_ = _cuda_lib()
    dev = x.device
    K = x.shape[-1]
    N = w.shape[0]
    lead = tuple(x.shape[:-1])
    M = 1
    for d in lead:
        M *= int(d)
    _need(x, "x", lead + (K,), torch.bfloat16, dev)
    _need(w, "w", (N, K), torch.bfloat16, dev)
    if bias is not None:
        _need(bias, "bias", (N,), torch.bfloat16, dev)
    if n_out < 1 or N % n_out != 0:
        raise QI21Error(QI21_ERR_INVALID_ARG, "N=%d does not split into %d segments" % (N, n_out))
    seg = N // n_out
    if out is None:
        out = [torch.empty(lead + (seg,), dtype=torch.bfloat16, device=dev) for _ in range(n_out)]
    if len(out) != n_out:
        raise QI21Error(QI21_ERR_INVALID_ARG, "need %d output tensors" % n_out)
    for i, o in enumerate(out):
        _need(o, "out[%d]" % i, lead + (seg,), torch.bfloat16, dev)
    if workspace is None:
        workspace = new_workspace(WORKSPACE_HEADER_BYTES, dev)
    ptrs = (_vp * n_out)(*[o.data_ptr() for o in out])
    with torch.cuda.device(dev):
        _check(L_.qi21_linear(M, N, K, _ptr(x), _ptr(w), _ptr(bias), ptrs, n_out, _ptr(workspace),
                              workspace.numel() * workspace.element_size(), _stream(dev)))
    return out


def linear_residual(x, w, bias, residual, alpha=1.0, out=None, workspace=None):
    """out = residual + alpha * (x W^T + b) on the tensor cores (bf16).

    x: [..., K], w: [N, K], bias: [N] or None, residual: [..., N]; ``out``
    defaults to a new tensor and may be ``residual`` itself."""
    L_ = _cuda_lib()
    dev = x.device
    K, N = x.shape[-1], w.shape[0]
    lead = tuple(x.shape[:-1])
    M = 1
    for d in lead:
        M *= int(d)
    _need(x, "x", lead + (K,), torch.bfloat16, dev)
    _need(w, "w", (N, K), torch.bfloat16, dev)
    if bias is not None:
        _need(bias, "bias", (N,), torch.bfloat16, dev)
    _need(residual, "residual", lead + (N,), torch.bfloat16, dev)
    if out is None:
        out = torch.empty_like(residual)
    _need(out, "out", lead + (N,), torch.bfloat16, dev)
    if workspace is None:
        workspace = new_workspace(WORKSPACE_HEADER_BYTES, dev)
    with torch.cuda.device(dev):
        _check(L_.qi21_linear_residual(M, N, K, _ptr(x), _ptr(w), _ptr(bias), _ptr(residual),
                                       ctypes.c_float(float(alpha)), _ptr(out), _ptr(workspace),
                                       workspace.numel() * workspace.element_size(), _stream(dev)))
    return out


def interleave_gate_up(t):
    """[gate; up] stacked along dim 0 (2F rows, or a 2F bias) -> the
    alternating 128-row blocks qi21_linear_swiglu reads (F a multiple of 128)."""
    F = t.shape[0] // 2
    rest = tuple(t.shape[1:])
    return t.reshape((2, F // 128, 128) + rest).transpose(0, 1).reshape((2 * F,) + rest).contiguous()


def linear_swiglu(x, w_il, bias_il=None, out=None, workspace=None):
    """silu(x W_gate^T + b_gate) * (x W_up^T + b_up) in one tensor-core launch.

    ``w_il`` [2F, K] and ``bias_il`` [2F] in the layout of
    :func:`interleave_gate_up`; returns [..., F]."""
    L_ = _cuda_lib()
    dev = x.device
    K, N = x.shape[-1], w_il.shape[0]
    lead = tuple(x.shape[:-1])
    M = 1
    for d in lead:
        M *= int(d)
    _need(x, "x", lead + (K,), torch.bfloat16, dev)
    _need(w_il, "w", (N, K), torch.bfloat16, dev)
    if bias_il is not None:
        _need(bias_il, "bias", (N,), torch.bfloat16, dev)
    if out is None:
        out = torch.empty(lead + (N // 2,), dtype=torch.bfloat16, device=dev)
    _need(out, "out", lead + (N // 2,), torch.bfloat16, dev)
    if workspace is None:
        workspace = new_workspace(WORKSPACE_HEADER_BYTES, dev)
    with torch.cuda.device(dev):
        _check(L_.qi21_linear_swiglu(M, N, K, _ptr(x), _ptr(w_il), _ptr(bias_il), _ptr(out), _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _stream(dev)))
    return out


def rmsnorm(x, w, eps, out=None):
    """Row RMSNorm over the last axis (bf16): x / sqrt(mean(x^2) + eps) * w."""
    L_ = _cuda_lib()
    dev, D = x.device, x.shape[-1]
    _need(x, "x", tuple(x.shape), torch.bfloat16, dev)
    _need(w, "w", (D,), torch.bfloat16, dev)
    if out is None:
        out = torch.empty_like(x)
    _need(out, "out", tuple(x.shape), torch.bfloat16, dev)
    with torch.cuda.device(dev):
        _check(L_.qi21_rmsnorm(x.numel() // D, D, _ptr(x), _ptr(w), ctypes.c_float(float(eps)), _ptr(out),
                               _stream(dev)))
    return out


def swiglu(g, u, out=None):
    """silu(g) * u elementwise (bf16)."""
    L_ = _cuda_lib()
    dev = g.device
    _need(g, "g", tuple(g.shape), torch.bfloat16, dev)
    _need(u, "u", tuple(g.shape), torch.bfloat16, dev)
    if out is None:
        out = torch.empty_like(g)
    _need(out, "out", tuple(g.shape), torch.bfloat16, dev)
    with torch.cuda.device(dev):
        _check(L_.qi21_swiglu(g.numel(), _ptr(g), _ptr(u), _ptr(out), _stream(dev)))
    return out


def workspace_status(workspace, device=None):
    """Synchronises the current stream and returns (and clears) the status word.

    ``workspace=None`` reads the built-in scratch of the allocation-free
    cached step (``qi21_attn_cached_noalloc``) on ``device`` (default: the
    current one)."""
    L_ = _cuda_lib()
    dev = workspace.device if workspace is not None else torch.device(
        "cuda", torch.cuda.current_device() if device is None else torch.device(device).index)
    with torch.cuda.device(dev):
        return int(L_.qi21_workspace_status(_ptr(workspace), _stream(dev)))


def selftest_wait_timeout(workspace, limit_ns, device=None):
    """One CTA waits (``limit_ns``) on a barrier nobody arrives at and records
    the timeout in the workspace header (``None``: the built-in scratch)."""
    L_ = _cuda_lib()
    dev = workspace.device if workspace is not None else torch.device(
        "cuda", torch.cuda.current_device() if device is None else torch.device(device).index)
    with torch.cuda.device(dev):
        _check(L_.qi21_selftest_wait_timeout(_ptr(workspace), int(limit_ns), _stream(dev)))


def launch_count():
    """Kernel launches this thread has enqueued through libqi21."""
    return int(load_library().qi21_launch_count())
