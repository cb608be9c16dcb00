"""One attention layer across the denoising loop, replayable as a CUDA graph.

The sampler of the Qwen-Image-2.1 overview (cards 6A and 6B: 8 Euler steps)
runs the same transformer at every step; the Prefix (text and reference
images) is at t = 0 in every step, so step 1 computes its keys and values
once and stores them, and steps 2..N compute only the target tokens against
that cache.  :class:`DenoiseLoop` owns every buffer of that sequence for one
layer -- inputs, outputs, the cache and the two workspaces -- allocated once,
so the N attention calls can be captured into one CUDA graph and replayed
with no per-call host work (tensor-map encoding, argument checks, launches).

It is plumbing around the C ABI: the calls are ``qi21_attn_full`` and
``qi21_attn_cached`` through the binding, in stream order, and every step of
the computation runs in libqi21's kernels.
"""

import torch

from . import _binding as qb
from .workloads import seg_tokens


class DenoiseLoop:
    """Attention of one layer over ``steps`` denoising steps.

    ``segments`` is the sequence layout (text first, references, target image
    last); B and H are batch and heads.  Step 1 attends the whole sequence
    with the block-causal mask and fills the cache; each later step s attends
    its own target Q/K/V (``target_q[s - 2]`` ...) against the cache.

    With ``projections=True`` (bf16) the loop runs the attention sublayer from
    hidden states instead: each step projects its tokens' hidden states
    (step 1: the whole sequence, ``x``; step s: the target tokens only,
    ``target_x[s - 2]``) with the fused Q/K/V projection straight into the
    Q/K/V buffers, attends, and applies the output projection into ``y`` /
    ``target_y[s - 2]``.  Weights are ``w_qkv`` [3D, D], ``b_qkv`` [3D],
    ``w_o`` [D, D], ``b_o`` [D] with D = H * 128.
    """

    def __init__(self, segments, B, H, steps, dtype=torch.bfloat16, device="cuda", projections=False):
        qb._cuda_lib()  # fails loudly without the library or a CUDA device
        if steps < 1:
            raise qb.QI21Error(qb.QI21_ERR_INVALID_ARG, "steps must be >= 1")
        if not segments or segments[-1]["kind"] != "image":
            raise qb.QI21Error(qb.QI21_ERR_INVALID_ARG, "the last segment must be the target image")
        dev = torch.device(device)
        if dev.index is None:
            dev = torch.device("cuda", torch.cuda.current_device())
        counts = [seg_tokens(s) for s in segments]
        self.L, self.T = sum(counts), counts[-1]
        self.P = self.L - self.T
        self.B, self.H, self.steps, self.dtype, self.device = B, H, steps, dtype, dev
        D = qb.HEAD_DIM
        mk = lambda *shape: torch.zeros(shape, dtype=dtype, device=dev)
        self.pos, self.kv_end = qb.rope_positions(segments, dev)
        self.pos_t = self.pos[self.P:].clone()  # own allocation: 16-byte aligned
        self.q, self.k, self.v = (mk(B, self.L, H, D) for _ in range(3))
        n = steps - 1
        self.target_q, self.target_k, self.target_v = (
            [mk(B, self.T, H, D) for _ in range(n)] for _ in range(3))
        self.out_full = mk(B, self.L, H, D)
        self.out_target = [mk(B, self.T, H, D) for _ in range(n)]
        self.k_cache, self.v_cache = qb.alloc_cache(B, H, self.P, dtype, dev)
        self.ws_full = qb.new_workspace(qb.full_workspace_size(B, H, self.L, self.P, dtype), dev)
        self.ws_cached = qb.new_workspace(qb.cached_workspace_size(B, H, self.P, self.T, dtype), dev)
        self.graph = None
        self.projections = projections
        if projections:
            if dtype != torch.bfloat16:
                raise qb.QI21Error(qb.QI21_ERR_UNSUPPORTED, "the projections run in bf16 only")
            Dm = H * D
            self.x = mk(B, self.L, Dm)
            self.target_x = [mk(B, self.T, Dm) for _ in range(n)]
            self.y = mk(B, self.L, Dm)
            self.target_y = [mk(B, self.T, Dm) for _ in range(n)]
            self.w_qkv, self.b_qkv = mk(3 * Dm, Dm), mk(3 * Dm)
            self.w_o, self.b_o = mk(Dm, Dm), mk(Dm)
            self.ws_linear = qb.new_workspace(qb.WORKSPACE_HEADER_BYTES, dev)

    def load(self, q, k, v, targets=()):
        """Copies step 1's Q/K/V ([B, L, H, 128]) and the later steps' target
        (q, k, v) triples ([B, T, H, 128]) into the loop's buffers."""
        for dst, src in ((self.q, q), (self.k, k), (self.v, v)):
            dst.copy_(src, non_blocking=True)
        if len(targets) != self.steps - 1:
            raise qb.QI21Error(qb.QI21_ERR_INVALID_ARG,
                               "need %d target triples, got %d" % (self.steps - 1, len(targets)))
        for i, (tq, tk, tv) in enumerate(targets):
            self.target_q[i].copy_(tq, non_blocking=True)
            self.target_k[i].copy_(tk, non_blocking=True)
            self.target_v[i].copy_(tv, non_blocking=True)

    def load_layer(self, x, targets_x, w_qkv, b_qkv, w_o, b_o):
        """Copies the hidden states (step 1: [B, L, D]; later steps: target
        [B, T, D] each) and the projection weights into the loop's buffers."""
        if not self.projections:
            raise qb.QI21Error(qb.QI21_ERR_INVALID_ARG, "the loop was built without projections")
        if len(targets_x) != self.steps - 1:
            raise qb.QI21Error(qb.QI21_ERR_INVALID_ARG,
                               "need %d target inputs, got %d" % (self.steps - 1, len(targets_x)))
        pairs = [(self.x, x), (self.w_qkv, w_qkv), (self.b_qkv, b_qkv), (self.w_o, w_o), (self.b_o, b_o)]
        pairs += list(zip(self.target_x, targets_x))
        for dst, src in pairs:
            dst.copy_(src, non_blocking=True)

    def _project_in(self, x, q, k, v):
        flat = lambda t: t.view(t.shape[0], t.shape[1], -1)
        qb.linear(x, self.w_qkv, self.b_qkv, n_out=3, out=[flat(q), flat(k), flat(v)], workspace=self.ws_linear)

    def _project_out(self, o, y):
        qb.linear(o.view(o.shape[0], o.shape[1], -1), self.w_o, self.b_o, out=[y], workspace=self.ws_linear)

    def run(self):
        """Enqueues the N steps (with their projections, if any) on the current stream."""
        if self.projections:
            self._project_in(self.x, self.q, self.k, self.v)
        qb.attn_full(self.q, self.k, self.v, self.pos, self.kv_end, self.P, self.k_cache, self.v_cache,
                     out=self.out_full, workspace=self.ws_full)
        if self.projections:
            self._project_out(self.out_full, self.y)
        for i in range(self.steps - 1):
            if self.projections:
                self._project_in(self.target_x[i], self.target_q[i], self.target_k[i], self.target_v[i])
            qb.attn_cached(self.target_q[i], self.target_k[i], self.target_v[i], self.pos_t,
                           self.k_cache, self.v_cache, out=self.out_target[i], workspace=self.ws_cached)
            if self.projections:
                self._project_out(self.out_target[i], self.target_y[i])

    def capture(self):
        """Captures :meth:`run` into a CUDA graph (after one eager run on a
        side stream, which also resolves the library's one-time lookups)."""
        side = torch.cuda.Stream(self.device)
        side.wait_stream(torch.cuda.current_stream(self.device))
        with torch.cuda.stream(side):
            self.run()
        torch.cuda.current_stream(self.device).wait_stream(side)
        self.check()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side, capture_error_mode="thread_local"):
            self.run()
        self.graph = g
        return g

    def replay(self):
        if self.graph is None:
            raise qb.QI21Error(qb.QI21_ERR_INVALID_ARG, "capture() the loop first")
        self.graph.replay()

    def check(self):
        """Synchronises and raises if a bounded device wait ran out in either
        workspace."""
        for ws in (self.ws_full, self.ws_cached) + ((self.ws_linear,) if self.projections else ()):
            st = qb.workspace_status(ws)
            if st != qb.QI21_OK:
                qb._check(st)
