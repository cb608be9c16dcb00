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
    """

    def __init__(self, segments, B, H, steps, dtype=torch.bfloat16, device="cuda"):
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

    def run(self):
        """Enqueues the N attention calls on the current stream."""
        qb.attn_full(self.q, self.k, self.v, self.pos, self.kv_end, self.P, self.k_cache, self.v_cache,
                     out=self.out_full, workspace=self.ws_full)
        for i in range(self.steps - 1):
            qb.attn_cached(self.target_q[i], self.target_k[i], self.target_v[i], self.pos_t,
                           self.k_cache, self.v_cache, out=self.out_target[i], workspace=self.ws_cached)

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
        for ws in (self.ws_full, self.ws_cached):
            st = qb.workspace_status(ws)
            if st != qb.QI21_OK:
                qb._check(st)
