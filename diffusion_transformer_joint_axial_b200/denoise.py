"""The denoising loop around the attention, in reduced form, on libqi21's kernels.

The Qwen-Image-2.1 overview's sampler (cards 4A, 5A, 6A, 6B): every Euler
step runs a stack of blocks -- RMSNorm -> attention -> residual, RMSNorm ->
SwiGLU feed-forward (3x wider) -> residual -- then maps the target tokens to
a velocity and moves the target latents, x <- x + (sigma' - sigma) v.  The
Prefix (text and reference images) takes no step-dependent input, so step 1
runs every token and stores each block's Prefix K/V, and steps 2..N run the
target tokens only against those caches (card 6A); ``cached=False`` runs
every token at every step instead, the recomputation the cache must match.

Reduced form: the time conditioning of the target is one embedding bias per
step, and the modulation of the blocks (cards 3B, 5A, 6B) is left out; what
the cache relies on -- the Prefix never attends the target and never sees the
step -- holds as in the full model.  One batch element (B = 1).  Parameters
are those of ``workloads.denoise_model`` (the oracle's ``denoise`` layout).

This module is plumbing: it allocates buffers once and enqueues library
calls (projections, RMSNorm, the projection with the SwiGLU gate in its
epilogue, RoPE/cache pre-pass, attention) in stream order; every arithmetic
step runs in libqi21's kernels.
"""

import torch

from . import _binding as qb
from .workloads import seg_tokens


class DenoiseModel:
    def __init__(self, segments, heads, channels, blocks, steps, sigmas, device="cuda", cached=True,
                 eps=1e-6):
        qb._cuda_lib()  # fails loudly without the library or a CUDA device
        if not segments or segments[-1]["kind"] != "image":
            raise qb.QI21Error(qb.QI21_ERR_INVALID_ARG, "the last segment must be the target image")
        if len(sigmas) != steps + 1:
            raise qb.QI21Error(qb.QI21_ERR_INVALID_ARG, "need steps + 1 sigmas")
        dev = torch.device(device)
        if dev.index is None:
            dev = torch.device("cuda", torch.cuda.current_device())
        counts = [seg_tokens(s) for s in segments]
        self.L, self.T = sum(counts), counts[-1]
        self.P = self.L - self.T
        self.H, self.C, self.n_blocks, self.steps = heads, channels, blocks, steps
        self.D, self.F = heads * qb.HEAD_DIM, 3 * heads * qb.HEAD_DIM
        self.sigmas, self.cached, self.eps, self.device = list(sigmas), cached, eps, dev
        D, F, C, L, T, P, H = self.D, self.F, self.C, self.L, self.T, self.P, self.H
        bf = torch.bfloat16
        z = lambda *shape: torch.zeros(shape, dtype=bf, device=dev)
        self.pos, self.kv_end = qb.rope_positions(segments, dev)
        self.pos_t = self.pos[P:].clone()  # own allocation: 16-byte aligned
        # parameters
        self.w_in, self.b_in = z(D, C), z(steps, D)
        self.blocks = [dict(norm1=z(D), w_qkv=z(3 * D, D), b_qkv=z(3 * D), w_o=z(D, D), b_o=z(D),
                            norm2=z(D), w_gu=z(2 * F, D), b_gu=z(2 * F), w_down=z(D, F), b_down=z(D))
                       for _ in range(blocks)]
        self.norm_out, self.w_v, self.b_v = z(D), z(C, D), z(C)
        # inputs and state
        self.x = z(1, T, C)
        self.prefix_h = z(1, P, D)
        # activations: every token (full path) and target tokens only (cached path)
        self.act = {n: self._acts(n) for n in ((L, T) if cached else (L,))}
        self.caches = [qb.alloc_cache(1, H, P, bf, dev) for _ in range(blocks)] if cached else None
        self.ws_full = qb.new_workspace(qb.full_workspace_size(1, H, L, P if cached else 0, bf), dev)
        self.ws_cached = qb.new_workspace(qb.cached_workspace_size(1, H, P, T, bf), dev)
        self.ws_linear = qb.new_workspace(qb.WORKSPACE_HEADER_BYTES, dev)
        self.graph = None

    def _acts(self, n):
        z = lambda *shape: torch.zeros(shape, dtype=torch.bfloat16, device=self.device)
        D, F, H = self.D, self.F, self.H
        return dict(h=z(1, n, D), a=z(1, n, D), q=z(1, n, H, 128), k=z(1, n, H, 128), v=z(1, n, H, 128),
                    o=z(1, n, H, 128), m=z(1, n, F))

    def load(self, params, x0, prefix_h):
        """Copies parameters (``workloads.denoise_model`` layout), the initial
        target latents [1, T, C] and the Prefix hidden states [1, P, D]."""
        pairs = [(self.w_in, params["w_in"]), (self.b_in, params["b_in"]), (self.norm_out, params["norm_out"]),
                 (self.w_v, params["w_v"]), (self.b_v, params["b_v"]), (self.x, x0), (self.prefix_h, prefix_h)]
        for mine, theirs in zip(self.blocks, params["blocks"]):
            pairs += [(mine[k], theirs[k]) for k in mine]
        for dst, src in pairs:
            dst.copy_(src, non_blocking=True)
        # the feed-forward layer's [gate; up] weights go to the alternating
        # 128-row blocks of the fused projection + SwiGLU launch
        for blk in self.blocks:
            blk["w_gu"].copy_(qb.interleave_gate_up(blk["w_gu"]))
            blk["b_gu"].copy_(qb.interleave_gate_up(blk["b_gu"]))

    def _block(self, i, A, n):
        """One block on the n tokens of activation set A."""
        blk, ws = self.blocks[i], self.ws_linear
        flat = lambda t: t.view(1, n, -1)
        qb.rmsnorm(A["h"], blk["norm1"], self.eps, out=A["a"])
        qb.linear(A["a"], blk["w_qkv"], blk["b_qkv"], n_out=3, out=[flat(A["q"]), flat(A["k"]), flat(A["v"])],
                  workspace=ws)
        if n == self.L:
            kc, vc = self.caches[i] if self.cached else (None, None)
            qb.attn_full(A["q"], A["k"], A["v"], self.pos, self.kv_end, self.P, kc, vc, out=A["o"],
                         workspace=self.ws_full)
        else:
            kc, vc = self.caches[i]
            qb.attn_cached(A["q"], A["k"], A["v"], self.pos_t, kc, vc, out=A["o"], workspace=self.ws_cached)
        qb.linear_residual(flat(A["o"]), blk["w_o"], blk["b_o"], A["h"], out=A["h"], workspace=ws)
        qb.rmsnorm(A["h"], blk["norm2"], self.eps, out=A["a"])
        qb.linear_swiglu(A["a"], blk["w_gu"], blk["b_gu"], out=A["m"], workspace=ws)
        qb.linear_residual(A["m"], blk["w_down"], blk["b_down"], A["h"], out=A["h"], workspace=ws)

    def run(self):
        """Enqueues the whole loop on the current stream; the result is ``x``."""
        L, T, P = self.L, self.T, self.P
        for step in range(self.steps):
            full = step == 0 or not self.cached
            A = self.act[L] if full else self.act[T]
            h_t = A["h"][:, P:] if full else A["h"]  # contiguous: one batch element
            if full:
                A["h"][:, :P].copy_(self.prefix_h, non_blocking=True)
            qb.linear(self.x, self.w_in, self.b_in[step], out=[h_t], workspace=self.ws_linear)
            for i in range(self.n_blocks):
                self._block(i, A, L if full else T)
            a_t = A["a"][:, P:] if full else A["a"]
            qb.rmsnorm(h_t, self.norm_out, self.eps, out=a_t)
            qb.linear_residual(a_t, self.w_v, self.b_v, self.x, alpha=self.sigmas[step + 1] - self.sigmas[step],
                               out=self.x, workspace=self.ws_linear)

    def capture(self):
        """Captures ``run`` into a CUDA graph (after one eager run on a side
        stream).  Replays restart from the latents ``x`` holds then."""
        side = torch.cuda.Stream(self.device)
        side.wait_stream(torch.cuda.current_stream(self.device))
        x0 = self.x.clone()
        with torch.cuda.stream(side):
            self.run()
        torch.cuda.current_stream(self.device).wait_stream(side)
        self.check()
        self.x.copy_(x0)
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
        """Synchronises and raises if a bounded device wait ran out."""
        for ws in (self.ws_full, self.ws_cached, self.ws_linear):
            st = qb.workspace_status(ws)
            if st != qb.QI21_OK:
                qb._check(st)

    def flops(self):
        """Algorithmic FLOPs of one run: projections, feed-forward layers and
        the attention's allowed pairs (full step: sum of kv_end; cached: T (P + T))."""
        D, F, C, L, T, P = self.D, self.F, self.C, self.L, self.T, self.P
        per_token = 2 * (C * D + self.n_blocks * (4 * D * D + 3 * D * F) + D * C)
        pairs_full = int(self.kv_end.sum().item())
        attn_full = 4 * 128 * pairs_full * self.H * self.n_blocks
        attn_cached = 4 * 128 * T * (P + T) * self.H * self.n_blocks
        full_tokens = L if self.cached else L * self.steps
        total = per_token * (full_tokens + (T * (self.steps - 1) if self.cached else 0))
        # the embedding and velocity run on the target tokens only
        total -= 2 * (C * D + D * C) * (L - T) * (1 if self.cached else self.steps)
        total += attn_full * (1 if self.cached else self.steps)
        if self.cached:
            total += attn_cached * (self.steps - 1)
        return float(total)
