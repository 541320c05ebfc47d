"""One MLA layer's decode step as the five C-ABI calls, in the pages' order.

[P5] "MLA · latent KV, decoupled RoPE và matrix absorption", section 2
"Luồng": project the hidden state to the latent, write the cache, then read
it and project the output.  Here that is: append the new latent rows, build
the absorbed queries, run split-KV decode over the paged cache, merge the
splits, and apply W_UV / W_O.  All buffers are allocated once, up front.
"""

from __future__ import annotations

from typing import Dict, Optional

import torch

from . import abi


class DecodeLayer:
    def __init__(self, cfg: abi.Config, weights: Dict[str, torch.Tensor], cache: abi.Cache,
                 batch: int, n_q: int, max_workers: int = 0, packed_query: bool = True):
        self.cfg, self.W, self.cache = cfg, weights, cache
        self.batch, self.n_q, self.max_workers = batch, n_q, max_workers
        n = batch * n_q
        dev = cache.pool.device
        dt = cfg.torch_dtype
        H = cfg.n_heads
        # An FP8 cache is appended as E4M3 rows; each step expands its visible
        # pages into a bf16 scratch cache (mla_cache_dequant_fp8) that the bf16
        # tensor-core path decodes: `dcfg` / `dcache` are what the queries, the
        # decode and the projections see.
        self.dcfg, self.dcache, self.fp8_scratch = cfg, cache, None
        if cfg.fp8_cache and packed_query:
            import dataclasses
            self.dcfg = dataclasses.replace(cfg, fp8_cache=False)
            mb = cache.block_table.shape[1]
            self.fp8_scratch = torch.empty(abi.mla_fp8_scratch_bytes(cfg, batch, mb), dtype=torch.uint8, device=dev)
            self.dcache = abi.fp8_scratch_cache(self.dcfg, self.fp8_scratch, batch, mb)
        cfg = self.dcfg
        # bf16: the absorbed query goes from the projection to the decode in the
        # decode's packed bf16 layout (no fp32 round trip); fp32: q_lat / q_rope
        self.packed = packed_query and abi.mla_query_packed_bytes(cfg, n) > 0
        if self.packed:
            rows = (2 if cfg.split_query else 1) * n
            self.q_packed = torch.empty(rows, H, cfg.d_c + cfg.d_r, dtype=torch.bfloat16, device=dev)
        else:
            self.q_lat = torch.empty(n, H, cfg.d_c, dtype=torch.float32, device=dev)
            self.q_rope = torch.empty(n, H, cfg.d_r, dtype=torch.float32, device=dev)
        self.o_lat = torch.empty(n, H, cfg.d_c, dtype=torch.float32, device=dev)
        self.y = torch.empty(n, cfg.hidden, dtype=dt, device=dev)
        # bf16: the split combine runs inside the W_UV projection (mla_combine_out_proj)
        self.fused_out = cfg.dtype == "bf16" and abi.mla_combine_out_proj_workspace_size(cfg, batch, n_q) > 0
        gemm_ws = max(abi.mla_cache_append_workspace_size(cfg, n), abi.mla_absorb_q_workspace_size(cfg, n),
                      abi.mla_out_proj_workspace_size(cfg, n),
                      abi.mla_combine_out_proj_workspace_size(cfg, batch, n_q) if self.fused_out else 0)
        self.ws_gemm = torch.empty(max(gemm_ws, 256), dtype=torch.uint8, device=dev)
        self.ws_decode = torch.empty(abi.mla_decode_workspace_size(cfg, batch, n_q, max_workers),
                                     dtype=torch.uint8, device=dev)
        # The step's append runs on a second stream beside the query projections
        # (fp64 work next to weight streaming), with a workspace of its own.
        self.side = torch.cuda.Stream(device=dev)
        self.ws_append = torch.empty(max(abi.mla_cache_append_workspace_size(cfg, n), 256), dtype=torch.uint8,
                                     device=dev)

    def _gemm_ws(self, n: int) -> torch.Tensor:
        need = max(abi.mla_cache_append_workspace_size(self.cfg, n), abi.mla_absorb_q_workspace_size(self.cfg, n),
                   abi.mla_out_proj_workspace_size(self.cfg, n))
        if need > self.ws_gemm.numel():
            self.ws_gemm = torch.empty(need, dtype=torch.uint8, device=self.ws_gemm.device)
        return self.ws_gemm

    def append(self, x, seq_idx, pos, stream=None):
        self._gemm_ws(x.shape[0])
        abi.mla_cache_append(self.cfg, x, self.W["W_DKV"], self.W["W_KR"], seq_idx, pos, self.cache,
                             self.ws_gemm, stream)

    def queries(self, x, pos, stream=None):
        W_DQ = self.W.get("W_DQ")
        W_UQ = self.W["W_UQ"] if "W_UQ" in self.W else self.W["W_Q"]
        if self.packed:
            abi.mla_absorb_q_packed(self.dcfg, x, W_DQ, W_UQ, self.W["W_UK"], pos, self.q_packed, self.ws_gemm,
                                    stream)
        else:
            abi.mla_absorb_q(self.dcfg, x, W_DQ, W_UQ, self.W["W_UK"], pos, self.q_lat, self.q_rope,
                             self.ws_gemm, stream)

    def queries_fp32(self):
        """(q_lat, q_rope) of the last step as fp32 tensors (for checks): the
        fp32 outputs, or the packed bf16 rows (plus their remainders in
        split-query mode) widened."""
        if not self.packed:
            return self.q_lat, self.q_rope
        n = self.batch * self.n_q
        q = self.q_packed[:n].float()
        if self.dcfg.split_query:
            q = q + self.q_packed[n:].float()
        return q[..., :self.dcfg.d_c], q[..., self.dcfg.d_c:]

    def append_and_queries(self, x, seq_idx, pos, stream=None, seq_lens=None):
        """The append and the query projections of one step, overlapped: the
        projections go first on ``stream`` (so their CTAs are placed first), the
        append on a side stream; ``stream`` waits for both before returning.
        With ``seq_lens`` (packed-query path) the side stream also computes the
        decode's split plan, and the next ``decode(..., planned=True)`` skips it."""
        main = stream or torch.cuda.current_stream()
        ready = torch.cuda.Event()
        ready.record(main)
        self.queries(x, pos, main)
        self.side.wait_event(ready)
        need = abi.mla_cache_append_workspace_size(self.cfg, x.shape[0])
        if need > self.ws_append.numel():
            self.ws_append = torch.empty(need, dtype=torch.uint8, device=self.ws_append.device)
        abi.mla_cache_append(self.cfg, x, self.W["W_DKV"], self.W["W_KR"], seq_idx, pos, self.cache,
                             self.ws_append, self.side)
        keep = [x, seq_idx, pos]
        if seq_lens is not None and self.packed:
            abi.mla_decode_plan(self.dcfg, self.batch, self.n_q, self.dcache, seq_lens, self.ws_decode,
                                self.max_workers, self.side)
            keep.append(seq_lens)
        done = torch.cuda.Event()
        done.record(self.side)
        main.wait_event(done)
        # keep the inputs alive until the side stream has used them
        for t in keep:
            t.record_stream(self.side)

    def decode(self, seq_lens, stream=None, planned=False):
        """Split-KV decode; ``planned``: the plan is already in the workspace
        (``append_and_queries`` with ``seq_lens``, same sequence lengths)."""
        if self.fp8_scratch is not None:   # this step's visible FP8 pages -> the bf16 scratch cache
            abi.mla_cache_dequant_fp8(self.cfg, self.cache, self.batch, seq_lens, self.fp8_scratch, stream)
        if self.packed and planned:
            abi.mla_decode_packed_planned(self.dcfg, self.q_packed, self.batch, self.n_q, self.dcache, seq_lens,
                                          self.ws_decode, self.max_workers, stream)
        elif self.packed:
            abi.mla_decode_packed(self.dcfg, self.q_packed, self.batch, self.n_q, self.dcache, seq_lens,
                                  self.ws_decode, self.max_workers, stream)
        else:
            abi.mla_decode(self.dcfg, self.q_lat, self.q_rope, self.batch, self.n_q, self.dcache, seq_lens,
                           self.ws_decode, self.max_workers, stream)

    def combine(self, stream=None):
        abi.mla_combine(self.dcfg, self.ws_decode, self.batch, self.n_q, self.o_lat, stream)

    def attend(self, seq_lens, stream=None):
        """Decode, then the latent output ``o_lat`` (merged splits, fp32)."""
        self.decode(seq_lens, stream)
        self.combine(stream)

    def project(self, stream=None, y=None):
        """``y`` from this step's decode: on the bf16 path the split merge runs
        inside the W_UV projection (``o_lat`` is not needed); otherwise from
        ``o_lat`` (after ``combine``)."""
        y = self.y if y is None else y
        if self.fused_out:
            abi.mla_combine_out_proj(self.dcfg, self.ws_decode, self.batch, self.n_q, self.W["W_UV"], self.W["W_O"],
                                     y, self.ws_gemm, self.max_workers, stream)
        else:
            abi.mla_out_proj(self.dcfg, self.o_lat, self.W["W_UV"], self.W["W_O"], y, self.ws_gemm, stream)

    def step(self, x, seq_idx, pos, seq_lens, stream=None, want_o_lat: bool = False) -> torch.Tensor:
        """Device-resident step: returns ``y`` ``[batch * n_q, hidden]`` (a reused buffer).
        ``want_o_lat`` also fills ``self.o_lat`` (always filled on the fp32 path)."""
        self.append_and_queries(x, seq_idx, pos, stream, seq_lens=seq_lens)
        self.decode(seq_lens, stream, planned=self.packed)
        if want_o_lat or not self.fused_out:
            self.combine(stream)
        self.project(stream)
        return self.y

    def capture_step(self, x, seq_idx, pos, seq_lens, want_o_lat: bool = False) -> torch.cuda.CUDAGraph:
        """Record one ``step`` on these device buffers as a CUDA graph: the
        launches (and the side-stream fork and join) are replayed by
        ``graph.replay()`` without host work.  Refill ``x``, ``seq_idx``,
        ``pos`` and ``seq_lens`` in place between replays; ``self.y`` holds the
        result.  One eager step runs first (outside the capture) so that every
        kernel's one-time setup is done; it appends the same rows the replays
        append again."""
        self.step(x, seq_idx, pos, seq_lens, want_o_lat=want_o_lat)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            self.step(x, seq_idx, pos, seq_lens, want_o_lat=want_o_lat)
        return graph

    def run_from_host(self, inputs, y_hosts, between=None, stream=None, copy_stream=None):
        """Several steps over host (pinned) inputs, pipelined.

        ``inputs[k]`` is ``(x, seq_idx, pos, seq_lens)`` on the host for step k;
        step k's ``y`` lands in ``y_hosts[k]``.  The host-to-device copy of step
        k + 1's inputs and the device-to-host copy of step k's ``y`` run on
        ``copy_stream`` while step k computes on ``stream`` (double-buffered
        device inputs and outputs), as a serving loop would overlap them.
        ``between(k)``, if given, runs on ``stream`` before step k's compute.
        Returns the host buffers; the caller synchronises."""
        stream = stream or torch.cuda.current_stream()
        copy_stream = copy_stream or self._copy_stream()
        dev = self.cache.pool.device
        n = len(inputs)
        if n == 0:
            return y_hosts
        shapes = tuple((tuple(t.shape), t.dtype) for t in inputs[0])
        if getattr(self, "_pipe_shapes", None) != shapes:   # kept across calls: work may still be in flight
            self._pipe_bufs = ([[torch.empty_like(t, device=dev) for t in inputs[0]] for _ in range(2)],
                               [torch.empty_like(self.y) for _ in range(2)])
            self._pipe_shapes = shapes
        dbuf, ybuf = self._pipe_bufs
        copy_stream.wait_stream(stream)   # nothing of this call starts before work already queued on stream
        loaded = [torch.cuda.Event() for _ in range(n)]
        computed = [torch.cuda.Event() for _ in range(n)]
        drained = [torch.cuda.Event() for _ in range(n)]

        def load(k):
            with torch.cuda.stream(copy_stream):
                if k >= 2:   # the step that last used this input buffer has finished
                    copy_stream.wait_event(computed[k - 2])
                for d, h in zip(dbuf[k % 2], inputs[k]):
                    d.copy_(h, non_blocking=True)
                loaded[k].record(copy_stream)

        load(0)
        for k in range(n):
            if k + 1 < n:
                load(k + 1)
            stream.wait_event(loaded[k])
            if k >= 2:       # the y buffer of step k - 2 has been copied out
                stream.wait_event(drained[k - 2])
            if between is not None:
                between(k)
            x, seq_idx, pos, seq_lens = dbuf[k % 2]
            self.append_and_queries(x, seq_idx, pos, stream, seq_lens=seq_lens)
            self.decode(seq_lens, stream, planned=self.packed)
            if not self.fused_out:
                self.combine(stream)
            self.project(stream, y=ybuf[k % 2])
            computed[k].record(stream)
            with torch.cuda.stream(copy_stream):
                copy_stream.wait_event(computed[k])
                y_hosts[k].copy_(ybuf[k % 2], non_blocking=True)
                drained[k].record(copy_stream)
        stream.wait_event(drained[n - 1])
        return y_hosts

    def _copy_stream(self):
        if getattr(self, "_copies", None) is None:
            self._copies = torch.cuda.Stream(device=self.cache.pool.device)
        return self._copies

    def step_from_host(self, x_host, seq_idx_host, pos_host, seq_lens_host, y_host,
                       stream: Optional[torch.cuda.Stream] = None):
        """Same step with host (pinned) inputs and output; copies are on ``stream``."""
        stream = stream or torch.cuda.current_stream()
        with torch.cuda.stream(stream):
            dev = self.cache.pool.device
            x = x_host.to(dev, non_blocking=True)
            seq_idx = seq_idx_host.to(dev, non_blocking=True)
            pos = pos_host.to(dev, non_blocking=True)
            seq_lens = seq_lens_host.to(dev, non_blocking=True)
            y = self.step(x, seq_idx, pos, seq_lens, stream)
            y_host.copy_(y, non_blocking=True)
        return y_host
