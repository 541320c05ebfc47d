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
                 batch: int, n_q: int, max_workers: int = 0):
        self.cfg, self.W, self.cache = cfg, weights, cache
        self.batch, self.n_q, self.max_workers = batch, n_q, max_workers
        n = batch * n_q
        dev = cache.pool.device
        dt = cfg.torch_dtype
        H = cfg.n_heads
        self.q_lat = torch.empty(n, H, cfg.d_c, dtype=torch.float32, device=dev)
        self.q_rope = torch.empty(n, H, cfg.d_r, dtype=torch.float32, device=dev)
        self.o_lat = torch.empty(n, H, cfg.d_c, dtype=torch.float32, device=dev)
        self.y = torch.empty(n, cfg.hidden, dtype=dt, device=dev)
        gemm_ws = max(abi.mla_cache_append_workspace_size(cfg, n), abi.mla_absorb_q_workspace_size(cfg, n),
                      abi.mla_out_proj_workspace_size(cfg, n))
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
        abi.mla_absorb_q(self.cfg, x, W_DQ, W_UQ, self.W["W_UK"], pos, self.q_lat, self.q_rope,
                         self.ws_gemm, stream)

    def append_and_queries(self, x, seq_idx, pos, stream=None):
        """The append and the query projections of one step, overlapped: the
        projections go first on ``stream`` (so their CTAs are placed first), the
        append on a side stream; ``stream`` waits for both before returning."""
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
        done = torch.cuda.Event()
        done.record(self.side)
        main.wait_event(done)
        # keep the inputs alive until the side stream has used them
        for t in (x, seq_idx, pos):
            t.record_stream(self.side)

    def decode(self, seq_lens, stream=None):
        abi.mla_decode(self.cfg, self.q_lat, self.q_rope, self.batch, self.n_q, self.cache, seq_lens,
                       self.ws_decode, self.max_workers, stream)

    def combine(self, stream=None):
        abi.mla_combine(self.cfg, self.ws_decode, self.batch, self.n_q, self.o_lat, stream)

    def attend(self, seq_lens, stream=None):
        self.decode(seq_lens, stream)
        self.combine(stream)

    def project(self, stream=None):
        abi.mla_out_proj(self.cfg, self.o_lat, self.W["W_UV"], self.W["W_O"], self.y, self.ws_gemm, stream)

    def step(self, x, seq_idx, pos, seq_lens, stream=None) -> torch.Tensor:
        """Device-resident step: returns ``y`` ``[batch * n_q, hidden]`` (a reused buffer)."""
        self.append_and_queries(x, seq_idx, pos, stream)
        self.attend(seq_lens, stream)
        self.project(stream)
        return self.y

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
