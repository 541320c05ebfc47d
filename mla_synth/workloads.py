"""Named MLA decode workloads and their seeded generator.

Shapes follow the DeepSeek-V2/V3 dimensions the pages quote for the latent
cache (kv_lora_rank 512 + rope dim 64 = 576 values per token per layer:
"GQA, MQA ve MLA", section "Multi-head latent attention (MLA)"), plus a tiny
fp32 shape that the fp64 oracle finishes in milliseconds.

Draw order for one workload, all from one CPU ``torch.Generator`` seeded
with ``workload.seed`` (fixed so that every consumer sees identical values):

1. weights, in the order W_DKV, W_KR, (W_DQ, W_UQ) or W_Q, W_UK, W_UV, W_O;
   each ``randn(fan_in, fan_out) * fan_in ** -0.5`` in fp32, then rounded to
   the workload dtype (round-to-nearest-even for bf16);
2. the cached context lengths (``randint(lo, hi + 1, (batch,))`` when ragged);
3. the new tokens' hidden states ``x_new`` ``[batch * n_q, hidden]``, N(0, 1);
4. the cached rows: either hidden states ``x_cached`` ``[L, hidden]`` whose
   latent rows the append step produces (tiny shape), or latent rows
   ``[sum L_b, d_c + d_r]`` drawn N(0, 1) directly, optionally with a
   Bernoulli(frac) subset of rows scaled by ``spike_scale``;
5. the physical block permutation of the paged pool (``randperm``), when
   the workload asks for shuffled blocks;
6. for an FP8 cache (``fp8_cache``), instead of step 4's latent rows: E4M3
   codes ``[sum L_b, d_c + d_r]`` (sign uniform; exponent field 6..15 drawn
   with the octave shares of a normal row whose 4-sigma value sits at 448;
   mantissa field uniform; never the NaN pattern) and one scale per row, a
   power of two as the format has it, ``2^k`` with k uniform in -8..-7
   (rows of one layer have similar norms, so their maxima, and with them
   the power-of-two scales, differ by about a factor of two).
   They are drawn after step 5, as codes are stored bytes, not values.
"""

from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field
from typing import Dict, Optional, Sequence, Tuple

import torch


@dataclass(frozen=True)
class MLAShape:
    """Per-layer MLA dimensions (row-vector convention, weights ``[in, out]``)."""

    name: str
    hidden: int
    n_heads: int
    d_c: int          # joint KV latent width (kv_lora_rank)
    d_r: int          # decoupled RoPE key width, shared by all heads
    qk_nope: int      # per-head no-position query/key width
    v_head: int       # per-head value width
    q_lora: int       # 0: queries are projected directly by W_Q
    rope_theta: float = 10000.0
    dtype: str = "bf16"  # "bf16" or "f32": storage type of weights, cache and activations
    block_size: int = 64

    @property
    def row(self) -> int:
        return self.d_c + self.d_r

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    @property
    def elem_bytes(self) -> int:
        return 2 if self.dtype == "bf16" else 4

    def weight_shapes(self) -> Dict[str, Tuple[int, int]]:
        """Weight name -> (fan_in, fan_out), in draw order."""
        H = self.n_heads
        q_width = H * (self.qk_nope + self.d_r)
        shapes = {
            "W_DKV": (self.hidden, self.d_c),
            "W_KR": (self.hidden, self.d_r),
        }
        if self.q_lora > 0:
            shapes["W_DQ"] = (self.hidden, self.q_lora)
            shapes["W_UQ"] = (self.q_lora, q_width)
        else:
            shapes["W_Q"] = (self.hidden, q_width)
        # W_UK and W_UV map the latent (fan_in d_c) to per-head key / value.
        shapes["W_UK"] = (self.d_c, H * self.qk_nope)
        shapes["W_UV"] = (self.d_c, H * self.v_head)
        shapes["W_O"] = (H * self.v_head, self.hidden)
        return shapes


SHAPES: Dict[str, MLAShape] = {
    "tiny": MLAShape("tiny", hidden=256, n_heads=4, d_c=64, d_r=16, qk_nope=32,
                     v_head=32, q_lora=0, dtype="f32"),
    "v2": MLAShape("v2", hidden=5120, n_heads=128, d_c=512, d_r=64, qk_nope=128,
                   v_head=128, q_lora=1536, dtype="bf16"),
    "v3": MLAShape("v3", hidden=7168, n_heads=128, d_c=512, d_r=64, qk_nope=128,
                   v_head=128, q_lora=1536, dtype="bf16"),
}


@dataclass(frozen=True)
class Workload:
    """One decode step over a batch of sequences.

    ``lengths`` fixes the cached context length of every sequence; when it is
    ``None`` the lengths are drawn uniformly from ``[len_lo, len_hi]``.  Each
    sequence then appends ``n_q`` new latent rows (positions ``L_b .. L_b +
    n_q - 1``) and each new token attends causally, itself included.
    """

    name: str
    shape: MLAShape
    batch: int
    n_q: int = 1
    lengths: Optional[Tuple[int, ...]] = None
    len_lo: int = 0
    len_hi: int = 0
    cached_from_append: bool = False   # cached rows come from x_cached via the append step
    shuffled_blocks: bool = False
    spike_frac: float = 0.0
    spike_scale: float = 1.0
    seed: int = 0
    description: str = ""
    # run option, not data: hold the query as a bf16 hi + lo pair in the decode
    # (strongly peaked softmaxes need more than bf16's 8 significant bits)
    split_query: bool = False
    # the cache holds E4M3 codes and one fp32 scale per row (weights stay bf16)
    fp8_cache: bool = False

    @property
    def cache_row_bytes(self) -> int:
        """Bytes of one cached row (with its scale for an FP8 cache)."""
        return self.shape.row + 4 if self.fp8_cache else self.shape.row * self.shape.elem_bytes

    @property
    def n_tok(self) -> int:
        return self.batch * self.n_q


WORKLOADS: Dict[str, Workload] = {
    "tiny_f32_b1_l128": Workload(
        "tiny_f32_b1_l128", SHAPES["tiny"], batch=1, n_q=1, lengths=(128,),
        cached_from_append=True,
        description="tiny fp32 MLA, 1 layer, 128 cached tokens + 1 decode token"),
    "v2_b16_l4096": Workload(
        "v2_b16_l4096", SHAPES["v2"], batch=16, n_q=1, lengths=(4096,) * 16,
        description="DeepSeek-V2-shaped decode, batch 16 x 4096 cached tokens, 1 new token each"),
    "v3_b64_ragged1k_8k": Workload(
        "v3_b64_ragged1k_8k", SHAPES["v3"], batch=64, n_q=1, len_lo=1024, len_hi=8192,
        shuffled_blocks=True,
        description="DeepSeek-V3-shaped decode, batch 64, ragged lengths U[1024, 8192], "
                    "64-token pages in shuffled order"),
    "v3_b4_long": Workload(
        "v3_b4_long", SHAPES["v3"], batch=4, n_q=1, lengths=(65536, 131072, 32768, 100000),
        spike_frac=0.01, spike_scale=8.0, split_query=True,
        description="V3-shaped long-context split-KV stress, contexts 65536/131072/32768/100000, "
                    "1% of latent rows scaled x8"),
    "v3_fp8_b64_ragged1k_8k": Workload(
        "v3_fp8_b64_ragged1k_8k", SHAPES["v3"], batch=64, n_q=1, len_lo=1024, len_hi=8192,
        shuffled_blocks=True, fp8_cache=True,
        description="the batch-64 V3 decode over an FP8 latent cache (E4M3 codes + fp32 row scale), "
                    "ragged lengths U[1024, 8192], 64-token pages in shuffled order"),
    "v3_b128_nq2_ragged512_16k": Workload(
        "v3_b128_nq2_ragged512_16k", SHAPES["v3"], batch=128, n_q=2, len_lo=512, len_hi=16384,
        description="V3-shaped multi-token decode, batch 128, 2 causal query tokens per sequence, "
                    "ragged lengths U[512, 16384], append 2 rows then attend"),
    "v3_prefill_b8_c64_ragged1k_4k": Workload(
        "v3_prefill_b8_c64_ragged1k_4k", SHAPES["v3"], batch=8, n_q=64, len_lo=1024, len_hi=4096,
        shuffled_blocks=True,
        description="V3-shaped chunked prefill over the latent cache, batch 8, a 64-token chunk per "
                    "sequence (appended, then each token attends causally), ragged cached lengths "
                    "U[1024, 4096], 64-token pages in shuffled order"),
}


def reduced(wl: Workload, *, batch: Optional[int] = None,
            lengths: Optional[Sequence[int]] = None,
            len_lo: Optional[int] = None, len_hi: Optional[int] = None,
            n_q: Optional[int] = None, seed: Optional[int] = None,
            name: Optional[str] = None) -> Workload:
    """The same shape and structure at a smaller batch / context size."""
    kw = {}
    if lengths is not None:
        kw["lengths"] = tuple(int(v) for v in lengths)
        kw["batch"] = len(kw["lengths"])
    if batch is not None:
        kw["batch"] = batch
        if lengths is None and wl.lengths is not None:
            base = wl.lengths
            kw["lengths"] = tuple(base[i % len(base)] for i in range(batch))
    if len_lo is not None:
        kw["len_lo"] = len_lo
    if len_hi is not None:
        kw["len_hi"] = len_hi
    if n_q is not None:
        kw["n_q"] = n_q
    if seed is not None:
        kw["seed"] = seed
    kw["name"] = name or (wl.name + "_reduced")
    return dataclasses.replace(wl, **kw)


@dataclass
class WorkloadData:
    """Seeded inputs of one workload, as CPU tensors in the workload dtype."""

    workload: Workload
    weights: Dict[str, torch.Tensor]
    cached_len: torch.Tensor              # int64 [B]: rows already in the cache
    x_new: torch.Tensor                   # [B*n_q, hidden], row b*n_q + j is token j of seq b
    cached_rows: Optional[torch.Tensor]   # [sum L_b, d_c + d_r] latent rows (None if from append or FP8)
    x_cached: Optional[torch.Tensor]      # [sum L_b, hidden] (only when cached_from_append)
    spike_mask: Optional[torch.Tensor]    # bool [sum L_b] rows scaled by spike_scale
    block_table: torch.Tensor             # int32 [B, max_blocks]
    num_blocks: int
    row_offsets: torch.Tensor = field(default=None)  # int64 [B+1] start of seq b in cached rows
    cached_codes: Optional[torch.Tensor] = None      # uint8 [sum L_b, d_c + d_r] E4M3 codes (FP8 cache)
    cached_scale: Optional[torch.Tensor] = None      # float32 [sum L_b] their row scales

    @property
    def seq_lens(self) -> torch.Tensor:
        """Rows per sequence after the append step (cached + new)."""
        return self.cached_len + self.workload.n_q

    def new_positions(self) -> torch.Tensor:
        """int32 [B*n_q]: absolute position of each new token (0-based)."""
        n_q = self.workload.n_q
        j = torch.arange(n_q, dtype=torch.int64)
        return (self.cached_len[:, None] + j[None, :]).reshape(-1).to(torch.int32)

    def new_seq_idx(self) -> torch.Tensor:
        """int32 [B*n_q]: sequence index of each new token."""
        n_q = self.workload.n_q
        return torch.arange(self.workload.batch, dtype=torch.int32).repeat_interleave(n_q)

    def seq_rows(self, b: int) -> torch.Tensor:
        """Cached latent rows of sequence b (before the append step)."""
        s, e = int(self.row_offsets[b]), int(self.row_offsets[b + 1])
        return self.cached_rows[s:e]


def _draw_weights(shape: MLAShape, g: torch.Generator) -> Dict[str, torch.Tensor]:
    out = {}
    for name, (fan_in, fan_out) in shape.weight_shapes().items():
        w = torch.randn(fan_in, fan_out, generator=g, dtype=torch.float32)
        w.mul_(fan_in ** -0.5)
        out[name] = w.to(shape.torch_dtype)
    return out


def _draw_rows(n: int, width: int, dtype: torch.dtype, g: torch.Generator,
               chunk: int = 1 << 20) -> torch.Tensor:
    """N(0, 1) rows drawn in row chunks (bounded fp32 temporaries)."""
    out = torch.empty(n, width, dtype=dtype)
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        out[s:e] = torch.randn(e - s, width, generator=g, dtype=torch.float32).to(dtype)
    return out


# Share of the octaves [2^(e-7), 2^(e-6)) of |N(0, 1)| * 112 for exponent
# fields e = 6 .. 15 (the lowest bin also takes everything below it, the top
# one everything above 256): the magnitudes of a normal row whose 4-sigma
# value is scaled to 448.
_FP8_EXPONENT_WEIGHTS = (0.013, 0.007, 0.014, 0.028, 0.056, 0.11, 0.20, 0.32, 0.23, 0.022)


def generate(wl: Workload, *, with_weights: bool = True) -> WorkloadData:
    """Draw every input of ``wl`` from its seed (see the module docstring)."""
    shape = wl.shape
    g = torch.Generator().manual_seed(wl.seed)
    dt = shape.torch_dtype

    weights: Dict[str, torch.Tensor] = {}
    if with_weights:
        weights = _draw_weights(shape, g)
    else:
        # Keep the stream aligned with the with-weights draw order.
        for _name, (fan_in, fan_out) in shape.weight_shapes().items():
            torch.randn(fan_in, fan_out, generator=g, dtype=torch.float32)

    if wl.lengths is not None:
        if len(wl.lengths) != wl.batch:
            raise ValueError("lengths must have one entry per sequence")
        cached_len = torch.tensor(wl.lengths, dtype=torch.int64)
    else:
        cached_len = torch.randint(wl.len_lo, wl.len_hi + 1, (wl.batch,), generator=g,
                                   dtype=torch.int64)

    x_new = torch.randn(wl.n_tok, shape.hidden, generator=g, dtype=torch.float32).to(dt)

    total = int(cached_len.sum())
    row_offsets = torch.zeros(wl.batch + 1, dtype=torch.int64)
    row_offsets[1:] = torch.cumsum(cached_len, 0)
    cached_rows = x_cached = spike_mask = None
    if wl.cached_from_append:
        x_cached = torch.randn(total, shape.hidden, generator=g, dtype=torch.float32).to(dt)
    elif wl.fp8_cache:
        pass  # codes and scales after the block table (step 6)
    else:
        cached_rows = _draw_rows(total, shape.row, dt, g)
        if wl.spike_frac > 0.0:
            spike_mask = torch.rand(total, generator=g) < wl.spike_frac
            idx = spike_mask.nonzero().squeeze(1)
            cached_rows[idx] = (cached_rows[idx].to(torch.float32) * wl.spike_scale).to(dt)

    bs = shape.block_size
    blocks_per_seq = (cached_len + wl.n_q + bs - 1) // bs
    num_blocks = int(blocks_per_seq.sum())
    max_blocks = int(blocks_per_seq.max()) if wl.batch > 0 else 1
    logical = torch.arange(num_blocks, dtype=torch.int64)
    if wl.shuffled_blocks:
        physical = torch.randperm(num_blocks, generator=g)
    else:
        physical = logical
    block_table = torch.full((wl.batch, max(max_blocks, 1)), -1, dtype=torch.int32)
    start = 0
    for b in range(wl.batch):
        nb = int(blocks_per_seq[b])
        block_table[b, :nb] = physical[start:start + nb].to(torch.int32)
        start += nb

    codes = scales = None
    if wl.fp8_cache and not wl.cached_from_append:
        sign = torch.randint(0, 2, (total, shape.row), generator=g, dtype=torch.int32)
        # exponent field 6..15 with the octave weights of |N(0, 1)| scaled so
        # that 4 sigma lands on the largest code (a row quantised with its own
        # max): most codes in [32, 256), a few percent at the top
        octaves = torch.tensor(_FP8_EXPONENT_WEIGHTS, dtype=torch.float64)
        expo = 6 + torch.multinomial(octaves, total * shape.row, replacement=True, generator=g)
        expo = expo.view(total, shape.row).to(torch.int32)
        mant = torch.randint(0, 8, (total, shape.row), generator=g, dtype=torch.int32)
        mant = torch.where((expo == 15) & (mant == 7), torch.full_like(mant, 6), mant)   # 0x7F / 0xFF: NaN
        codes = ((sign << 7) | (expo << 3) | mant).to(torch.uint8)
        scales = torch.pow(2.0, torch.randint(-8, -6, (total,), generator=g).to(torch.float32))

    return WorkloadData(wl, weights, cached_len, x_new, cached_rows, x_cached, spike_mask,
                        block_table, num_blocks, row_offsets, codes, scales)


def build_pool(data: WorkloadData, rows: Optional[torch.Tensor] = None,
               fill: float = float("nan")) -> torch.Tensor:
    """Scatter cached latent rows into a paged pool ``[num_blocks, block, d_c + d_r]``.

    Pure data movement: row ``t`` of sequence ``b`` goes to
    ``pool[block_table[b, t // block], t % block]``.  Slots no sequence has
    written yet keep ``fill`` (NaN by default), so a consumer that reads past
    a sequence's valid rows is caught.
    """
    wl = data.workload
    shape = wl.shape
    bs = shape.block_size
    if wl.fp8_cache:   # E4M3 codes; unwritten slots hold the NaN code 0x7F
        src = data.cached_codes if rows is None else rows
        pool = torch.full((max(data.num_blocks, 1), bs, shape.row), 0x7F, dtype=torch.uint8)
        return _scatter(data, pool, src)
    src = data.cached_rows if rows is None else rows
    pool = torch.full((max(data.num_blocks, 1), bs, shape.row), fill, dtype=shape.torch_dtype)
    return _scatter(data, pool, src)


def _scatter(data: WorkloadData, pool: torch.Tensor, src: Optional[torch.Tensor]) -> torch.Tensor:
    """Row ``t`` of sequence ``b`` of ``src`` -> ``pool[block_table[b, t // block], t % block]``."""
    wl = data.workload
    bs = wl.shape.block_size
    flat = pool.view(pool.shape[0] * pool.shape[1], *pool.shape[2:])
    if src is None:          # rows are produced later by the append step
        return pool
    for b in range(wl.batch):
        L = int(data.cached_len[b])
        if L == 0:
            continue
        t = torch.arange(L, dtype=torch.int64)
        phys = data.block_table[b].to(torch.int64)[t // bs]
        dst = phys * bs + (t % bs)
        s = int(data.row_offsets[b])
        flat[dst] = src[s:s + L]
    return pool


def build_row_scale(data: WorkloadData) -> Optional[torch.Tensor]:
    """FP8 cache: the rows' scales in the pool's layout ``[num_blocks, block]``
    (unwritten slots NaN); None for other caches."""
    if not data.workload.fp8_cache:
        return None
    bs = data.workload.shape.block_size
    scale = torch.full((max(data.num_blocks, 1), bs), float("nan"), dtype=torch.float32)
    return _scatter(data, scale, data.cached_scale)


def device_inputs(data: WorkloadData, device, pool: Optional[torch.Tensor] = None) -> Dict[str, object]:
    """Copies of the seeded inputs on ``device`` (pure data movement)."""
    dev = torch.device(device)
    out: Dict[str, object] = {
        "weights": {k: v.to(dev) for k, v in data.weights.items()},
        "pool": (build_pool(data) if pool is None else pool).to(dev),
        "block_table": data.block_table.to(dev),
        "seq_lens": data.seq_lens.to(torch.int32).to(dev),
        "x_new": data.x_new.to(dev),
        "pos": data.new_positions().to(dev),
        "seq_idx": data.new_seq_idx().to(dev),
        "row_scale": None if not data.workload.fp8_cache else build_row_scale(data).to(dev),
    }
    if data.x_cached is not None:
        L = int(data.cached_len.sum())
        out["x_cached"] = data.x_cached.to(dev)
        out["pos_cached"] = torch.cat([torch.arange(int(n), dtype=torch.int32)
                                       for n in data.cached_len]).to(dev) if L else None
        out["seq_idx_cached"] = torch.arange(data.workload.batch, dtype=torch.int32).repeat_interleave(
            data.cached_len).to(dev)
    return out
