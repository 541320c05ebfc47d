"""ctypes binding of libmla.so (argument marshalling only).

Each function here has the name of the C entry point it wraps, takes torch
tensors that already live on the current CUDA device, checks their dtype,
shape and contiguity, and passes raw pointers and sizes to the library.  No
arithmetic of the method happens in Python, and there is no fallback: if
the shared library is missing the import fails.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from pathlib import Path
from typing import Optional

import torch

_LIB_PATH = Path(__file__).resolve().parent / "libmla.so"

MLA_OK = 0
MLA_ERR_INVALID_ARG = -1
MLA_ERR_UNSUPPORTED = -2
MLA_ERR_CUDA = -3
MLA_ERR_BOUNDS = -4
MLA_ERR_TIMEOUT = -5
MLA_ERR_WORKSPACE = -6
MLA_F32 = 0
MLA_BF16 = 1
MLA_FLAG_SPLIT_QUERY = 1
MLA_FLAG_FP8_CACHE = 2
MLA_APPEND_NOALLOC_SCRATCH_BYTES = 4 << 20

# Every symbol the header declares, with (restype, argtypes).
_vp, _i32, _sz, _d, _f = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t, ctypes.c_double, ctypes.c_float


class MLAConfig(ctypes.Structure):
    """Mirror of ``mla_config``."""

    _fields_ = [("hidden", _i32), ("n_heads", _i32), ("d_c", _i32), ("d_r", _i32),
                ("qk_nope", _i32), ("v_head", _i32), ("q_lora", _i32),
                ("rope_theta", _d), ("softmax_scale", _f), ("block_size", _i32),
                ("dtype", _i32), ("flags", _i32)]


class MLACache(ctypes.Structure):
    """Mirror of ``mla_cache``."""

    _fields_ = [("pool", _vp), ("num_blocks", _i32), ("block_table", _vp), ("batch", _i32),
                ("max_blocks_per_seq", _i32), ("row_scale", _vp)]


_P_CFG = ctypes.POINTER(MLAConfig)
_P_CACHE = ctypes.POINTER(MLACache)

SIGNATURES = {
    "mla_abi_version": (_i32, []),
    "mla_kernel_launches": (ctypes.c_int64, []),
    "mla_status_string": (ctypes.c_char_p, [_i32]),
    "mla_cache_append_workspace_size": (_sz, [_P_CFG, _i32]),
    "mla_cache_append": (_i32, [_P_CFG, _vp, _i32, _vp, _vp, _vp, _vp, _P_CACHE, _vp, _sz, _vp]),
    "mla_cache_append_noalloc": (_i32, [_P_CFG, _vp, _i32, _vp, _vp, _vp, _vp, _P_CACHE, _vp]),
    "mla_absorb_q_workspace_size": (_sz, [_P_CFG, _i32]),
    "mla_absorb_q": (_i32, [_P_CFG, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "mla_query_packed_bytes": (_sz, [_P_CFG, _i32]),
    "mla_fp8_scratch_bytes": (_sz, [_P_CFG, _i32, _i32]),
    "mla_cache_dequant_fp8": (_i32, [_P_CFG, _P_CACHE, _i32, _vp, _vp, _sz, _vp]),
    "mla_absorb_q_packed": (_i32, [_P_CFG, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "mla_decode_packed": (_i32, [_P_CFG, _vp, _i32, _i32, _P_CACHE, _vp, _i32, _vp, _sz, _vp]),
    "mla_decode_packed_planned": (_i32, [_P_CFG, _vp, _i32, _i32, _P_CACHE, _vp, _i32, _vp, _sz, _vp]),
    "mla_decode_plan": (_i32, [_P_CFG, _i32, _i32, _P_CACHE, _vp, _i32, _vp, _sz, _vp]),
    "mla_decode_workspace_size": (_sz, [_P_CFG, _i32, _i32, _i32]),
    "mla_decode": (_i32, [_P_CFG, _vp, _vp, _i32, _i32, _P_CACHE, _vp, _i32, _vp, _sz, _vp]),
    "mla_combine": (_i32, [_P_CFG, _vp, _sz, _i32, _i32, _vp, _vp]),
    "mla_combine_lse": (_i32, [_P_CFG, _vp, _sz, _i32, _i32, _vp, _vp, _vp]),
    "mla_merge_shards": (_i32, [_P_CFG, _i32, _i32, _vp, _vp, _vp, _vp, _vp]),
    "mla_combine_out_proj_workspace_size": (_sz, [_P_CFG, _i32, _i32]),
    "mla_combine_out_proj": (_i32, [_P_CFG, _vp, _sz, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _sz, _vp]),
    "mla_out_proj_workspace_size": (_sz, [_P_CFG, _i32]),
    "mla_out_proj": (_i32, [_P_CFG, _vp, _i32, _vp, _vp, _vp, _vp, _sz, _vp]),
    "mla_get_device_error": (_i32, [_vp, ctypes.POINTER(_i32)]),
    "mla_check_wait_timeout": (_i32, [ctypes.c_int64, _vp]),
}


def load_library(path: Optional[os.PathLike] = None) -> ctypes.CDLL:
    p = Path(path) if path is not None else _LIB_PATH
    if not p.exists():
        raise ImportError(f"libmla.so not built at {p}; run `python -m mla_latent_kv_39_b200.build`")
    lib = ctypes.CDLL(str(p))
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = load_library()
    return _lib


class MLAError(RuntimeError):
    def __init__(self, status: int, where: str, detail=None):
        msg = lib().mla_status_string(status).decode()
        super().__init__(f"{where}: {msg} (status {status})" + (f" detail={detail}" if detail else ""))
        self.status = status
        self.detail = detail


def _check(status: int, where: str):
    if status != MLA_OK:
        raise MLAError(status, where)


# --------------------------------------------------------------- config

@dataclass(frozen=True)
class Config:
    hidden: int
    n_heads: int
    d_c: int
    d_r: int
    qk_nope: int
    v_head: int
    q_lora: int
    rope_theta: float = 10000.0
    softmax_scale: float = 0.0
    block_size: int = 64
    dtype: str = "bf16"
    split_query: bool = False
    fp8_cache: bool = False       # E4M3 cache rows with one fp32 scale each (bf16 weights)

    @staticmethod
    def from_shape(shape, split_query: bool = False, fp8_cache: bool = False) -> "Config":
        return Config(shape.hidden, shape.n_heads, shape.d_c, shape.d_r, shape.qk_nope,
                      shape.v_head, shape.q_lora, float(shape.rope_theta), 0.0,
                      shape.block_size, shape.dtype, split_query, fp8_cache)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    @property
    def cache_torch_dtype(self) -> torch.dtype:
        """Element type of the cache pool (uint8 E4M3 codes for an FP8 cache)."""
        return torch.uint8 if self.fp8_cache else self.torch_dtype

    def c(self) -> MLAConfig:
        return MLAConfig(self.hidden, self.n_heads, self.d_c, self.d_r, self.qk_nope, self.v_head,
                         self.q_lora, self.rope_theta, self.softmax_scale, self.block_size,
                         MLA_BF16 if self.dtype == "bf16" else MLA_F32,
                         (MLA_FLAG_SPLIT_QUERY if self.split_query else 0)
                         | (MLA_FLAG_FP8_CACHE if self.fp8_cache else 0))


class Cache:
    """A paged latent cache: pool ``[num_blocks, block, d_c + d_r]`` + block table
    (+ ``row_scale`` float32 ``[num_blocks, block]`` for an FP8 pool of E4M3 codes)."""

    def __init__(self, pool: torch.Tensor, block_table: torch.Tensor, row_scale: Optional[torch.Tensor] = None):
        _need(pool, "pool", ndim=3)
        _need(block_table, "block_table", dtype=torch.int32, ndim=2)
        if row_scale is not None:
            _need(row_scale, "row_scale", dtype=torch.float32, shape=tuple(pool.shape[:2]))
        self.pool, self.block_table, self.row_scale = pool, block_table, row_scale
        self.c = MLACache(pool.data_ptr(), pool.shape[0], block_table.data_ptr(),
                          block_table.shape[0], block_table.shape[1],
                          None if row_scale is None else row_scale.data_ptr())


def _need(t: torch.Tensor, name: str, dtype=None, ndim=None, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


# --------------------------------------------------------------- sizes

def mla_cache_append_workspace_size(cfg: Config, n_tok: int) -> int:
    return lib().mla_cache_append_workspace_size(ctypes.byref(cfg.c()), n_tok)


def mla_absorb_q_workspace_size(cfg: Config, n_tok: int) -> int:
    return lib().mla_absorb_q_workspace_size(ctypes.byref(cfg.c()), n_tok)


def mla_decode_workspace_size(cfg: Config, batch: int, n_q: int, max_workers: int = 0) -> int:
    return lib().mla_decode_workspace_size(ctypes.byref(cfg.c()), batch, n_q, max_workers)


def mla_out_proj_workspace_size(cfg: Config, n_tok: int) -> int:
    return lib().mla_out_proj_workspace_size(ctypes.byref(cfg.c()), n_tok)


# --------------------------------------------------------------- the five steps

def mla_cache_append(cfg: Config, x, W_DKV, W_KR, seq_idx, pos, cache: Cache, workspace, stream=None):
    dt = cfg.torch_dtype
    n = x.shape[0]
    _need(x, "x", dt, shape=(n, cfg.hidden))
    _need(W_DKV, "W_DKV", dt, shape=(cfg.hidden, cfg.d_c))
    _need(W_KR, "W_KR", dt, shape=(cfg.hidden, cfg.d_r))
    _need(seq_idx, "seq_idx", torch.int32, shape=(n,))
    _need(pos, "pos", torch.int32, shape=(n,))
    _need(workspace, "workspace", torch.uint8)
    if cache.pool.dtype != cfg.cache_torch_dtype or cache.pool.shape[1:] != (cfg.block_size, cfg.d_c + cfg.d_r):
        raise ValueError("cache pool dtype/shape does not match the config")
    _check(lib().mla_cache_append(ctypes.byref(cfg.c()), _ptr(x), n, _ptr(W_DKV), _ptr(W_KR),
                                  _ptr(seq_idx), _ptr(pos), ctypes.byref(cache.c), _ptr(workspace),
                                  workspace.numel(), _stream(stream)), "mla_cache_append")


def mla_cache_append_noalloc(cfg: Config, x, W_DKV, W_KR, seq_idx, pos, cache: Cache, stream=None):
    """mla_cache_append without a caller workspace, for callers that cannot
    allocate device memory: the scratch is the library's fixed device array
    (shared by all calls on a device; overlapping calls race)."""
    dt = cfg.torch_dtype
    n = x.shape[0]
    _need(x, "x", dt, shape=(n, cfg.hidden))
    _need(W_DKV, "W_DKV", dt, shape=(cfg.hidden, cfg.d_c))
    _need(W_KR, "W_KR", dt, shape=(cfg.hidden, cfg.d_r))
    _need(seq_idx, "seq_idx", torch.int32, shape=(n,))
    _need(pos, "pos", torch.int32, shape=(n,))
    if cache.pool.dtype != cfg.cache_torch_dtype or cache.pool.shape[1:] != (cfg.block_size, cfg.d_c + cfg.d_r):
        raise ValueError("cache pool dtype/shape does not match the config")
    _check(lib().mla_cache_append_noalloc(ctypes.byref(cfg.c()), _ptr(x), n, _ptr(W_DKV), _ptr(W_KR),
                                          _ptr(seq_idx), _ptr(pos), ctypes.byref(cache.c),
                                          _stream(stream)), "mla_cache_append_noalloc")


def mla_absorb_q(cfg: Config, x, W_DQ, W_UQ, W_UK, pos, q_lat, q_rope, workspace, stream=None):
    dt = cfg.torch_dtype
    n = x.shape[0]
    H = cfg.n_heads
    _need(x, "x", dt, shape=(n, cfg.hidden))
    if cfg.q_lora > 0:
        _need(W_DQ, "W_DQ", dt, shape=(cfg.hidden, cfg.q_lora))
        _need(W_UQ, "W_UQ", dt, shape=(cfg.q_lora, H * (cfg.qk_nope + cfg.d_r)))
    else:
        if W_DQ is not None:
            raise ValueError("W_DQ must be None without query compression")
        _need(W_UQ, "W_Q", dt, shape=(cfg.hidden, H * (cfg.qk_nope + cfg.d_r)))
    _need(W_UK, "W_UK", dt, shape=(cfg.d_c, H * cfg.qk_nope))
    _need(pos, "pos", torch.int32, shape=(n,))
    _need(q_lat, "q_lat", torch.float32, shape=(n, H, cfg.d_c))
    _need(q_rope, "q_rope", torch.float32, shape=(n, H, cfg.d_r))
    _need(workspace, "workspace", torch.uint8)
    _check(lib().mla_absorb_q(ctypes.byref(cfg.c()), _ptr(x), n, _ptr(W_DQ), _ptr(W_UQ), _ptr(W_UK),
                              _ptr(pos), _ptr(q_lat), _ptr(q_rope), _ptr(workspace), workspace.numel(),
                              _stream(stream)), "mla_absorb_q")


def mla_query_packed_bytes(cfg: Config, n_tok: int) -> int:
    return int(lib().mla_query_packed_bytes(ctypes.byref(cfg.c()), n_tok))


def mla_absorb_q_packed(cfg: Config, x, W_DQ, W_UQ, W_UK, pos, q_packed, workspace, stream=None):
    dt = cfg.torch_dtype
    n = x.shape[0]
    H = cfg.n_heads
    _need(x, "x", dt, shape=(n, cfg.hidden))
    if cfg.q_lora > 0:
        _need(W_DQ, "W_DQ", dt, shape=(cfg.hidden, cfg.q_lora))
        _need(W_UQ, "W_UQ", dt, shape=(cfg.q_lora, H * (cfg.qk_nope + cfg.d_r)))
    else:
        if W_DQ is not None:
            raise ValueError("W_DQ must be None without query compression")
        _need(W_UQ, "W_Q", dt, shape=(cfg.hidden, H * (cfg.qk_nope + cfg.d_r)))
    _need(W_UK, "W_UK", dt, shape=(cfg.d_c, H * cfg.qk_nope))
    _need(pos, "pos", torch.int32, shape=(n,))
    _need(q_packed, "q_packed", torch.bfloat16,
          shape=((2 if cfg.split_query else 1) * n, H, cfg.d_c + cfg.d_r))
    _need(workspace, "workspace", torch.uint8)
    _check(lib().mla_absorb_q_packed(ctypes.byref(cfg.c()), _ptr(x), n, _ptr(W_DQ), _ptr(W_UQ), _ptr(W_UK),
                                     _ptr(pos), _ptr(q_packed), _ptr(workspace), workspace.numel(),
                                     _stream(stream)), "mla_absorb_q_packed")


def mla_decode_packed(cfg: Config, q_packed, batch: int, n_q: int, cache: Cache, seq_lens, workspace,
                      max_workers: int = 0, stream=None):
    H = cfg.n_heads
    _need(q_packed, "q_packed", torch.bfloat16,
          shape=((2 if cfg.split_query else 1) * batch * n_q, H, cfg.d_c + cfg.d_r))
    _need(seq_lens, "seq_lens", torch.int32, shape=(batch,))
    _need(workspace, "workspace", torch.uint8)
    _check(lib().mla_decode_packed(ctypes.byref(cfg.c()), _ptr(q_packed), batch, n_q, ctypes.byref(cache.c),
                                   _ptr(seq_lens), max_workers, _ptr(workspace), workspace.numel(),
                                   _stream(stream)), "mla_decode_packed")


def mla_decode_plan(cfg: Config, batch: int, n_q: int, cache: Cache, seq_lens, workspace, max_workers: int = 0,
                    stream=None):
    _need(seq_lens, "seq_lens", torch.int32, shape=(batch,))
    _need(workspace, "workspace", torch.uint8)
    _check(lib().mla_decode_plan(ctypes.byref(cfg.c()), batch, n_q, ctypes.byref(cache.c), _ptr(seq_lens),
                                 max_workers, _ptr(workspace), workspace.numel(), _stream(stream)),
           "mla_decode_plan")


def mla_decode_packed_planned(cfg: Config, q_packed, batch: int, n_q: int, cache: Cache, seq_lens, workspace,
                              max_workers: int = 0, stream=None):
    H = cfg.n_heads
    _need(q_packed, "q_packed", torch.bfloat16,
          shape=((2 if cfg.split_query else 1) * batch * n_q, H, cfg.d_c + cfg.d_r))
    _need(seq_lens, "seq_lens", torch.int32, shape=(batch,))
    _need(workspace, "workspace", torch.uint8)
    _check(lib().mla_decode_packed_planned(ctypes.byref(cfg.c()), _ptr(q_packed), batch, n_q,
                                           ctypes.byref(cache.c), _ptr(seq_lens), max_workers, _ptr(workspace),
                                           workspace.numel(), _stream(stream)), "mla_decode_packed_planned")


def mla_decode(cfg: Config, q_lat, q_rope, batch: int, n_q: int, cache: Cache, seq_lens, workspace,
               max_workers: int = 0, stream=None):
    dt = cfg.torch_dtype
    H = cfg.n_heads
    _need(q_lat, "q_lat", torch.float32, shape=(batch * n_q, H, cfg.d_c))
    _need(q_rope, "q_rope", torch.float32, shape=(batch * n_q, H, cfg.d_r))
    _need(seq_lens, "seq_lens", torch.int32, shape=(batch,))
    _need(workspace, "workspace", torch.uint8)
    _check(lib().mla_decode(ctypes.byref(cfg.c()), _ptr(q_lat), _ptr(q_rope), batch, n_q,
                            ctypes.byref(cache.c), _ptr(seq_lens), max_workers, _ptr(workspace),
                            workspace.numel(), _stream(stream)), "mla_decode")


def mla_combine(cfg: Config, workspace, batch: int, n_q: int, o_lat, stream=None):
    _need(workspace, "workspace", torch.uint8)
    _need(o_lat, "o_lat", torch.float32, shape=(batch * n_q, cfg.n_heads, cfg.d_c))
    _check(lib().mla_combine(ctypes.byref(cfg.c()), _ptr(workspace), workspace.numel(), batch, n_q,
                             _ptr(o_lat), _stream(stream)), "mla_combine")


def mla_fp8_scratch_bytes(cfg: Config, batch: int, max_blocks_per_seq: int) -> int:
    return int(lib().mla_fp8_scratch_bytes(ctypes.byref(cfg.c()), batch, max_blocks_per_seq))


def fp8_scratch_cache(cfg: Config, scratch, batch: int, max_blocks_per_seq: int) -> "Cache":
    """The bf16 cache view of an ``mla_cache_dequant_fp8`` scratch (layout in
    ``include/mla.h``): decode it with ``cfg`` without ``fp8_cache``."""
    _need(scratch, "scratch", torch.uint8)
    slots = batch * max_blocks_per_seq
    off = (4 * slots + 255) // 256 * 256
    table = scratch[:4 * slots].view(torch.int32).view(batch, max_blocks_per_seq)
    pages = scratch[off:off + slots * cfg.block_size * (cfg.d_c + cfg.d_r) * 2].view(torch.bfloat16)
    return Cache(pages.view(slots, cfg.block_size, cfg.d_c + cfg.d_r), table)


def mla_cache_dequant_fp8(cfg: Config, cache: "Cache", batch: int, seq_lens, scratch, stream=None):
    _need(seq_lens, "seq_lens", torch.int32, shape=(batch,))
    _need(scratch, "scratch", torch.uint8)
    _check(lib().mla_cache_dequant_fp8(ctypes.byref(cfg.c()), ctypes.byref(cache.c), batch, _ptr(seq_lens),
                                       _ptr(scratch), scratch.numel(), _stream(stream)), "mla_cache_dequant_fp8")


def mla_combine_lse(cfg: Config, workspace, batch: int, n_q: int, o_lat, lse, stream=None):
    _need(workspace, "workspace", torch.uint8)
    _need(o_lat, "o_lat", torch.float32, shape=(batch * n_q, cfg.n_heads, cfg.d_c))
    _need(lse, "lse", torch.float32, shape=(batch * n_q, cfg.n_heads))
    _check(lib().mla_combine_lse(ctypes.byref(cfg.c()), _ptr(workspace), workspace.numel(), batch, n_q,
                                 _ptr(o_lat), _ptr(lse), _stream(stream)), "mla_combine_lse")


def mla_merge_shards(cfg: Config, o_parts, lse_parts, o_lat, lse=None, stream=None):
    """``o_parts`` [S, rows, H, d_c], ``lse_parts`` [S, rows, H] -> ``o_lat`` [rows, H, d_c] (+ ``lse``)."""
    _need(o_parts, "o_parts", torch.float32, ndim=4)
    S, rows = o_parts.shape[0], o_parts.shape[1]
    _need(lse_parts, "lse_parts", torch.float32, shape=(S, rows, cfg.n_heads))
    _need(o_lat, "o_lat", torch.float32, shape=(rows, cfg.n_heads, cfg.d_c))
    if lse is not None:
        _need(lse, "lse", torch.float32, shape=(rows, cfg.n_heads))
    _check(lib().mla_merge_shards(ctypes.byref(cfg.c()), S, rows, _ptr(o_parts), _ptr(lse_parts), _ptr(o_lat),
                                  _ptr(lse), _stream(stream)), "mla_merge_shards")


def mla_combine_out_proj_workspace_size(cfg: Config, batch: int, n_q: int) -> int:
    return int(lib().mla_combine_out_proj_workspace_size(ctypes.byref(cfg.c()), batch, n_q))


def mla_combine_out_proj(cfg: Config, decode_ws, batch: int, n_q: int, W_UV, W_O, y, workspace,
                         max_workers: int = 0, stream=None):
    dt = cfg.torch_dtype
    H = cfg.n_heads
    _need(decode_ws, "decode_ws", torch.uint8)
    _need(W_UV, "W_UV", dt, shape=(cfg.d_c, H * cfg.v_head))
    _need(W_O, "W_O", dt, shape=(H * cfg.v_head, cfg.hidden))
    _need(y, "y", dt, shape=(batch * n_q, cfg.hidden))
    _need(workspace, "workspace", torch.uint8)
    _check(lib().mla_combine_out_proj(ctypes.byref(cfg.c()), _ptr(decode_ws), decode_ws.numel(), batch, n_q,
                                      max_workers, _ptr(W_UV), _ptr(W_O), _ptr(y), _ptr(workspace),
                                      workspace.numel(), _stream(stream)), "mla_combine_out_proj")


def mla_out_proj(cfg: Config, o_lat, W_UV, W_O, y, workspace, stream=None):
    dt = cfg.torch_dtype
    n = o_lat.shape[0]
    H = cfg.n_heads
    _need(o_lat, "o_lat", torch.float32, shape=(n, H, cfg.d_c))
    _need(W_UV, "W_UV", dt, shape=(cfg.d_c, H * cfg.v_head))
    _need(W_O, "W_O", dt, shape=(H * cfg.v_head, cfg.hidden))
    _need(y, "y", dt, shape=(n, cfg.hidden))
    _need(workspace, "workspace", torch.uint8)
    _check(lib().mla_out_proj(ctypes.byref(cfg.c()), _ptr(o_lat), n, _ptr(W_UV), _ptr(W_O), _ptr(y),
                              _ptr(workspace), workspace.numel(), _stream(stream)), "mla_out_proj")


def mla_get_device_error(stream=None):
    """(status, detail[3]) of the first device-side error since the last call; clears it."""
    detail = (_i32 * 3)()
    status = lib().mla_get_device_error(_stream(stream), detail)
    return status, list(detail)


def mla_check_wait_timeout(limit_ns: int, stream=None):
    """Launch the library's bounded-wait check (a wait that must give up after ``limit_ns``)."""
    _check(lib().mla_check_wait_timeout(int(limit_ns), _stream(stream)), "mla_check_wait_timeout")


def mla_kernel_launches() -> int:
    return int(lib().mla_kernel_launches())


def check_device_error(stream=None):
    status, detail = mla_get_device_error(stream)
    if status != MLA_OK:
        raise MLAError(status, "device", detail)
