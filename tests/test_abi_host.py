"""The C-ABI library on a machine without a GPU: it loads, exports every
symbol the header declares, its structs have the header's layout, and the
synchronous argument checks answer before any launch."""

import ctypes
import re
import subprocess
from pathlib import Path

import pytest

from mla_latent_kv_39_b200 import abi, build

ROOT = Path(__file__).resolve().parents[1]
HEADER = ROOT / "include" / "mla.h"


@pytest.fixture(scope="module")
def lib():
    build.build()
    return abi.load_library()


def declared_functions():
    text = re.sub(r"/\*.*?\*/", "", HEADER.read_text(), flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_five_steps():
    names = declared_functions()
    for step in ("mla_cache_append", "mla_absorb_q", "mla_decode", "mla_combine", "mla_out_proj"):
        assert step in names


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", str(abi._LIB_PATH)], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\b(mla_[a-z0-9_]+)\b", out))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    assert set(abi.SIGNATURES) == set(declared_functions())


def test_struct_layout_matches_the_header(tmp_path):
    src = tmp_path / "layout.c"
    src.write_text(
        '#include <stdio.h>\n#include <stddef.h>\n#include "mla.h"\n'
        "int main(void){printf(\"%zu %zu %zu %zu %zu %zu %zu\\n\", sizeof(mla_config),"
        " offsetof(mla_config, rope_theta), offsetof(mla_config, flags), sizeof(mla_cache),"
        " offsetof(mla_cache, block_table), offsetof(mla_cache, max_blocks_per_seq),"
        " offsetof(mla_cache, row_scale));return 0;}\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", f"-I{ROOT / 'include'}", str(src), "-o", str(exe)], check=True)
    got = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True,
                                          check=True).stdout.split()]
    want = [ctypes.sizeof(abi.MLAConfig), abi.MLAConfig.rope_theta.offset, abi.MLAConfig.flags.offset,
            ctypes.sizeof(abi.MLACache), abi.MLACache.block_table.offset,
            abi.MLACache.max_blocks_per_seq.offset, abi.MLACache.row_scale.offset]
    assert got == want


def _cfg(**kw):
    base = dict(hidden=256, n_heads=4, d_c=64, d_r=16, qk_nope=32, v_head=32, q_lora=0, dtype="f32")
    base.update(kw)
    return abi.Config(**base).c()


def test_abi_version(lib):
    assert lib.mla_abi_version() == 2


def test_invalid_configs_are_rejected_synchronously(lib):
    P = ctypes.byref
    assert lib.mla_cache_append(None, None, 1, None, None, None, None, None, None, 0, None) == abi.MLA_ERR_INVALID_ARG
    for bad in (dict(d_r=15), dict(n_heads=0), dict(block_size=0), dict(dtype=7), dict(rope_theta=0.0)):
        if "dtype" in bad:
            c = _cfg()
            c.dtype = bad["dtype"]
        else:
            c = _cfg(**bad)
        assert lib.mla_decode_workspace_size(P(c), 1, 1, 0) == 0
        assert lib.mla_out_proj(P(c), None, 1, None, None, None, None, 0, None) == abi.MLA_ERR_INVALID_ARG


def test_null_pointers_and_small_workspace_answer_before_launch(lib):
    P = ctypes.byref
    c = _cfg()
    fake = ctypes.c_void_p(0x1000)   # never dereferenced: every check below fails first
    assert lib.mla_absorb_q(P(c), None, 2, None, fake, fake, fake, fake, fake, fake, 1 << 20, None) \
        == abi.MLA_ERR_INVALID_ARG
    # W_DQ given although q_lora == 0
    assert lib.mla_absorb_q(P(c), fake, 2, fake, fake, fake, fake, fake, fake, fake, 1 << 20, None) \
        == abi.MLA_ERR_INVALID_ARG
    need = lib.mla_out_proj_workspace_size(P(c), 5)
    assert need > 0
    assert lib.mla_out_proj(P(c), fake, 5, fake, fake, fake, fake, need - 1, None) == abi.MLA_ERR_WORKSPACE
    cache = abi.MLACache(0x2000, 4, 0x3000, 1, 2)
    need = lib.mla_decode_workspace_size(P(c), 1, 1, 8)
    assert lib.mla_decode(P(c), fake, fake, 1, 1, P(cache), fake, 8, fake, need - 1, None) == abi.MLA_ERR_WORKSPACE
    assert lib.mla_decode(P(c), fake, fake, 2, 1, P(cache), fake, 8, fake, need, None) == abi.MLA_ERR_INVALID_ARG
    assert lib.mla_decode(P(c), fake, fake, 1, 0, P(cache), fake, 8, fake, need, None) == abi.MLA_ERR_INVALID_ARG


def test_empty_work_is_a_no_op(lib):
    P = ctypes.byref
    c = _cfg()
    assert lib.mla_cache_append(P(c), None, 0, None, None, None, None, None, None, 0, None) == abi.MLA_OK
    assert lib.mla_absorb_q(P(c), None, 0, None, None, None, None, None, None, None, 0, None) == abi.MLA_OK
    assert lib.mla_decode(P(c), None, None, 0, 1, None, None, 0, None, 0, None) == abi.MLA_OK
    assert lib.mla_combine(P(c), None, 0, 0, 1, None, None) == abi.MLA_OK
    assert lib.mla_out_proj(P(c), None, 0, None, None, None, None, 0, None) == abi.MLA_OK
    assert lib.mla_combine_out_proj(P(c), None, 0, 0, 1, 0, None, None, None, None, 0, None) == abi.MLA_OK


def test_decode_workspace_grows_with_workers_and_batch(lib):
    P = ctypes.byref
    c = _cfg(hidden=7168, n_heads=128, d_c=512, d_r=64, qk_nope=128, v_head=128, q_lora=1536, dtype="bf16")
    a = lib.mla_decode_workspace_size(P(c), 64, 1, 74)
    b = lib.mla_decode_workspace_size(P(c), 64, 1, 148)
    d = lib.mla_decode_workspace_size(P(c), 64, 2, 74)
    seg_bytes = 128 * 512 * 2     # bf16 partial output of one segment, all heads
    # one partial slot per worker and per query row
    assert b - a >= 74 * seg_bytes and d - a >= 64 * seg_bytes


def test_status_strings(lib):
    for code in range(-6, 1):
        assert lib.mla_status_string(code)


def test_unaligned_tensors_are_rejected_on_the_bf16_path(lib):
    """TMA and 16-byte vector accesses need 16-byte aligned tensors; the bf16
    entry points refuse an unaligned pointer before any launch."""
    P = ctypes.byref
    c = _cfg(hidden=7168, n_heads=128, d_c=512, d_r=64, qk_nope=128, v_head=128, q_lora=1536, dtype="bf16")
    ok, bad = ctypes.c_void_p(0x10000), ctypes.c_void_p(0x10008)
    need = lib.mla_absorb_q_workspace_size(P(c), 4)
    assert need > 0
    for i in range(7):
        args = [ok] * 7
        args[i] = bad          # x, W_DQ, W_UQ, W_UK, q_lat, q_rope, workspace (pos is int32, any alignment)
        x, wdq, wuq, wuk, ql, qr, ws = args
        assert lib.mla_absorb_q(P(c), x, 4, wdq, wuq, wuk, ok, ql, qr, ws, need, None) == abi.MLA_ERR_INVALID_ARG
    need = lib.mla_out_proj_workspace_size(P(c), 4)
    for i in range(5):
        args = [ok] * 5
        args[i] = bad
        o, wuv, wo, y, ws = args
        assert lib.mla_out_proj(P(c), o, 4, wuv, wo, y, ws, need, None) == abi.MLA_ERR_INVALID_ARG
    cache = abi.MLACache(0x10008, 4, 0x3000, 1, 2)   # pool off the 16-byte grid
    need = lib.mla_decode_workspace_size(P(c), 1, 1, 8)
    assert lib.mla_decode(P(c), ok, ok, 1, 1, P(cache), ok, 8, ok, need, None) == abi.MLA_ERR_INVALID_ARG
    assert lib.mla_combine(P(c), ok, need, 1, 1, bad, None) == abi.MLA_ERR_INVALID_ARG


def test_fused_projection_checks_its_arguments(lib):
    P = ctypes.byref
    c = _cfg(hidden=7168, n_heads=128, d_c=512, d_r=64, qk_nope=128, v_head=128, q_lora=1536, dtype="bf16")
    fake = ctypes.c_void_p(1 << 20)
    need = lib.mla_combine_out_proj_workspace_size(P(c), 64, 1)
    # W_O partials (none for 64 tokens with one K split) + the bf16 head outputs
    assert need >= 64 * 128 * 128 * 2
    dws = lib.mla_decode_workspace_size(P(c), 64, 1, 0)
    assert lib.mla_combine_out_proj(P(c), None, dws, 64, 1, 0, fake, fake, fake, fake, need, None) == \
        abi.MLA_ERR_INVALID_ARG
    assert lib.mla_combine_out_proj(P(c), fake, dws - 256, 64, 1, 0, fake, fake, fake, fake, need, None) == \
        abi.MLA_ERR_WORKSPACE
    assert lib.mla_combine_out_proj(P(c), fake, dws, 64, 1, 0, fake, fake, fake, fake, need - 256, None) == \
        abi.MLA_ERR_WORKSPACE
    # more than 512 segments (rows + workers - 1) is not supported by the fused path
    assert lib.mla_combine_out_proj(P(c), fake, 1 << 40, 600, 1, 0, fake, fake, fake, fake, 1 << 40, None) == \
        abi.MLA_ERR_UNSUPPORTED
    f32 = _cfg(dtype="f32")
    assert lib.mla_combine_out_proj_workspace_size(P(f32), 1, 1) == 0



def test_fp8_cache_configuration_is_checked_before_any_launch(lib):
    """MLA_FLAG_FP8_CACHE needs bf16 weights and the cache's row scales; the
    packed-query (tensor-core) path does not take an FP8 cache."""
    P = ctypes.byref
    v3 = dict(hidden=7168, n_heads=128, d_c=512, d_r=64, qk_nope=128, v_head=128, q_lora=1536)
    fp8 = abi.Config(**v3, dtype="bf16", fp8_cache=True).c()
    assert fp8.flags & abi.MLA_FLAG_FP8_CACHE
    f32 = _cfg(fp8_cache=True)                      # FP8 cache over fp32 weights: invalid
    assert lib.mla_decode_workspace_size(P(f32), 1, 1, 0) == 0
    fake = ctypes.c_void_p(1 << 20)
    no_scale = abi.MLACache(1 << 20, 4, 1 << 21, 1, 2, None)
    need = lib.mla_decode_workspace_size(P(fp8), 1, 1, 8)
    assert need > 0
    assert lib.mla_decode(P(fp8), fake, fake, 1, 1, P(no_scale), fake, 8, fake, need, None) == abi.MLA_ERR_INVALID_ARG
    assert lib.mla_cache_append(P(fp8), fake, 1, fake, fake, fake, fake, P(no_scale), fake, 1 << 30, None) \
        == abi.MLA_ERR_INVALID_ARG
    odd_scale = abi.MLACache(1 << 20, 4, 1 << 21, 1, 2, (1 << 22) + 2)   # not 4-byte aligned
    assert lib.mla_decode(P(fp8), fake, fake, 1, 1, P(odd_scale), fake, 8, fake, need, None) == abi.MLA_ERR_INVALID_ARG
    assert lib.mla_query_packed_bytes(P(fp8), 4) == 0
    assert lib.mla_combine_out_proj_workspace_size(P(fp8), 64, 1) == 0
    with_scale = abi.MLACache(1 << 20, 4, 1 << 21, 1, 2, 1 << 22)
    assert lib.mla_decode_packed(P(fp8), fake, 1, 1, P(with_scale), fake, 8, fake, need, None) \
        == abi.MLA_ERR_UNSUPPORTED
    # the CUDA-core decode's workspace: fp32 partial outputs
    bf = abi.Config(**v3, dtype="bf16").c()
    assert lib.mla_decode_workspace_size(P(fp8), 64, 1, 74) > lib.mla_decode_workspace_size(P(bf), 64, 1, 74)


def test_shard_merge_checks_its_arguments(lib):
    P = ctypes.byref
    c = _cfg()
    fake = ctypes.c_void_p(1 << 20)
    assert lib.mla_merge_shards(P(c), 0, 4, fake, fake, fake, None, None) == abi.MLA_ERR_INVALID_ARG
    assert lib.mla_merge_shards(P(c), 2, -1, fake, fake, fake, None, None) == abi.MLA_ERR_INVALID_ARG
    assert lib.mla_merge_shards(P(c), 2, 0, None, None, None, None, None) == abi.MLA_OK      # no rows
    assert lib.mla_merge_shards(P(c), 2, 4, None, fake, fake, None, None) == abi.MLA_ERR_INVALID_ARG
    odd = ctypes.c_void_p((1 << 20) + 8)
    assert lib.mla_merge_shards(P(c), 2, 4, odd, fake, fake, None, None) == abi.MLA_ERR_INVALID_ARG
    assert lib.mla_combine_lse(P(c), fake, 1 << 20, 1, 1, fake, None, None) == abi.MLA_ERR_INVALID_ARG


def test_fp8_scratch_size_and_dequant_checks(lib):
    P = ctypes.byref
    v3 = dict(hidden=7168, n_heads=128, d_c=512, d_r=64, qk_nope=128, v_head=128, q_lora=1536)
    fp8 = abi.Config(**v3, dtype="bf16", fp8_cache=True).c()
    bf = abi.Config(**v3, dtype="bf16").c()
    need = lib.mla_fp8_scratch_bytes(P(fp8), 3, 5)
    assert need == 256 + 3 * 5 * 64 * 576 * 2          # table (60 B, padded to 256) + bf16 pages
    assert lib.mla_fp8_scratch_bytes(P(bf), 3, 5) == 0
    fake = ctypes.c_void_p(1 << 20)
    cache = abi.MLACache(1 << 20, 8, 1 << 21, 3, 5, 1 << 22)
    assert lib.mla_cache_dequant_fp8(P(bf), P(cache), 3, fake, fake, need, None) == abi.MLA_ERR_INVALID_ARG
    assert lib.mla_cache_dequant_fp8(P(fp8), P(cache), 3, fake, fake, need - 1, None) == abi.MLA_ERR_WORKSPACE
    assert lib.mla_cache_dequant_fp8(P(fp8), P(cache), 3, None, fake, need, None) == abi.MLA_ERR_INVALID_ARG
    assert lib.mla_cache_dequant_fp8(P(fp8), P(cache), 3, fake, ctypes.c_void_p((1 << 20) + 8), need, None) \
        == abi.MLA_ERR_INVALID_ARG
    assert lib.mla_cache_dequant_fp8(P(fp8), P(cache), 0, None, None, 0, None) == abi.MLA_OK
