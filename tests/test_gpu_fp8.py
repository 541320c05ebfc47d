"""FP8 latent cache (E4M3 codes + one fp32 scale per row): the append writes
the oracle's codes and scales bit for bit, and the decode over the codes
(through the bf16 scratch cache on the tensor cores, or on CUDA cores) gives
the oracle's outputs for every token."""

import dataclasses

import numpy as np
import pytest
import torch

from mla_synth import WORKLOADS, generate, reduced
from mla_latent_kv_39_b200 import Cache, Config, MLAError, abi
import oracle
from mla_gpu_cases import check_new_cache_rows, check_outputs, oracle_expect, run_gpu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("tensor_cores", [True, False])
def test_fp8_cache_step_matches_the_oracle(tensor_cores):
    """Tensor cores: the step's pages expanded into the bf16 scratch cache,
    then the bf16 path (packed query, fused combine); else the CUDA-core
    decode of the codes (fp32 query)."""
    wl = reduced(WORKLOADS["v3_fp8_b64_ragged1k_8k"], lengths=[700, 65, 1, 130, 63])
    data, dev, layer = run_gpu(wl, packed_query=tensor_cores)
    assert layer.packed == tensor_cores and layer.fused_out == tensor_cores
    exp = oracle_expect(data, order="absorbed")
    check_new_cache_rows(layer, data, exp)
    worst = check_outputs(layer, data, exp, range(wl.n_tok))
    assert worst["o_lat"] < 1e-2 and worst["y"] < 1e-2


def test_fp8_scratch_pages_are_the_codes_times_their_scales():
    """mla_cache_dequant_fp8: every visible row of the scratch cache equals
    bf16(code * row scale) of the FP8 row (one rounding), the table maps
    (b, k) to b * max_blocks + k, and pages past a sequence are not touched."""
    wl = reduced(WORKLOADS["v3_fp8_b64_ragged1k_8k"], lengths=[130, 1, 64])
    data, dev, layer = run_gpu(wl)
    mb = dev["block_table"].shape[1]
    table = layer.dcache.block_table.cpu().numpy()
    assert np.array_equal(table, np.arange(wl.batch * mb).reshape(wl.batch, mb))
    pages = layer.dcache.pool.cpu()
    codes = layer.cache.pool.cpu().numpy()
    scale = layer.cache.row_scale.cpu().numpy()
    bs = wl.shape.block_size
    for b in range(wl.batch):
        L = int(data.seq_lens[b])
        for t in range(L):
            phys = int(data.block_table[b, t // bs])
            want = oracle.round_to_bf16(oracle.e4m3_value(codes[phys, t % bs]) * float(scale[phys, t % bs]))
            got = oracle.to64(pages[b * mb + t // bs, t % bs])
            assert np.array_equal(got, want), (b, t)


def test_fp8_cache_full_size_sampled_sequences():
    wl = WORKLOADS["v3_fp8_b64_ragged1k_8k"]
    data, dev, layer = run_gpu(wl)
    lens = data.cached_len.numpy()
    seqs = sorted({int(np.argmin(lens)), int(np.argmax(lens)), 17, 42})
    exp = oracle_expect(data, seqs=seqs, order="absorbed")
    check_new_cache_rows(layer, data, exp)
    check_outputs(layer, data, exp, seqs)


def test_fp8_cache_configuration_errors():
    wl = reduced(WORKLOADS["v3_fp8_b64_ragged1k_8k"], lengths=[100])
    data, dev, layer = run_gpu(wl, packed_query=False)
    cfg = layer.cfg
    assert abi.mla_query_packed_bytes(cfg, 1) == 0
    q = torch.zeros(1, cfg.n_heads, cfg.d_c + cfg.d_r, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(MLAError) as e:
        abi.mla_decode_packed(cfg, q, 1, 1, layer.cache, dev["seq_lens"], layer.ws_decode)
    assert e.value.status == abi.MLA_ERR_UNSUPPORTED
    no_scale = Cache(dev["pool"], dev["block_table"])
    with pytest.raises(MLAError) as e:
        abi.mla_decode(cfg, layer.q_lat, layer.q_rope, 1, 1, no_scale, dev["seq_lens"], layer.ws_decode)
    assert e.value.status == abi.MLA_ERR_INVALID_ARG
    f32 = dataclasses.replace(Config.from_shape(WORKLOADS["tiny_f32_b1_l128"].shape), fp8_cache=True)
    ql = torch.zeros(1, f32.n_heads, f32.d_c, device="cuda")
    qr = torch.zeros(1, f32.n_heads, f32.d_r, device="cuda")
    with pytest.raises(MLAError) as e:      # an FP8 cache needs bf16 weights
        abi.mla_decode(f32, ql, qr, 1, 1, layer.cache, dev["seq_lens"], layer.ws_decode)
    assert e.value.status == abi.MLA_ERR_INVALID_ARG
