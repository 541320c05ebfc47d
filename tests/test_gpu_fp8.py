"""FP8 latent cache (E4M3 codes + one fp32 scale per row): the append writes
the oracle's codes and scales bit for bit, and the decode over the codes
gives the oracle's outputs for every token."""

import dataclasses

import numpy as np
import pytest
import torch

from mla_synth import WORKLOADS, generate, reduced
from mla_latent_kv_39_b200 import Cache, Config, MLAError, abi
from mla_gpu_cases import check_new_cache_rows, check_outputs, oracle_expect, run_gpu

pytestmark = pytest.mark.gpu


def test_fp8_cache_step_matches_the_oracle():
    wl = reduced(WORKLOADS["v3_fp8_b64_ragged1k_8k"], lengths=[700, 65, 1, 130, 63])
    data, dev, layer = run_gpu(wl)
    assert not layer.packed and not layer.fused_out       # CUDA-core decode of the codes
    exp = oracle_expect(data, order="absorbed")
    check_new_cache_rows(layer, data, exp)
    worst = check_outputs(layer, data, exp, range(wl.n_tok))
    assert worst["o_lat"] < 1e-2 and worst["y"] < 1e-2


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
    data, dev, layer = run_gpu(wl)
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
