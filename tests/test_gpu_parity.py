"""CUDA path vs the fp64 oracle, through the C ABI, on seeded inputs.

Small cases compare every output element; full-size workloads (the same
launch configuration the benchmark times) compare sampled sequences, which
the oracle computes one by one in the absorbed order (itself pinned to the
decompressed order to 1e-10).  The cache rows that a step appends must be
bit-identical to the oracle's once-rounded rows.
"""

import numpy as np
import pytest
import torch

import oracle
from mla_synth import WORKLOADS, build_pool, generate, reduced
from mla_latent_kv_39_b200 import (MLAError, Cache, Config, DecodeLayer, abi, check_device_error,
                                   mla_get_device_error)

from mla_gpu_cases import (check_new_cache_rows, check_outputs, oracle_expect, pool_row, run_gpu,
                           tol_for, assert_close)

pytestmark = pytest.mark.gpu


def test_tiny_fp32_whole_config():
    wl = WORKLOADS["tiny_f32_b1_l128"]
    data, dev, layer = run_gpu(wl)
    exp = oracle_expect(data, order="decompressed")
    exp_abs = oracle_expect(data, order="absorbed")
    # every cached row (appended by the library from x_cached) is exact
    for p in range(int(data.cached_len[0])):
        want = np.concatenate([exp["cached_c"][0][p], exp["cached_kr"][0][p]])
        assert np.array_equal(pool_row(layer, data, 0, p), want), p
    check_new_cache_rows(layer, data, exp)
    exp["o_lat"] = exp_abs["o_lat"]
    check_outputs(layer, data, exp, range(wl.n_tok))


SMALL_CASES = [
    # name, reduced lengths, n_q  (page-boundary, single-row and long rows)
    ("v2_b16_l4096", [4096, 63, 64, 65, 0], None),
    ("v3_b64_ragged1k_8k", [700, 1, 130, 191, 257, 64], None),
    ("v3_b4_long", [5000, 20000], None),
    ("v3_b128_nq2_ragged512_16k", [0, 1, 62, 63, 64, 300], 2),
    # 260 new tokens: the projections run in two token chunks
    ("v3_b128_nq2_ragged512_16k", [3] * 130, 2),
    # chunked prefill: 16 causal query tokens per sequence, one with an empty cache
    ("v3_prefill_b8_c64_ragged1k_4k", [0, 65, 200], 16),
]


@pytest.mark.parametrize("name,lengths,n_q", SMALL_CASES,
                         ids=[f"{c[0]}-{i}" for i, c in enumerate(SMALL_CASES)])
def test_small_cases_every_element(name, lengths, n_q):
    wl = reduced(WORKLOADS[name], lengths=lengths, n_q=n_q)
    data, dev, layer = run_gpu(wl)
    exp = oracle_expect(data, order="decompressed")
    exp_abs = oracle_expect(data, order="absorbed")
    check_new_cache_rows(layer, data, exp)
    exp["o_lat"] = exp_abs["o_lat"]
    check_outputs(layer, data, exp, range(wl.n_tok))


FULL = ["v2_b16_l4096", "v3_b64_ragged1k_8k", "v3_b4_long", "v3_b128_nq2_ragged512_16k",
        "v3_prefill_b8_c64_ragged1k_4k"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_every_sequence(name):
    """The benchmark's launch configuration at full size: every query token of
    every sequence (all segments and merges of the split plan) against the
    absorbed-order oracle, itself pinned to the decompressed order."""
    wl = WORKLOADS[name]
    data, dev, layer = run_gpu(wl)
    exp = oracle_expect(data, order="absorbed")
    check_new_cache_rows(layer, data, exp)
    check_outputs(layer, data, exp, range(wl.n_tok))


def test_split_query_mode_on_an_unspiked_case():
    import dataclasses
    wl = dataclasses.replace(reduced(WORKLOADS["v3_b64_ragged1k_8k"], lengths=[700, 1, 130]), split_query=True)
    data, dev, layer = run_gpu(wl)
    exp = oracle_expect(data, order="absorbed")
    worst = check_outputs(layer, data, exp, range(wl.n_tok))
    # hi + lo query: what is left is P and the per-segment outputs rounded to
    # bf16 (a relative 2^-9 each), well inside the 1e-2 bound
    assert worst["o_lat"] < 2.5 * 2.0 ** -9


def test_split_query_tightens_the_spiked_case():
    import dataclasses
    base = reduced(WORKLOADS["v3_b4_long"], lengths=[5000, 20000])
    errs = {}
    for split in (False, True):
        wl = dataclasses.replace(base, split_query=split)
        data, dev, layer = run_gpu(wl)
        exp = oracle_expect(data, order="absorbed")
        o = layer.o_lat.cpu().double().numpy()
        errs[split] = max(np.max(np.abs(o[t] - exp["o_lat"][t])) / np.max(np.abs(exp["o_lat"][t]))
                          for t in range(wl.n_tok))
    assert errs[True] < 1e-2 and errs[True] < 0.5 * errs[False], errs


def test_split_count_does_not_change_the_result():
    wl = reduced(WORKLOADS["v3_b64_ragged1k_8k"], lengths=[3000, 70, 1500])
    data = generate(wl)
    outs = []
    for workers in (1, 3, 7, 0):
        _, _, layer = run_gpu(wl, data=data, max_workers=workers)
        outs.append(layer.o_lat.cpu().double().numpy())
    # Different cuts change where the running max is taken and so how P rounds
    # to bf16, and how each piece's normalised output rounds to bf16 (relative
    # step 2^-9 each); two such pairs of roundings bound the difference.
    for o in outs[1:]:
        assert np.max(np.abs(o - outs[0])) <= 4 * 2.0 ** -9 * np.max(np.abs(outs[0]))


def test_physical_page_order_does_not_change_the_result():
    wl = reduced(WORKLOADS["v3_b64_ragged1k_8k"], lengths=[900, 333])
    a = generate(wl)
    _, _, la = run_gpu(wl, data=a)
    # same logical rows, pages placed in reverse physical order
    b = generate(wl)
    b.block_table = torch.where(b.block_table >= 0, b.num_blocks - 1 - b.block_table, b.block_table)
    _, _, lb = run_gpu(wl, data=b)
    assert torch.equal(la.o_lat, lb.o_lat)
    assert torch.equal(la.y, lb.y)


def test_bad_block_id_is_reported_not_faulted():
    wl = reduced(WORKLOADS["v3_b64_ragged1k_8k"], lengths=[200, 100])
    data, dev, layer = run_gpu(wl)
    dev["block_table"][1, 0] = data.num_blocks + 5      # outside the pool
    layer.decode(dev["seq_lens"])
    status, detail = mla_get_device_error()
    assert status == abi.MLA_ERR_BOUNDS and detail[1] == 1
    assert mla_get_device_error()[0] == abi.MLA_OK    # cleared by the first read
    dev["block_table"][1, 0] = 0
    pos = torch.tensor([130], dtype=torch.int32, device="cuda")
    seq = torch.tensor([1], dtype=torch.int32, device="cuda")
    dev["block_table"][1, 2] = -7                        # append into a missing page
    layer.append(dev["x_new"][1:2], seq, pos)
    status, detail = mla_get_device_error()
    assert status == abi.MLA_ERR_BOUNDS


def test_sequence_shorter_than_its_queries_is_reported():
    wl = reduced(WORKLOADS["v3_b128_nq2_ragged512_16k"], lengths=[10, 20], n_q=2)
    data = generate(wl)
    _, dev, layer = run_gpu(wl, data=data)
    bad = dev["seq_lens"].clone()
    bad[0] = 1
    layer.attend(bad)
    status, detail = mla_get_device_error()
    assert status == abi.MLA_ERR_BOUNDS and detail[1] == 0
    assert torch.count_nonzero(layer.o_lat[0:2]) == 0     # that sequence's output is zero
    assert torch.count_nonzero(layer.o_lat[2:4]) > 0


def test_combine_rejects_a_workspace_decode_never_wrote():
    wl = reduced(WORKLOADS["v2_b16_l4096"], lengths=[64])
    _, dev, layer = run_gpu(wl)
    layer.ws_decode.zero_()
    abi.mla_combine(layer.cfg, layer.ws_decode, 1, 1, layer.o_lat)
    status, _ = mla_get_device_error()
    assert status == abi.MLA_ERR_WORKSPACE
    assert torch.count_nonzero(layer.o_lat) == 0


def test_workspace_too_small_raises_before_launch():
    wl = reduced(WORKLOADS["v2_b16_l4096"], lengths=[64])
    _, dev, layer = run_gpu(wl, packed_query=False)
    with pytest.raises(MLAError) as e:
        abi.mla_decode(layer.cfg, layer.q_lat, layer.q_rope, 1, 1, layer.cache, dev["seq_lens"],
                       layer.ws_decode[:100], 0)
    assert e.value.status == abi.MLA_ERR_WORKSPACE
    _, dev, layer = run_gpu(wl)
    with pytest.raises(MLAError) as e:
        abi.mla_decode_packed(layer.cfg, layer.q_packed, 1, 1, layer.cache, dev["seq_lens"], layer.ws_decode[:100], 0)
    assert e.value.status == abi.MLA_ERR_WORKSPACE


def test_empty_batch_is_a_no_op():
    wl = reduced(WORKLOADS["v2_b16_l4096"], lengths=[64])
    _, dev, layer = run_gpu(wl)
    cfg = layer.cfg
    H = cfg.n_heads
    e = torch.empty(0, H, cfg.d_c, dtype=torch.float32, device="cuda")
    abi.mla_decode(cfg, e, torch.empty(0, H, cfg.d_r, dtype=torch.float32, device="cuda"), 0, 1,
                   layer.cache, torch.empty(0, dtype=torch.int32, device="cuda"), layer.ws_decode, 0)
    abi.mla_decode_packed(cfg, torch.empty(0, H, cfg.d_c + cfg.d_r, dtype=torch.bfloat16, device="cuda"), 0, 1,
                          layer.cache, torch.empty(0, dtype=torch.int32, device="cuda"), layer.ws_decode, 0)
    torch.cuda.synchronize()
    check_device_error()


def test_fused_combine_projection_matches_the_two_step_path():
    """y from mla_combine_out_proj (split merge inside W_UV) agrees with
    mla_combine + mla_out_proj on the same decode workspace."""
    wl = reduced(WORKLOADS["v3_b64_ragged1k_8k"], lengths=[3000, 70, 1500, 1])
    data, dev, layer = run_gpu(wl, max_workers=9)       # several segments per row
    assert layer.fused_out
    y_fused = layer.y.clone()
    y_two = torch.empty_like(layer.y)
    abi.mla_out_proj(layer.cfg, layer.o_lat, layer.W["W_UV"], layer.W["W_O"], y_two, layer.ws_gemm)
    torch.cuda.synchronize()
    a, b = y_fused.double(), y_two.double()
    assert torch.max(torch.abs(a - b)) <= 1e-2 * torch.max(torch.abs(b))


def test_fused_projection_rejects_a_workspace_decode_never_wrote():
    wl = reduced(WORKLOADS["v3_b64_ragged1k_8k"], lengths=[64, 3])
    _, dev, layer = run_gpu(wl)
    layer.ws_decode.zero_()
    layer.project()
    status, _ = mla_get_device_error()
    assert status == abi.MLA_ERR_WORKSPACE
    assert torch.count_nonzero(layer.y) == 0


def test_fp32_query_handoff_gives_the_packed_paths_result():
    """mla_absorb_q + mla_decode (fp32 query across the ABI, packed by the
    decode) and mla_absorb_q_packed + mla_decode_packed round the query the
    same way: identical latent outputs."""
    wl = reduced(WORKLOADS["v3_b64_ragged1k_8k"], lengths=[900, 65, 1])
    data = generate(wl)
    _, _, a = run_gpu(wl, data=data, packed_query=True)
    _, _, b = run_gpu(wl, data=data, packed_query=False)
    assert a.packed and not b.packed
    assert torch.equal(a.o_lat, b.o_lat)
    assert torch.equal(a.y, b.y)



def test_plan_on_the_side_stream_gives_the_same_result():
    """step() computes the split plan with mla_decode_plan beside the query
    projections and decodes with mla_decode_packed_planned; planning inside
    mla_decode_packed gives identical o_lat and y."""
    wl = reduced(WORKLOADS["v3_b64_ragged1k_8k"], lengths=[3000, 70, 1500, 1])
    data, dev, layer = run_gpu(wl, max_workers=9)
    o_a, y_a = layer.o_lat.clone(), layer.y.clone()
    layer.ws_decode.zero_()
    layer.decode(dev["seq_lens"])                 # plan + decode in one call
    layer.combine()
    layer.project()
    torch.cuda.synchronize()
    check_device_error()
    assert torch.equal(layer.o_lat, o_a)
    assert torch.equal(layer.y, y_a)


def test_graph_replay_of_the_step_matches_the_eager_step():
    """capture_step records the whole step (fork to the side stream and join
    included); replays give the eager step's y and o_lat, also after the
    inputs are refilled in place."""
    wl = reduced(WORKLOADS["v3_b64_ragged1k_8k"], lengths=[700, 64, 1, 130])
    data, dev, layer = run_gpu(wl)
    x, si, pos, sl = dev["x_new"], dev["seq_idx"], dev["pos"], dev["seq_lens"]
    y_eager, o_eager = layer.y.clone(), layer.o_lat.clone()
    graph = layer.capture_step(x, si, pos, sl, want_o_lat=True)
    layer.y.zero_()
    layer.o_lat.zero_()
    graph.replay()
    torch.cuda.synchronize()
    check_device_error()
    assert torch.equal(layer.y, y_eager)
    assert torch.equal(layer.o_lat, o_eager)
    # new hidden states for the same positions: replay == eager
    x.copy_(torch.flip(x, dims=[1]))
    graph.replay()
    torch.cuda.synchronize()
    y_graph, o_graph = layer.y.clone(), layer.o_lat.clone()
    layer.step(x, si, pos, sl, want_o_lat=True)
    torch.cuda.synchronize()
    check_device_error()
    assert not torch.equal(y_graph, y_eager)
    assert torch.equal(layer.y, y_graph)
    assert torch.equal(layer.o_lat, o_graph)
