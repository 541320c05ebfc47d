"""Sequence split across GPUs, its arithmetic on one GPU: every shard of the
pages decoded in turn (the exchange being a stack), merged by
mla_merge_shards, against the oracle's decode over the whole sequence and
against the unsplit decode's output and log-sum-exp."""

import numpy as np
import pytest
import torch

from mla_synth import WORKLOADS, reduced
from mla_latent_kv_39_b200 import Cache, abi, check_device_error, decode_sharded, shard_plan
from mla_gpu_cases import assert_close, oracle_expect, run_gpu, tol_for

pytestmark = pytest.mark.gpu


def _split_vs_whole(wl, n_shards, max_workers=0):
    data, dev, layer = run_gpu(wl, max_workers=max_workers)
    cfg, rows, H = layer.cfg, wl.n_tok, wl.shape.n_heads
    # the unsplit decode's (o_lat, lse), from the step's decode workspace
    o_whole = torch.empty(rows, H, wl.shape.d_c, dtype=torch.float32, device="cuda")
    lse_whole = torch.empty(rows, H, dtype=torch.float32, device="cuda")
    abi.mla_combine_lse(cfg, layer.ws_decode, wl.batch, wl.n_q, o_whole, lse_whole)
    assert torch.equal(o_whole, layer.o_lat)      # same merge as mla_combine
    plan = shard_plan(dev["block_table"].cpu(), dev["seq_lens"].cpu(), wl.n_q, wl.shape.block_size, n_shards)
    caches = [Cache(dev["pool"], t.cuda()) for t in plan.block_tables]
    lens = [s.cuda() for s in plan.seq_lens]
    ws = torch.empty(abi.mla_decode_workspace_size(cfg, rows, 1, max_workers), dtype=torch.uint8, device="cuda")
    o = torch.empty_like(o_whole)
    lse = torch.empty_like(lse_whole)
    decode_sharded(cfg, layer.q_packed, rows, caches, lens, ws, o, lse, max_workers=max_workers)
    torch.cuda.synchronize()
    check_device_error()
    return data, plan, o, lse, o_whole, lse_whole


@pytest.mark.parametrize("n_shards", [2, 3])
def test_long_sequences_split_over_shards_match_the_whole_decode(n_shards):
    wl = reduced(WORKLOADS["v3_b4_long"], lengths=[9000, 20000, 3])
    data, plan, o, lse, o_whole, lse_whole = _split_vs_whole(wl, n_shards)
    assert int((plan.seq_lens[0] == 0).sum()) >= 1          # the 3-row sequence's first shard is empty
    exp = oracle_expect(data)
    tol = tol_for(wl.shape)
    got = o.cpu().double().numpy()
    for t in range(wl.n_tok):
        assert_close(got[t], exp["o_lat"][t], tol, f"split o_lat[{t}]")
    # both merge bf16 partial outputs of different cuts: equal to their rounding
    assert_close(got, o_whole.cpu().double().numpy(), tol, "split vs whole o_lat")
    assert torch.all(torch.isfinite(lse))
    assert torch.allclose(lse, lse_whole, rtol=0, atol=1e-4 * float(lse_whole.abs().max()))


def test_causal_rows_and_empty_shards_merge_correctly():
    """Two causal queries per sequence, one sequence shorter than a page:
    most of its shards hold no row (length 0: o = 0, lse = -inf)."""
    wl = reduced(WORKLOADS["v3_b128_nq2_ragged512_16k"], lengths=[10, 700, 130], n_q=2)
    data, plan, o, lse, o_whole, lse_whole = _split_vs_whole(wl, 3, max_workers=5)
    assert int((plan.seq_lens[0] == 0).sum()) >= 2          # the short sequence: all in the last shard
    exp = oracle_expect(data)
    got = o.cpu().double().numpy()
    for t in range(wl.n_tok):
        assert_close(got[t], exp["o_lat"][t], tol_for(wl.shape), f"split o_lat[{t}]")
    assert torch.allclose(lse, lse_whole, rtol=0, atol=1e-4 * float(lse_whole.abs().max()))


def test_merge_of_one_shard_is_that_shard_and_empty_rows_stay_empty():
    cfg = abi.Config.from_shape(WORKLOADS["tiny_f32_b1_l128"].shape)
    assert (cfg.n_heads, cfg.d_c) == (4, 64)
    g = torch.Generator().manual_seed(3)
    o = torch.randn(1, 5, 4, 64, generator=g).cuda()
    lse = torch.randn(1, 5, 4, generator=g).cuda()
    lse[0, 2] = -float("inf")
    out = torch.empty(5, 4, 64, device="cuda")
    lse_out = torch.empty(5, 4, device="cuda")
    abi.mla_merge_shards(cfg, o, lse, out, lse_out)
    torch.cuda.synchronize()
    want = o[0].clone()
    want[2] = 0
    assert torch.equal(out, want)
    assert torch.equal(lse_out, lse[0])
    # two shards: weights 2^lse_r / sum, in fp64 on the host
    o2 = torch.randn(2, 5, 4, 64, generator=g)
    l2 = torch.randn(2, 5, 4, generator=g) * 4
    abi.mla_merge_shards(cfg, o2.cuda(), l2.cuda(), out, lse_out)
    torch.cuda.synchronize()
    w = torch.pow(2.0, l2.double())
    ref = (w[..., None] * o2.double()).sum(0) / w.sum(0)[..., None]
    assert np.max(np.abs(out.cpu().double().numpy() - ref.numpy())) <= 1e-5 * float(ref.abs().max())
    assert np.max(np.abs(lse_out.cpu().double().numpy() - torch.log2(w.sum(0)).numpy())) <= 1e-5
