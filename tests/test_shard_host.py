"""Host side of the sequence split across GPUs: the shard plan, and the
exchange of per-shard (o_lat, lse) between two gloo ranks on CPU."""

import os
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from mla_latent_kv_39_b200.shard import gather_partials, shard_plan  # noqa: E402


def _check_plan(bt, lens, n_q, bs, n_shards):
    plan = shard_plan(bt, lens, n_q, bs, n_shards)
    batch = lens.numel()
    for b in range(batch):
        pages = (int(lens[b]) + bs - 1) // bs
        bounds = plan.page_bounds[b].tolist()
        assert bounds[0] == 0 and bounds[-1] == pages
        assert all(bounds[r] <= bounds[r + 1] for r in range(n_shards))
        assert max(bounds[r + 1] - bounds[r] for r in range(n_shards)) - \
            min(bounds[r + 1] - bounds[r] for r in range(n_shards)) <= 1      # even cut
        for j in range(n_q):
            v = b * n_q + j
            vis = int(lens[b]) - n_q + j + 1
            got = [int(plan.seq_lens[r][v]) for r in range(n_shards)]
            assert sum(got) == vis, (b, j, got, vis)
            # the visible rows are a prefix: shard r holds rows [64 lo_r, ...) in order
            for r in range(n_shards):
                lo, hi = bounds[r], bounds[r + 1]
                assert 0 <= got[r] <= (hi - lo) * bs
                if got[r] > 0:
                    assert sum(got[:r]) == lo * bs
                used = (got[r] + bs - 1) // bs
                assert plan.block_tables[r][v, :used].tolist() == bt[b, lo:lo + used].tolist()
    return plan


def test_shard_plan_splits_every_row_into_contiguous_page_ranges():
    g = torch.Generator().manual_seed(7)
    bs = 64
    for n_q in (1, 2, 3):
        for n_shards in (1, 2, 3, 5):
            batch = 6
            lens = torch.randint(n_q, 3000, (batch,), generator=g, dtype=torch.int32)
            lens[0] = n_q                       # shorter than one page
            lens[1] = 64 * 7                    # whole pages
            max_blocks = int((lens.max() + bs - 1) // bs) + 2
            bt = torch.randperm(batch * max_blocks, generator=g).reshape(batch, max_blocks).to(torch.int32)
            plan = _check_plan(bt, lens, n_q, bs, n_shards)
            assert len(plan.block_tables) == n_shards and plan.block_tables[0].dtype == torch.int32
            assert all(t.shape[0] == batch * n_q for t in plan.block_tables)


def test_shard_plan_rejects_bad_lengths():
    bt = torch.zeros(2, 4, dtype=torch.int32)
    for lens in ([0, 5], [5, 4 * 64 + 1]):
        try:
            shard_plan(bt, torch.tensor(lens, dtype=torch.int32), 1, 64, 2)
        except ValueError:
            continue
        raise AssertionError(f"accepted {lens}")


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        o = torch.full((3, 2, 8), float(rank + 1))
        lse = torch.full((3, 2), -float(rank))
        o_parts, lse_parts = gather_partials(o, lse)
        out[rank] = (tuple(o_parts.shape), o_parts[:, 0, 0, 0].tolist(), lse_parts[:, 0, 0].tolist())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_gather_partials_in_rank_order():
    world, port = 2, 29531
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    for r in range(world):
        assert out[r][0] == (2, 3, 2, 8)
        assert out[r][1] == [1.0, 2.0]
        assert out[r][2] == [0.0, -1.0]


def test_gather_without_a_process_group_is_the_local_pair():
    o, lse = torch.ones(2, 3, 4), torch.zeros(2, 3)
    a, b = gather_partials(o, lse)
    assert a.shape == (1, 2, 3, 4) and b.shape == (1, 2, 3)


def test_shard_plan_partials_merge_to_the_whole_attention():
    """Host-side plan against the oracle: for every query row, attention over
    each shard's visible rows (oracle), merged with the split merge, equals
    attention over all the rows the row sees (empty shards left out, as their
    lse is -inf on the device)."""
    import numpy as np
    import oracle
    g = np.random.default_rng(3)
    bs, H, d_c, d_r, n_q = 4, 2, 6, 2, 2
    lens = torch.tensor([1 + n_q, 9, 23], dtype=torch.int32)          # pages: 1, 3, 6
    batch = lens.numel()
    mb = 6
    bt = torch.arange(batch * mb, dtype=torch.int32).reshape(batch, mb)
    rows = {b: g.standard_normal((int(lens[b]), d_c + d_r)) for b in range(batch)}
    for n_shards in (2, 3, 4):
        plan = shard_plan(bt, lens, n_q, bs, n_shards)
        for b in range(batch):
            for j in range(n_q):
                v = b * n_q + j
                q_lat, q_r = g.standard_normal((H, d_c)), g.standard_normal((H, d_r))
                vis = int(lens[b]) - n_q + j + 1
                whole, lse_whole, _ = oracle.attend_absorbed(q_lat, q_r, rows[b][:vis, :d_c], rows[b][:vis, d_c:], 0.3)
                parts, lses = [], []
                for r in range(n_shards):
                    n = int(plan.seq_lens[r][v])
                    if n == 0:
                        continue
                    lo = int(plan.page_bounds[b, r]) * bs
                    o, lse, _ = oracle.attend_absorbed(q_lat, q_r, rows[b][lo:lo + n, :d_c], rows[b][lo:lo + n, d_c:], 0.3)
                    parts.append(o)
                    lses.append(lse)
                o, lse = oracle.merge_splits(np.stack(parts), np.stack(lses))
                assert np.allclose(o, whole, rtol=0, atol=1e-12) and np.allclose(lse, lse_whole, rtol=0, atol=1e-12)
