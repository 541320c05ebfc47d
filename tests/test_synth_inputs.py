"""The seeded input generator: determinism, shapes and paged-layout validity."""

import torch

from mla_synth import WORKLOADS, build_pool, generate, reduced


def test_same_seed_same_values():
    wl = reduced(WORKLOADS["v3_b64_ragged1k_8k"], batch=3, len_lo=10, len_hi=200)
    a, b = generate(wl), generate(wl)
    for k in a.weights:
        assert torch.equal(a.weights[k], b.weights[k])
    assert torch.equal(a.cached_rows, b.cached_rows)
    assert torch.equal(a.block_table, b.block_table)
    c = generate(reduced(wl, seed=1))
    assert not torch.equal(a.x_new, c.x_new)


def test_without_weights_keeps_the_stream_aligned():
    wl = reduced(WORKLOADS["v2_b16_l4096"], lengths=[5, 7])
    a, b = generate(wl), generate(wl, with_weights=False)
    assert torch.equal(a.x_new, b.x_new) and torch.equal(a.cached_rows, b.cached_rows)


def test_ragged_lengths_in_range_and_blocks_cover_appended_rows():
    wl = reduced(WORKLOADS["v3_b128_nq2_ragged512_16k"], batch=20)
    d = generate(wl, with_weights=False)
    assert int(d.cached_len.min()) >= 512 and int(d.cached_len.max()) <= 16384
    bs = wl.shape.block_size
    used = []
    for b in range(wl.batch):
        need = (int(d.seq_lens[b]) + bs - 1) // bs
        row = d.block_table[b]
        assert bool((row[:need] >= 0).all()) and bool((row[need:] == -1).all())
        used.extend(row[:need].tolist())
    assert sorted(used) == list(range(d.num_blocks))   # every physical block used exactly once


def test_shuffled_blocks_are_a_permutation_not_identity():
    wl = reduced(WORKLOADS["v3_b64_ragged1k_8k"], batch=8, len_lo=100, len_hi=400)
    d = generate(wl, with_weights=False)
    flat = torch.cat([d.block_table[b][d.block_table[b] >= 0] for b in range(wl.batch)])
    assert sorted(flat.tolist()) == list(range(d.num_blocks))
    assert flat.tolist() != list(range(d.num_blocks))


def test_pool_places_row_t_of_seq_b_in_its_page():
    wl = reduced(WORKLOADS["v3_b64_ragged1k_8k"], batch=4, len_lo=1, len_hi=150)
    d = generate(wl, with_weights=False)
    pool = build_pool(d)
    bs = wl.shape.block_size
    for b in range(wl.batch):
        rows = d.seq_rows(b)
        for t in [0, len(rows) // 2, len(rows) - 1]:
            page = int(d.block_table[b, t // bs])
            assert torch.equal(pool[page, t % bs], rows[t])
        # slots past the cached rows are still NaN
        L = len(rows)
        page = int(d.block_table[b, L // bs])
        assert bool(torch.isnan(pool[page, L % bs].float()).all())


def test_spiked_rows_are_scaled_by_eight():
    wl = reduced(WORKLOADS["v3_b4_long"], lengths=[3000, 2000])
    d = generate(wl, with_weights=False)
    frac = float(d.spike_mask.float().mean())
    assert 0.005 < frac < 0.015
    big = d.cached_rows[d.spike_mask].float().abs().mean()
    small = d.cached_rows[~d.spike_mask].float().abs().mean()
    assert 6.0 < float(big / small) < 10.0


def test_fp8_workload_draws_codes_scales_and_keeps_the_weights():
    from mla_synth import build_row_scale
    wl = reduced(WORKLOADS["v3_fp8_b64_ragged1k_8k"], lengths=[70, 3])
    data = generate(wl)
    assert isinstance(data.weights, dict) and set(data.weights) >= {"W_DKV", "W_KR", "W_UK", "W_UV", "W_O"}
    assert data.cached_rows is None and data.cached_codes.dtype == torch.uint8
    assert data.cached_codes.shape == (73, wl.shape.row) and data.cached_scale.shape == (73,)
    codes = data.cached_codes.to(torch.int64)
    assert not bool(((codes & 0x7F) == 0x7F).any())            # never the NaN pattern
    m, _ = torch.frexp(data.cached_scale)
    assert bool((m == 0.5).all())                                   # powers of two, as the format has them
    pool = build_pool(data)
    scale = build_row_scale(data)
    assert pool.dtype == torch.uint8 and scale.shape == pool.shape[:2]
    b, t = 0, 65
    phys = int(data.block_table[b, t // 64])
    assert torch.equal(pool[phys, t % 64], data.cached_codes[t]) and scale[phys, t % 64] == data.cached_scale[t]
    assert generate(wl).cached_codes.equal(data.cached_codes)    # seeded
