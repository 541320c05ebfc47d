"""Pins of the fp64 oracle against what the pages and mathematics fix.

None of these tests re-types an oracle formula.  Each pins the oracle to
something independent of it: a number the pages print, an IEEE rounding
case, a closed form, an invariant, an identity between the two computation
orders the pages name, or a brute-force loop evaluation on tiny inputs.
"""

from __future__ import annotations

import math
from pathlib import Path

import numpy as np
import pytest
import torch

import oracle
from oracle import (
    absorb_query,
    attend_absorbed,
    attend_decompressed,
    decode_step,
    gqa_cache_bytes_per_token,
    heads_from_latent,
    latent_rows,
    merge_splits,
    mha_cache_bytes_per_token,
    mla_cache_bytes_per_token,
    output_projection,
    queries,
    rope,
    round_to_bf16,
    softmax_scale,
)
from mla_synth import SHAPES, WORKLOADS, MLAShape, generate, reduced

GOLDEN = Path(__file__).parent / "golden"


def _golden(name):
    out = {}
    for line in (GOLDEN / name).read_text().splitlines():
        if not line.strip() or line.startswith("#"):
            continue
        key, rest = line.split("=", 1)
        out[key.strip()] = float(rest.split(";")[0])
    return out


# ---------------------------------------------------------------- rounding

def test_bf16_ties_go_to_even():
    # 1 + 2^-8 is exactly halfway between bf16 neighbours 1 and 1 + 2^-7.
    assert round_to_bf16(1.0 + 2.0 ** -8) == 1.0
    assert round_to_bf16(-(1.0 + 2.0 ** -8)) == -1.0
    # 1 + 3*2^-8 is halfway between 1 + 2^-7 (odd) and 1 + 2^-6 (even).
    assert round_to_bf16(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6
    # carry into the exponent: just below 2 rounds up to 2.
    assert round_to_bf16(2.0 - 2.0 ** -9) == 2.0


def test_bf16_rounds_once_from_float64():
    # Slightly above the midpoint: the correct result is 1 + 2^-7.  Going
    # through float32 first would drop the 2^-30 and land on the tie (-> 1.0).
    v = 1.0 + 2.0 ** -8 + 2.0 ** -30
    assert round_to_bf16(v) == 1.0 + 2.0 ** -7
    assert float(torch.tensor(v, dtype=torch.float32).to(torch.bfloat16)) == 1.0


def test_bf16_agrees_with_torch_cast_on_fp32_values():
    g = torch.Generator().manual_seed(1)
    a = torch.randn(200000, generator=g) * torch.exp2(torch.randint(-40, 40, (200000,), generator=g).float())
    ref = a.to(torch.bfloat16).to(torch.float64).numpy()
    got = round_to_bf16(a.to(torch.float64).numpy())
    assert np.array_equal(ref, got)


def test_bf16_special_values():
    big = (2.0 - 2.0 ** -7) * 2.0 ** 127
    got = round_to_bf16(np.array([0.0, -0.0, big, 2.0 ** 128, np.inf, -np.inf]))
    assert got[0] == 0.0 and got[1] == 0.0 and np.signbit(got[1])
    assert got[2] == big
    assert np.isinf(got[3]) and got[4] == np.inf and got[5] == -np.inf
    assert np.isnan(round_to_bf16(np.nan))


# -------------------------------------------------------------------- RoPE

def test_rope_is_identity_at_position_zero():
    v = np.random.default_rng(0).standard_normal((5, 64))
    assert np.array_equal(rope(v, np.zeros(5), 1e4), v)


def _rope_hand_case(fn):
    # d = 4, theta = 100, position 1: pair 0 turns by 1 rad, pair 1 by 100^(-1/2) = 0.1 rad.
    got = fn(np.array([1.0, 0.0, 0.0, 1.0]), 1, 100.0)
    want = [0.5403023058681398, 0.8414709848078965, -0.09983341664682815, 0.9950041652780258]
    assert np.allclose(got, want, rtol=0, atol=1e-15)


def test_rope_hand_evaluated_rotation():
    _rope_hand_case(rope)


def test_rope_preserves_norm_and_depends_on_relative_position():
    rng = np.random.default_rng(2)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    for m, n in [(0, 7), (100, 3), (131072, 65536)]:
        assert np.isclose(np.linalg.norm(rope(q, m, 1e4)), np.linalg.norm(q), rtol=1e-14)
        d0 = rope(q, m, 1e4) @ rope(k, n, 1e4)
        d1 = rope(q, m + 1234, 1e4) @ rope(k, n + 1234, 1e4)
        assert abs(d0 - d1) < 1e-9 * (1 + abs(d0))
    # and the rotation does depend on the offset
    assert abs(rope(q, 10, 1e4) @ rope(k, 0, 1e4) - q @ k) > 1e-6


# ------------------------------------------------------------- cache sizes

def test_worked_cache_example_of_the_pages():
    g = _golden("cache_sizes.txt")
    assert mla_cache_bytes_per_token(32, 512, 64, 2) == g["mla_L32_dc512_dr64_b2_bytes"]
    assert gqa_cache_bytes_per_token(32, 8, 128, 2) == g["gqa_L32_kv8_dh128_b2_bytes"]


def test_deepseek_v3_cache_figures():
    g = _golden("cache_sizes.txt")
    L, H = int(g["v3_layers"]), int(g["v3_query_heads"])
    per_tok = mla_cache_bytes_per_token(L, 512, 64, 2)
    assert 512 + 64 == g["v3_values_per_token"]
    assert round(per_tok / 1024, 1) == g["v3_kib_per_token"]
    # The page's per-head figure takes head_dim = hidden / heads = 7168 / 128 = 56;
    # that reading reproduces both printed numbers (24.9x and 13.34 GiB).
    per_head = mha_cache_bytes_per_token(L, H, 7168 // H, 2)
    assert round(per_head / per_tok, 1) == g["v3_ratio_vs_per_head"]
    assert round(8192 * per_tok / 2 ** 20) == g["v3_8k_mib"]
    assert round(8192 * per_head / 2 ** 30, 2) == g["v3_8k_per_head_gib"]
    # the footprint that the shapes here allocate per token and layer
    assert SHAPES["v3"].row * SHAPES["v3"].elem_bytes * L == per_tok


def test_mla_equals_gqa_with_2_25_groups():
    g = _golden("cache_sizes.txt")
    groups = mla_cache_bytes_per_token(1, 512, 64, 2) / gqa_cache_bytes_per_token(1, 1, 128, 2)
    assert groups == g["v2_equivalent_gqa_groups"]


def test_head_ratio_table():
    for line in (GOLDEN / "head_ratio_table.txt").read_text().splitlines():
        if not line.strip() or line.startswith("#"):
            continue
        _model, hq, hkv, factor = [s.strip() for s in line.split(";")]
        for layers, d_h in [(32, 128), (80, 128), (28, 96)]:
            mha = mha_cache_bytes_per_token(layers, int(hq), d_h, 2)
            gqa = gqa_cache_bytes_per_token(layers, int(hkv), d_h, 2)
            assert mha / gqa == float(factor)


# ------------------------------------------------ decoupled position (page 5 §5)

def _tiny_weights(seed=0):
    return generate(reduced(WORKLOADS["tiny_f32_b1_l128"], lengths=[4], seed=seed)).weights


def test_equal_latent_with_different_rotary_key_scores_differently():
    shape = SHAPES["tiny"]
    w = _tiny_weights()
    x = np.random.default_rng(3).standard_normal((1, shape.hidden))
    x2 = np.concatenate([x, x])
    c, kr = latent_rows(x2, w["W_DKV"], w["W_KR"], np.array([5, 9]), shape.rope_theta, "f32")
    assert np.array_equal(c[0], c[1])          # same content latent
    assert not np.allclose(kr[0], kr[1])      # different rotary key
    rng = np.random.default_rng(4)
    q_lat = rng.standard_normal((shape.n_heads, shape.d_c))
    q_r = rng.standard_normal((shape.n_heads, shape.d_r))
    scale = softmax_scale(shape.qk_nope, shape.d_r)
    _, _, s = attend_absorbed(q_lat, q_r, c, kr, scale)
    assert np.all(np.abs(s[:, 0] - s[:, 1]) > 1e-6)
    _, _, s0 = attend_absorbed(q_lat, np.zeros_like(q_r), c, kr, scale)
    assert np.array_equal(s0[:, 0], s0[:, 1])   # without the rotary branch position is lost


# ----------------------------------------------------------- brute force

def _brute_force(shape: MLAShape, W, x_cached, x_new, n_q):
    """Every quantity by explicit loops over scalars (one sequence)."""
    H, dc, dr, nope, dv, hid = (shape.n_heads, shape.d_c, shape.d_r, shape.qk_nope,
                                shape.v_head, shape.hidden)
    theta = shape.rope_theta

    def matvec(xrow, M, cols):
        return [sum(xrow[i] * M[i][j] for i in range(len(xrow))) for j in range(cols)]

    def rot(v, p):
        out = list(v)
        d = len(v)
        for i in range(d // 2):
            a = p * theta ** (-2.0 * i / d)
            out[2 * i] = v[2 * i] * math.cos(a) - v[2 * i + 1] * math.sin(a)
            out[2 * i + 1] = v[2 * i] * math.sin(a) + v[2 * i + 1] * math.cos(a)
        return out

    Wl = {k: np.asarray(v, dtype=np.float64).tolist() for k, v in W.items()}
    xs = [list(r) for r in np.asarray(x_cached, np.float64)] + [list(r) for r in np.asarray(x_new, np.float64)]
    L = len(xs) - n_q
    rows_c, rows_k = [], []
    for t, xr in enumerate(xs):
        rows_c.append([float(round_to_bf16(v)) if shape.dtype == "bf16" else float(np.float32(v))
                       for v in matvec(xr, Wl["W_DKV"], dc)])
        kr = rot(matvec(xr, Wl["W_KR"], dr), t)
        rows_k.append([float(round_to_bf16(v)) if shape.dtype == "bf16" else float(np.float32(v))
                       for v in kr])
    scale = 1.0 / math.sqrt(nope + dr)
    ys = []
    for j in range(n_q):
        t = L + j
        if "W_DQ" in Wl:
            q = matvec(matvec(xs[t], Wl["W_DQ"], shape.q_lora), Wl["W_UQ"], H * (nope + dr))
        else:
            q = matvec(xs[t], Wl["W_Q"], H * (nope + dr))
        o_all = []
        for h in range(H):
            qh = q[h * (nope + dr):(h + 1) * (nope + dr)]
            qn, qr = qh[:nope], rot(qh[nope:], t)
            logits = []
            for u in range(t + 1):
                k_n = [sum(rows_c[u][a] * Wl["W_UK"][a][h * nope + n] for a in range(dc)) for n in range(nope)]
                logits.append(scale * (sum(qn[n] * k_n[n] for n in range(nope)) +
                                       sum(qr[n] * rows_k[u][n] for n in range(dr))))
            mx = max(logits)
            ws = [math.exp(s - mx) for s in logits]
            z = sum(ws)
            o_h = [0.0] * dv
            for u in range(t + 1):
                v_u = [sum(rows_c[u][a] * Wl["W_UV"][a][h * dv + n] for a in range(dc)) for n in range(dv)]
                for n in range(dv):
                    o_h[n] += ws[u] / z * v_u[n]
            o_all.extend(o_h)
        ys.append(matvec(o_all, Wl["W_O"], hid))
    return np.array(rows_c), np.array(rows_k), np.array(ys)


BRUTE_SHAPE = MLAShape("brute", hidden=6, n_heads=2, d_c=5, d_r=4, qk_nope=3, v_head=2,
                       q_lora=0, rope_theta=50.0, dtype="f32")
BRUTE_SHAPE_Q = MLAShape("brute_q", hidden=7, n_heads=3, d_c=4, d_r=2, qk_nope=2, v_head=3,
                         q_lora=3, rope_theta=20.0, dtype="bf16")


@pytest.mark.parametrize("n_q,shape", [(1, BRUTE_SHAPE), (2, BRUTE_SHAPE), (2, BRUTE_SHAPE_Q), (5, BRUTE_SHAPE)])
def test_oracle_matches_brute_force_loops(n_q, shape):
    rng = np.random.default_rng(10 + n_q)
    W = {k: rng.standard_normal(s) / math.sqrt(s[0]) for k, s in shape.weight_shapes().items()}
    x_cached = rng.standard_normal((5, shape.hidden))
    x_new = rng.standard_normal((n_q, shape.hidden))
    rc, rk, ys = _brute_force(shape, W, x_cached, x_new, n_q)
    L = len(x_cached)
    c_old, kr_old = latent_rows(x_cached, W["W_DKV"], W["W_KR"], np.arange(L), shape.rope_theta,
                                shape.dtype)
    assert np.allclose(c_old, rc[:L], rtol=1e-6, atol=1e-7)   # both round to fp32 storage
    assert np.allclose(kr_old, rk[:L], rtol=1e-6, atol=1e-7)
    for order in ("decompressed", "absorbed"):
        out = decode_step(shape, W, x_new, L + np.arange(n_q), [rc[:L]], [rk[:L]], n_q, order=order)
        assert np.allclose(out["c_new"], rc[L:], rtol=1e-6, atol=1e-7)
        for j in range(n_q):
            assert np.allclose(out["y"][j], ys[j], rtol=1e-10, atol=1e-12), order


# ----------------------------------------------- the two computation orders

ORDER_CASES = [
    ("tiny_f32_b1_l128", None, None),
    ("v2_b16_l4096", [37, 5], None),
    ("v3_b64_ragged1k_8k", [70, 1], None),
    ("v3_b4_long", [150], None),
    ("v3_b128_nq2_ragged512_16k", [9, 66], 2),
]


@pytest.mark.parametrize("name,lengths,n_q", ORDER_CASES, ids=[c[0] for c in ORDER_CASES])
def test_absorbed_order_equals_decompressed_order(name, lengths, n_q):
    """Matrix absorption reorders the computation but keeps the function."""
    wl = WORKLOADS[name]
    if lengths is not None:
        wl = reduced(wl, lengths=lengths, n_q=n_q)
    d = generate(wl)
    shape = wl.shape
    if wl.cached_from_append:
        L = int(d.cached_len[0])
        c, kr = latent_rows(d.x_cached, d.weights["W_DKV"], d.weights["W_KR"], np.arange(L),
                            shape.rope_theta, shape.dtype)
        cc, ck = [c], [kr]
    else:
        rows = [oracle.to64(d.seq_rows(b)) for b in range(wl.batch)]
        cc = [r[:, :shape.d_c] for r in rows]
        ck = [r[:, shape.d_c:] for r in rows]
    pos = d.new_positions().numpy()
    a = decode_step(shape, d.weights, d.x_new, pos, cc, ck, wl.n_q, order="decompressed")
    b = decode_step(shape, d.weights, d.x_new, pos, cc, ck, wl.n_q, order="absorbed")
    for t in a["y"]:
        for key in ("logits", "o_heads", "y"):
            ref = a[key][t]
            assert np.max(np.abs(b[key][t] - ref)) <= 1e-10 * np.max(np.abs(ref)), key


# -------------------------------------------------------- closed forms

def test_single_visible_row_returns_it():
    rng = np.random.default_rng(5)
    c = rng.standard_normal((1, 8))
    kr = rng.standard_normal((1, 4))
    o, lse, s = attend_absorbed(rng.standard_normal((3, 8)), rng.standard_normal((3, 4)), c, kr, 0.3)
    assert np.array_equal(o, np.repeat(c, 3, axis=0))
    assert np.array_equal(lse, s[:, 0])


def test_zero_query_averages_rows():
    rng = np.random.default_rng(6)
    c = rng.standard_normal((7, 8))
    o, lse, _ = attend_absorbed(np.zeros((2, 8)), np.zeros((2, 4)), c, rng.standard_normal((7, 4)), 1.0)
    assert np.allclose(o, np.mean(c, axis=0)[None], rtol=0, atol=1e-15)
    assert np.allclose(lse, math.log(7), rtol=0, atol=1e-15)


def test_two_row_hand_case():
    # rows c = 1 and 3, query 1, scale 0.5 -> logits 0.5 and 1.5 -> o = 1 + 2*sigmoid(1)
    o, lse, _ = attend_absorbed(np.array([[1.0]]), np.zeros((1, 2)), np.array([[1.0], [3.0]]),
                                np.zeros((2, 2)), 0.5)
    assert abs(o[0, 0] - 2.4621171572600098) < 1e-15
    assert abs(lse[0] - 1.8132616875182228) < 1e-15   # log(e^0.5 + e^1.5)


def test_first_new_token_does_not_see_the_second():
    shape = BRUTE_SHAPE
    rng = np.random.default_rng(7)
    W = {k: rng.standard_normal(s) / math.sqrt(s[0]) for k, s in shape.weight_shapes().items()}
    x_cached = rng.standard_normal((4, shape.hidden))
    c, kr = latent_rows(x_cached, W["W_DKV"], W["W_KR"], np.arange(4), shape.rope_theta, "f32")
    x_new = rng.standard_normal((2, shape.hidden))
    x_alt = x_new.copy()
    x_alt[1] *= 50.0     # a very different second token
    pos = np.array([4, 5])
    a = decode_step(shape, W, x_new, pos, [c], [kr], 2)
    b = decode_step(shape, W, x_alt, pos, [c], [kr], 2)
    assert np.array_equal(a["y"][0], b["y"][0])
    assert not np.allclose(a["y"][1], b["y"][1])


# --------------------------------------------------------- split merge

def test_merge_of_parts_equals_attention_over_union():
    rng = np.random.default_rng(8)
    T, H, dc, dr = 50, 3, 6, 2
    c, kr = rng.standard_normal((T, dc)), rng.standard_normal((T, dr))
    q_lat, q_r = 3 * rng.standard_normal((H, dc)), rng.standard_normal((H, dr))
    full_o, full_lse, _ = attend_absorbed(q_lat, q_r, c, kr, 0.7)
    cuts = [0, 1, 17, 49, 50]
    parts = [attend_absorbed(q_lat, q_r, c[a:b], kr[a:b], 0.7) for a, b in zip(cuts[:-1], cuts[1:])]
    o, lse = merge_splits(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
    assert np.allclose(o, full_o, rtol=0, atol=1e-13)
    assert np.allclose(lse, full_lse, rtol=0, atol=1e-13)
    o1, l1 = merge_splits(full_o[None], full_lse[None])
    assert np.array_equal(o1, full_o) and np.array_equal(l1, full_lse)


# ---------------------------------------------- planted mistakes are caught

def test_a_planted_rope_sign_error_is_caught():
    def wrong_rope(v, pos, theta):
        v = np.asarray(v, dtype=np.float64)
        d = v.shape[-1]
        i = np.arange(d // 2)
        ang = np.asarray(pos, dtype=np.float64)[..., None] * np.power(float(theta), -2.0 * i / d)
        out = np.empty(np.broadcast_shapes(v.shape, ang.shape[:-1] + (d,)))
        out[..., 0::2] = v[..., 0::2] * np.cos(ang) + v[..., 1::2] * np.sin(ang)
        out[..., 1::2] = -v[..., 0::2] * np.sin(ang) + v[..., 1::2] * np.cos(ang)
        return out

    with pytest.raises(AssertionError):
        _rope_hand_case(wrong_rope)


def test_a_planted_transposed_head_slice_is_caught(monkeypatch):
    """Slicing W_UK per head the wrong way must break the brute-force pin."""
    import oracle.mla as m
    orig = m.attend_decompressed

    def wrong(q_nope, q_r, c, k_r, W_UK, W_UV, n_heads, qk_nope, v_head, scale):
        W = np.asarray(W_UK, dtype=np.float64)
        Wt = W.reshape(W.shape[0], qk_nope, n_heads).transpose(0, 2, 1).reshape(W.shape)
        return orig(q_nope, q_r, c, k_r, Wt, W_UV, n_heads, qk_nope, v_head, scale)

    monkeypatch.setattr(m, "attend_decompressed", wrong)
    with pytest.raises(AssertionError):
        test_oracle_matches_brute_force_loops(1, BRUTE_SHAPE)


def test_a_planted_dropped_rotary_term_is_caught(monkeypatch):
    import oracle.mla as m

    def wrong(q_lat, q_r, c, k_r, scale):
        return attend_absorbed(q_lat, np.zeros_like(np.asarray(q_r, dtype=np.float64)), c, k_r, scale)

    monkeypatch.setattr(m, "attend_absorbed", wrong)
    with pytest.raises(AssertionError):
        test_oracle_matches_brute_force_loops(1, BRUTE_SHAPE)


# ---------------------------------------------------------------- FP8 cache format

def test_e4m3_value_of_every_code_matches_torch_float8_e4m3fn():
    codes = np.arange(256, dtype=np.uint8)
    mine = oracle.e4m3_value(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(mine), np.isnan(ref))
    assert np.array_equal(mine[~np.isnan(mine)], ref[~np.isnan(ref)])
    assert np.nanmax(mine) == 448.0 and oracle.e4m3_value(np.array([1], np.uint8))[0] == 2.0 ** -9
    assert np.isnan(mine[0x7F]) and np.isnan(mine[0xFF]) and np.sum(np.isnan(mine)) == 2


def test_round_to_e4m3_matches_torch_on_fp32_values_and_ties():
    g = np.random.default_rng(5)
    x = (g.standard_normal(100000) * np.exp(g.uniform(-14, 6.5, 100000))).astype(np.float32)
    x = x[np.abs(x) <= 448]
    table = oracle.e4m3_value(np.arange(256, dtype=np.uint8))
    grid = np.unique(table[np.isfinite(table)])
    ties = ((grid[:-1] + grid[1:]) / 2).astype(np.float32)       # exact midpoints (fp32-exact)
    for v in (x, ties):
        ref = torch.from_numpy(v).to(torch.float8_e4m3fn).to(torch.float64).numpy()
        assert np.array_equal(oracle.round_to_e4m3(v.astype(np.float64)), ref)
    # ties to even: 1 + 1/16 lies between 1 and 1.125 -> 1 (even mantissa); 1 + 3/16 -> 1.25
    assert oracle.round_to_e4m3(np.array([1.0625, 1.1875, -1.0625]))[[0, 1, 2]].tolist() == [1.0, 1.25, -1.0]
    # saturation beyond the largest finite value (torch gives NaN there)
    assert oracle.round_to_e4m3(np.array([449.0, 1e9, -1e9])).tolist() == [448.0, 448.0, -448.0]
    # one rounding from float64 (no fp32 detour): just above a tie goes up
    above = 1.0625 + 2.0 ** -40
    assert oracle.round_to_e4m3(np.array([above]))[0] == 1.125
    codes = oracle.e4m3_code(np.array([1.0, -448.0, 2.0 ** -9, 0.0, -0.0]))
    assert codes.tolist() == [0x38, 0xFE, 0x01, 0x00, 0x80]
    every = np.arange(256, dtype=np.uint8)
    finite = np.isfinite(oracle.e4m3_value(every))
    assert np.array_equal(oracle.e4m3_code(oracle.e4m3_value(every))[finite], every[finite])
    assert np.signbit(oracle.round_to_e4m3(np.array([-2.0 ** -12]))[0])    # underflow keeps the sign


def test_fp8_row_quantize_takes_the_smallest_power_of_two_scale_within_half_a_step():
    g = np.random.default_rng(9)
    rows = g.standard_normal((50, 576)) * np.exp(g.uniform(-8, 8, (50, 1)))
    codes, scale = oracle.fp8_row_quantize(rows)
    m, _ = np.frexp(scale)
    assert np.all(m == 0.5)                                               # powers of two
    amax = np.max(np.abs(rows), axis=1)
    assert np.all(amax / scale <= 448.0) and np.all(amax / scale > 224.0)  # the smallest such power
    big = np.max(np.abs(codes), axis=1)
    assert np.all((big >= 224.0) & (big <= 448.0))       # (224, 448] rounds into [224, 448]
    # a row whose max is exactly 448 * 2^k takes scale 2^k (the boundary case)
    edge = np.zeros((1, 8))
    edge[0, 3] = 448.0 * 2.0 ** -5
    ce, se = oracle.fp8_row_quantize(edge)
    assert se[0] == 2.0 ** -5 and ce[0, 3] == 448.0
    # the stored value code * scale is a bf16 number (4 significant bits times 2^k)
    assert np.array_equal(oracle.round_to_bf16(codes * scale[:, None]), codes * scale[:, None])
    # |row / s - code| <= half the code step at that magnitude (subnormal step 2^-9)
    _, e = np.frexp(np.abs(codes) + (codes == 0))
    step = np.ldexp(1.0, np.maximum(e - 4, -9))
    assert np.all(np.abs(rows / scale[:, None] - codes) <= step / 2 * (1 + 1e-12))
    # an all-zero row: scale 1, codes 0
    z_codes, z_scale = oracle.fp8_row_quantize(np.zeros((1, 8)))
    assert z_scale[0] == 1.0 and not np.any(z_codes)
    # the fp8 storage path of latent_rows returns code * scale per row
    c, k = oracle.latent_rows(rows[:3, :64], np.eye(64)[:, :48], np.eye(64)[:, 48:], np.zeros(3), 1e4, "fp8")
    joined = np.concatenate([c, k], axis=1)
    cc, ss = oracle.fp8_row_quantize(rows[:3, :64])
    assert np.array_equal(joined, cc * ss[:, None])
