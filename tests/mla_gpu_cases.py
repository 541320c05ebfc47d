"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
on seeded inputs, and compute the oracle's expectation for the same inputs."""

from __future__ import annotations

from typing import Dict, Iterable, Optional

import numpy as np
import torch

import oracle
from mla_synth import device_inputs, generate
from mla_latent_kv_39_b200 import Cache, Config, DecodeLayer, check_device_error


def tol_for(shape) -> float:
    """max|err| <= tol * max|ref| (bf16 storage: 1e-2; fp32: 1e-4)."""
    return 1e-2 if shape.dtype == "bf16" else 1e-4


def run_gpu(wl, data=None, max_workers: int = 0, pool: Optional[torch.Tensor] = None, packed_query: bool = True):
    data = data if data is not None else generate(wl)
    dev = device_inputs(data, "cuda", pool=pool)
    cfg = Config.from_shape(wl.shape, split_query=wl.split_query, fp8_cache=wl.fp8_cache)
    cache = Cache(dev["pool"], dev["block_table"], dev["row_scale"])
    layer = DecodeLayer(cfg, dev["weights"], cache, wl.batch, wl.n_q, max_workers, packed_query=packed_query)
    if wl.cached_from_append:
        layer.append(dev["x_cached"], dev["seq_idx_cached"], dev["pos_cached"])
    layer.step(dev["x_new"], dev["seq_idx"], dev["pos"], dev["seq_lens"], want_o_lat=True)
    torch.cuda.synchronize()
    check_device_error()
    return data, dev, layer


def oracle_cached_rows(data):
    """(c, k_R) rows already cached for every sequence, from the seeded inputs only."""
    wl, shape = data.workload, data.workload.shape
    cc, ck = [], []
    for b in range(wl.batch):
        s, e = int(data.row_offsets[b]), int(data.row_offsets[b + 1])
        if wl.cached_from_append:
            c, kr = oracle.latent_rows(data.x_cached[s:e], data.weights["W_DKV"], data.weights["W_KR"],
                                       np.arange(e - s), shape.rope_theta, shape.dtype)
        elif wl.fp8_cache:     # the values the stored codes and scales stand for
            rows = oracle.e4m3_value(data.cached_codes[s:e].numpy()) * \
                oracle.to64(data.cached_scale[s:e])[:, None]
            c, kr = rows[:, :shape.d_c], rows[:, shape.d_c:]
        else:
            rows = oracle.to64(data.cached_rows[s:e])
            c, kr = rows[:, :shape.d_c], rows[:, shape.d_c:]
        cc.append(c)
        ck.append(kr)
    return cc, ck


def oracle_expect(data, seqs: Optional[Iterable[int]] = None, order: str = "absorbed") -> Dict:
    wl = data.workload
    cc, ck = oracle_cached_rows(data)
    out = oracle.decode_step(wl.shape, data.weights, data.x_new, data.new_positions().numpy(), cc, ck,
                             wl.n_q, order=order, seqs=seqs, cache_dtype="fp8" if wl.fp8_cache else None)
    out["cached_c"], out["cached_kr"] = cc, ck
    return out


def assert_close(got, ref, tol, what):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = np.max(np.abs(got - ref))
    bound = tol * np.max(np.abs(ref))
    assert err <= bound, f"{what}: max|err| {err:.3e} > {tol:g} * max|ref| = {bound:.3e}"
    return err / max(np.max(np.abs(ref)), 1e-300)


def pool_row(layer, data, b: int, p: int) -> np.ndarray:
    bs = data.workload.shape.block_size
    page = int(data.block_table[b, p // bs])
    return oracle.to64(layer.cache.pool[page, p % bs].cpu())


def check_new_cache_rows(layer, data, exp):
    """Rows appended by the step are bit-identical to the oracle's rounded rows
    (for an FP8 cache: the E4M3 bytes and the fp32 row scale)."""
    wl = data.workload
    pos = data.new_positions().numpy()
    if wl.fp8_cache:
        W = data.weights
        c, k = oracle.latent_rows_exact(data.x_new, W["W_DKV"], W["W_KR"], pos, wl.shape.rope_theta)
        codes, scale = oracle.fp8_row_quantize(np.concatenate([c, k], axis=1))
        want = oracle.e4m3_code(codes)
        bs = wl.shape.block_size
        for t in range(wl.n_tok):
            b = t // wl.n_q
            page = int(data.block_table[b, int(pos[t]) // bs])
            got = layer.cache.pool[page, int(pos[t]) % bs].cpu().numpy()
            bad = np.nonzero(got != want[t])[0]
            assert bad.size == 0, f"token {t}: {bad.size} FP8 codes differ, first at {bad[:5]}"
            got_s = float(layer.cache.row_scale[page, int(pos[t]) % bs].cpu())
            assert got_s == scale[t], f"token {t}: row scale {got_s!r} != {scale[t]!r}"
        return
    want = np.concatenate([exp["c_new"], exp["kr_new"]], axis=1)
    for t in range(wl.n_tok):
        b = t // wl.n_q
        got = pool_row(layer, data, b, int(pos[t]))
        bad = np.nonzero(got != want[t])[0]
        assert bad.size == 0, f"token {t}: {bad.size} cache values differ, first at {bad[:5]}"


def check_outputs(layer, data, exp, tokens: Iterable[int]):
    wl = data.workload
    tol = tol_for(wl.shape)
    ql, qr = layer.queries_fp32()
    q_lat = oracle.to64(ql.cpu())
    q_rope = oracle.to64(qr.cpu())
    o_lat = layer.o_lat.cpu().double().numpy()
    y = oracle.to64(layer.y.cpu())
    worst = {}
    for t in tokens:
        worst.setdefault("q_lat", []).append(assert_close(q_lat[t], exp["q_lat"][t], tol, f"q_lat[{t}]"))
        worst.setdefault("q_rope", []).append(assert_close(q_rope[t], exp["q_r"][t], tol, f"q_rope[{t}]"))
        worst.setdefault("o_lat", []).append(assert_close(o_lat[t], exp["o_lat"][t], tol, f"o_lat[{t}]"))
        worst.setdefault("y", []).append(assert_close(y[t], exp["y"][t], tol, f"y[{t}]"))
    return {k: max(v) for k, v in worst.items()}
