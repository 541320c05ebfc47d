"""Plain fp64 NumPy restatement of MLA decode (test infrastructure only).

Sources, cited by page title and section:

* "Multi-head Latent Attention (MLA) Nedir?" (yapayzekasozluk.tr), section
  "MLA nasıl çalışır?": each token's hidden state is compressed to a small
  latent c_KV that is the only thing cached (Compression); full K and V are
  rebuilt from it when attention runs (Decompression); position goes through
  a separate RoPE key kept outside the compression (Decoupled RoPE); queries
  get the same kind of compression.
* "GQA, MQA ve MLA: attention KV cache'i nasıl belirler" (LLMScale), section
  "Multi-head latent attention (MLA)": per token and layer the cache holds one
  latent of kv_lora_rank values plus one small rotary key; the cost is
  layers x (kv_lora_rank + qk_rope_head_dim) x bytes, with no head factor.
* "MLA · latent KV, decoupled RoPE và matrix absorption" (openarchlab),
  section 1 "Định nghĩa": the decompression matrix can be folded into the
  query and output matrices (matrix absorption), which reorders the
  computation without changing the function; section 2 "Luồng": project
  hidden to latent, write the cache, read it and project the output; section
  3 "Giải pháp": the cache-size formulas; section 5 "Ví dụ": a worked
  byte count and the rule that equal latents with different rotary keys give
  different scores.

The pages give no equations, so every open point takes the plainest
reading (listed in the design notes): row-vector convention ``y = x W`` with
weights stored ``[in, out]``; RoPE rotates adjacent pairs ``(2i, 2i+1)`` by
``pos * theta**(-2i/d)``; softmax scale ``1/sqrt(qk_nope + d_r)``; a new token
attends to every cached row and to itself (causal); no norms or biases.

Everything here runs in float64.  The latent rows are rounded once, to the
cache storage type, because those rounded values *are* the cache.
"""

from __future__ import annotations

import math
from typing import Dict, Iterable, List, Optional, Sequence, Tuple

import numpy as np

# --------------------------------------------------------------------------
# Storage rounding
# --------------------------------------------------------------------------

_BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127


def round_to_bf16(a) -> np.ndarray:
    """Nearest bfloat16 value of each float64 entry, ties to even, as float64.

    bfloat16 keeps 8 significant bits (7 stored) and fp32's exponent range.
    The rounding is taken directly from the float64 value (never through an
    intermediate float32, which could round twice).
    """
    a = np.asarray(a, dtype=np.float64)
    out = np.array(a, dtype=np.float64, copy=True)
    fin = np.isfinite(a) & (a != 0.0)
    if np.any(fin):
        v = a[fin]
        _, e = np.frexp(v)                   # v = m * 2**e with 0.5 <= |m| < 1
        q = np.maximum(e - 8, -133)          # quantum: 2**(e-8); bf16 subnormal step 2**-133
        r = np.rint(np.ldexp(v, -q))         # exact scaling, then ties-to-even
        w = np.ldexp(r, q)
        w = np.where(np.abs(w) > _BF16_MAX, np.copysign(np.inf, w), w)
        out[fin] = w
    return out


def round_to_storage(a, dtype: str) -> np.ndarray:
    """Round float64 values to the cache storage type ("bf16" or "f32")."""
    if dtype == "bf16":
        return round_to_bf16(a)
    if dtype == "f32":
        return np.asarray(a, dtype=np.float64).astype(np.float32).astype(np.float64)
    raise ValueError(f"unknown storage dtype {dtype!r}")


# OCP 8-bit floating point, E4M3 variant: 1 sign bit, 4 exponent bits (bias
# 7), 3 mantissa bits; no infinities, exponent field 15 with mantissa 7 is
# NaN, so the largest finite magnitude is 1.75 * 2**8 = 448; subnormals
# (exponent field 0) are m * 2**-9.  The pages fix no cache number format;
# this is the common FP8 cache format, with one scale per row ("MLA ve diğer
# optimizasyonlarla ilişkisi": quantization is used together with MLA).
_E4M3_MAX = 448.0


def e4m3_value(codes) -> np.ndarray:
    """The value of each E4M3 byte (uint8 array), as float64 (NaN codes -> NaN)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.power(2.0, e - 7))
    mag = np.where((e == 15) & ((c & 0x7) == 7), np.nan, mag)
    return sign * mag


def round_to_e4m3(a) -> np.ndarray:
    """Nearest E4M3 value of each float64 entry, ties to even, magnitudes
    beyond 448 saturating to +-448; as float64."""
    a = np.asarray(a, dtype=np.float64)
    out = np.array(a, dtype=np.float64, copy=True)
    fin = np.isfinite(a) & (a != 0.0)
    if np.any(fin):
        v = a[fin]
        _, e = np.frexp(v)                   # v = m * 2**e with 0.5 <= |m| < 1
        q = np.maximum(e - 4, -9)            # 4 significant bits; subnormal step 2**-9
        w = np.ldexp(np.rint(np.ldexp(v, -q)), q)
        out[fin] = np.clip(w, -_E4M3_MAX, _E4M3_MAX)
    return out


def e4m3_code(values) -> np.ndarray:
    """The byte of each E4M3 value (inverse of ``e4m3_value`` on finite
    values; the sign of a zero is kept: -0 is 0x80)."""
    v = np.asarray(values, dtype=np.float64)
    table = e4m3_value(np.arange(256, dtype=np.uint8))
    codes = np.zeros(v.shape, dtype=np.uint8)
    for c in range(256):
        if table[c] == 0.0 or not np.isfinite(table[c]):
            continue
        codes[v == table[c]] = c
    codes[(v == 0.0) & np.signbit(v)] = 0x80
    return codes


def fp8_row_quantize(rows) -> Tuple[np.ndarray, np.ndarray]:
    """Per-row scaled E4M3 of float64 rows ``[..., width]``.

    ``scale`` = the smallest power of two with ``max |row| / scale <= 448``
    (1 where the row is zero); the stored codes are ``round_to_e4m3(row /
    scale)``.  Returns ``(code_values, scale)`` as float64; the cached row
    stands for ``code_values * scale`` (exact in bf16: 4 significant bits
    times a power of two).
    """
    r = np.asarray(rows, dtype=np.float64)
    amax = np.max(np.abs(r), axis=-1)
    f, e = np.frexp(amax / _E4M3_MAX)          # amax / 448 = f 2**e, 0.5 <= f < 1
    scale = np.ldexp(1.0, np.where(f == 0.5, e - 1, e))
    scale = np.where(amax == 0.0, 1.0, scale)
    return round_to_e4m3(r / scale[..., None]), scale


def to64(t) -> np.ndarray:
    """A CPU tensor or array as float64 NumPy (bf16 and fp32 widen exactly)."""
    if hasattr(t, "detach"):
        import torch
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


# --------------------------------------------------------------------------
# Decoupled RoPE
# --------------------------------------------------------------------------

def rope(v: np.ndarray, pos, theta: float) -> np.ndarray:
    """Rotary position embedding of the last axis of ``v``.

    Adjacent pairs ``(v[2i], v[2i+1])`` are rotated counter-clockwise by the
    angle ``pos * theta**(-2i/d)``, i = 0 .. d/2-1 (the RoFormer form).
    ``pos`` broadcasts against the leading axes of ``v``.
    """
    v = np.asarray(v, dtype=np.float64)
    d = v.shape[-1]
    if d % 2:
        raise ValueError("RoPE width must be even")
    i = np.arange(d // 2, dtype=np.float64)
    inv_freq = np.power(float(theta), -2.0 * i / d)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * inv_freq
    cos, sin = np.cos(ang), np.sin(ang)
    even, odd = v[..., 0::2], v[..., 1::2]
    out = np.empty(np.broadcast_shapes(v.shape, ang.shape[:-1] + (d,)), dtype=np.float64)
    out[..., 0::2] = even * cos - odd * sin
    out[..., 1::2] = even * sin + odd * cos
    return out


def softmax_scale(qk_nope: int, d_r: int) -> float:
    """Scaled dot product over the full per-head key ``[k_nope, k_R]``."""
    return 1.0 / math.sqrt(qk_nope + d_r)


# --------------------------------------------------------------------------
# Step 1: hidden -> latent row (the cache)
# --------------------------------------------------------------------------

def latent_rows_exact(x, W_DKV, W_KR, pos, theta: float) -> Tuple[np.ndarray, np.ndarray]:
    """``c_KV = x W_DKV`` (the compressed latent) and ``k_R = RoPE(x W_KR, pos)``
    (the decoupled rotary key) of tokens ``x`` at positions ``pos``, unrounded."""
    x = to64(x)
    c = x @ to64(W_DKV)
    r = x @ to64(W_KR)
    return c, rope(r, np.asarray(pos), theta)


def latent_rows(x, W_DKV, W_KR, pos, theta: float, dtype: str) -> Tuple[np.ndarray, np.ndarray]:
    """Cache rows ``(c_KV, k_R)`` of tokens ``x`` at absolute positions ``pos``,
    each value rounded once to the cache storage type; for ``"fp8"`` the
    values the FP8 rows stand for (``fp8_row_quantize`` of ``[c_KV | k_R]``)."""
    c, k_r = latent_rows_exact(x, W_DKV, W_KR, pos, theta)
    if dtype == "fp8":
        codes, scale = fp8_row_quantize(np.concatenate([c, k_r], axis=-1))
        v = codes * scale[..., None]
        return v[..., :c.shape[-1]], v[..., c.shape[-1]:]
    return round_to_storage(c, dtype), round_to_storage(k_r, dtype)


# --------------------------------------------------------------------------
# Step 2: queries and absorption of W_UK
# --------------------------------------------------------------------------

def queries(x, weights: Dict[str, np.ndarray], n_heads: int, qk_nope: int, d_r: int,
            pos, theta: float) -> Tuple[np.ndarray, np.ndarray]:
    """Per-head query parts ``(q_nope [n, H, qk_nope], q_R [n, H, d_r])``.

    With query compression ``q = (x W_DQ) W_UQ``, else ``q = x W_Q``.  Head h
    owns columns ``[h (qk_nope + d_r), (h + 1)(qk_nope + d_r))`` of q: first
    its no-position part, then its rotary part, which is rotated at the
    token's position.  Nothing is rounded.
    """
    x = to64(x)
    if "W_DQ" in weights:
        q = (x @ to64(weights["W_DQ"])) @ to64(weights["W_UQ"])
    else:
        q = x @ to64(weights["W_Q"])
    n = x.shape[0]
    q = q.reshape(n, n_heads, qk_nope + d_r)
    q_nope = q[..., :qk_nope]
    q_r = rope(q[..., qk_nope:], np.asarray(pos)[:, None], theta)
    return q_nope, q_r


def absorb_query(q_nope, W_UK, n_heads: int, qk_nope: int) -> np.ndarray:
    """Fold W_UK into the no-position query: ``q_lat_h = W_UK_h q_nope_h``.

    ``W_UK`` is ``[d_c, H * qk_nope]``; head h's key is ``k_h = c W_UK_h`` with
    ``W_UK_h = W_UK[:, h qk_nope:(h + 1) qk_nope]``, so
    ``q_nope_h . k_h = (W_UK_h q_nope_h) . c``.  Returns ``[..., H, d_c]``.
    """
    W = to64(W_UK).reshape(W_UK.shape[0], n_heads, qk_nope)      # [d_c, H, nope]
    return np.einsum("chn,...hn->...hc", W, to64(q_nope))


# --------------------------------------------------------------------------
# Step 3: attention, in both orders
# --------------------------------------------------------------------------

def _softmax(s: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    z = np.sum(e, axis=-1, keepdims=True)
    return e / z, (m + np.log(z))[..., 0]


def attend_decompressed(q_nope, q_r, c, k_r, W_UK, W_UV, n_heads: int, qk_nope: int,
                        v_head: int, scale: float):
    """Textbook attention of one query token over visible cache rows.

    For every head h the full key and value are rebuilt from the latent
    (decompression): ``K_h = [c W_UK_h, k_R]`` (``[T, qk_nope + d_r]``) and
    ``V_h = c W_UV_h`` (``[T, v_head]``).  Then ``s = K_h q_h * scale``,
    ``p = softmax(s)`` and ``o_h = p V_h``.

    Inputs: ``q_nope [H, qk_nope]``, ``q_r [H, d_r]``, ``c [T, d_c]``,
    ``k_r [T, d_r]`` (only the rows this query may see).
    Returns ``(o_heads [H, v_head], logits [H, T])``.
    """
    c, k_r = to64(c), to64(k_r)
    W_UK, W_UV = to64(W_UK), to64(W_UV)
    q_nope, q_r = to64(q_nope), to64(q_r)
    T = c.shape[0]
    o = np.zeros((n_heads, v_head))
    logits = np.zeros((n_heads, T))
    for h in range(n_heads):
        K = np.concatenate([c @ W_UK[:, h * qk_nope:(h + 1) * qk_nope], k_r], axis=1)
        V = c @ W_UV[:, h * v_head:(h + 1) * v_head]
        q = np.concatenate([q_nope[h], q_r[h]])
        s = (K @ q) * scale
        p, _ = _softmax(s)
        o[h] = p @ V
        logits[h] = s
    return o, logits


def attend_absorbed(q_lat, q_r, c, k_r, scale: float):
    """Attention in latent space, with W_UK already folded into the query.

    ``s_t = (q_lat_h . c_t + q_R_h . k_R_t) * scale``, ``p = softmax(s)``,
    ``o_lat_h = sum_t p_t c_t``.  Inputs ``q_lat [H, d_c]``, ``q_r [H, d_r]``,
    ``c [T, d_c]``, ``k_r [T, d_r]``.  Returns ``(o_lat [H, d_c],
    lse [H] (natural log-sum-exp of the scaled logits), logits [H, T])``.
    """
    c, k_r = to64(c), to64(k_r)
    s = (to64(q_lat) @ c.T + to64(q_r) @ k_r.T) * scale
    p, lse = _softmax(s)
    return p @ c, lse, s


def merge_splits(o_parts, lse_parts) -> Tuple[np.ndarray, np.ndarray]:
    """Merge softmax-normalised partial outputs of disjoint row subsets.

    Part s holds ``o_s = sum_{t in s} e^{s_t} c_t / sum_{t in s} e^{s_t}`` and
    ``lse_s = log sum_{t in s} e^{s_t}``.  The result over the union is
    ``sum_s e^{lse_s - M} o_s / sum_s e^{lse_s - M}`` with ``M = max_s lse_s``,
    and its log-sum-exp is ``M + log sum_s e^{lse_s - M}``.
    Arrays are stacked on axis 0 (``o_parts [S, ..., d]``, ``lse_parts [S, ...]``).
    """
    o_parts = to64(o_parts)
    lse_parts = to64(lse_parts)
    M = np.max(lse_parts, axis=0)
    w = np.exp(lse_parts - M)
    z = np.sum(w, axis=0)
    o = np.sum(w[..., None] * o_parts, axis=0) / z[..., None]
    return o, M + np.log(z)


# --------------------------------------------------------------------------
# Step 4: output side
# --------------------------------------------------------------------------

def heads_from_latent(o_lat, W_UV, n_heads: int, v_head: int) -> np.ndarray:
    """Fold W_UV into the output side: ``o_h = o_lat_h W_UV_h`` (``[..., H, v_head]``)."""
    W = to64(W_UV).reshape(W_UV.shape[0], n_heads, v_head)        # [d_c, H, v]
    return np.einsum("...hc,chv->...hv", to64(o_lat), W)


def output_projection(o_heads, W_O) -> np.ndarray:
    """``y = concat_h(o_h) W_O`` for ``o_heads [n, H, v_head]``."""
    o = to64(o_heads)
    return o.reshape(o.shape[0], -1) @ to64(W_O)


# --------------------------------------------------------------------------
# A whole decode step
# --------------------------------------------------------------------------

def decode_step(shape, weights, x_new, pos_new, cached_c: Sequence, cached_kr: Sequence,
                n_q: int, order: str = "decompressed", seqs: Optional[Iterable[int]] = None,
                want_y: bool = True, cache_dtype: Optional[str] = None) -> Dict[str, object]:
    """One decode step of one layer (cache append, queries, attention, output).

    ``cached_c[b]`` / ``cached_kr[b]`` are the rows already cached for
    sequence b (storage-rounded values).  Token ``b * n_q + j`` (hidden state
    ``x_new``, position ``pos_new``) first appends its own latent row, then
    attends to the ``len(cached_c[b]) + j + 1`` rows up to and including its
    own.  ``order`` picks the decompressed textbook order or the absorbed
    order; ``seqs`` restricts the attention to some sequences (the append and
    query projections always cover every token).

    Returns a dict with ``c_new, kr_new, q_nope, q_r, q_lat`` for every token
    and, per attended token t (dict keyed by t), ``o_heads`` and, in the
    absorbed order, ``o_lat``/``lse``; plus ``y`` rows for attended tokens.
    ``cache_dtype`` ("fp8" for the E4M3 cache) overrides the storage type of
    the appended rows, which is otherwise the shape's.
    """
    H, nope, dr, dv = shape.n_heads, shape.qk_nope, shape.d_r, shape.v_head
    scale = softmax_scale(nope, dr)
    W = {k: to64(v) for k, v in weights.items()}
    pos_new = np.asarray(pos_new)
    c_new, kr_new = latent_rows(x_new, W["W_DKV"], W["W_KR"], pos_new, shape.rope_theta,
                                cache_dtype or shape.dtype)
    q_nope, q_r = queries(x_new, W, H, nope, dr, pos_new, shape.rope_theta)
    q_lat = absorb_query(q_nope, W["W_UK"], H, nope)
    B = len(cached_c)
    seqs = range(B) if seqs is None else list(seqs)
    out: Dict[str, object] = {"c_new": c_new, "kr_new": kr_new, "q_nope": q_nope,
                              "q_r": q_r, "q_lat": q_lat, "o_heads": {}, "o_lat": {},
                              "lse": {}, "logits": {}, "y": {}}
    for b in seqs:
        c_b, kr_b = to64(cached_c[b]), to64(cached_kr[b])
        for j in range(n_q):
            t = b * n_q + j
            rows_c = np.concatenate([c_b, c_new[b * n_q:t + 1]], axis=0)
            rows_kr = np.concatenate([kr_b, kr_new[b * n_q:t + 1]], axis=0)
            if order == "decompressed":
                o_h, logits = attend_decompressed(q_nope[t], q_r[t], rows_c, rows_kr, W["W_UK"],
                                                  W["W_UV"], H, nope, dv, scale)
            elif order == "absorbed":
                o_lat, lse, logits = attend_absorbed(q_lat[t], q_r[t], rows_c, rows_kr, scale)
                o_h = heads_from_latent(o_lat, W["W_UV"], H, dv)
                out["o_lat"][t] = o_lat
                out["lse"][t] = lse
            else:
                raise ValueError(order)
            out["o_heads"][t] = o_h
            out["logits"][t] = logits
            if want_y:
                out["y"][t] = output_projection(o_h[None], W["W_O"])[0]
    return out


# --------------------------------------------------------------------------
# Cache-size formulas
# --------------------------------------------------------------------------

def mla_cache_bytes_per_token(layers: int, d_c: int, d_r: int, elem_bytes: int) -> int:
    """MLA: layers x (d_c + d_R) x bytes; the head count drops out."""
    return layers * (d_c + d_r) * elem_bytes


def gqa_cache_bytes_per_token(layers: int, kv_heads: int, d_h: int, elem_bytes: int) -> int:
    """GQA with uniform groups: 2 (K and V) x layers x KV heads x head dim x bytes."""
    return 2 * layers * kv_heads * d_h * elem_bytes


def mha_cache_bytes_per_token(layers: int, heads: int, d_h: int, elem_bytes: int) -> int:
    """MHA: every query head keeps its own K and V head."""
    return 2 * layers * heads * d_h * elem_bytes
