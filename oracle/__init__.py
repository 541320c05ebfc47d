"""fp64 CPU oracle for the MLA latent-KV decode path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package.  The product
path (the C-ABI library and its Python binding) never calls it and has no
CPU fallback.

Parity status per function (pins live in ``tests/test_oracle_pins.py``):

* ``round_to_bf16``           pinned (IEEE ties-to-even cases, torch's fp32->bf16
                              cast on fp32-representable values, a double-rounding trap)
* ``rope``                    pinned (closed forms: identity at position 0, a
                              hand-evaluated rotation, norm and relative-position invariants)
* ``latent_rows``             pinned (same-x-different-position case, brute force)
* ``queries``                 pinned (brute force loops on the tiny shape)
* ``attend_decompressed``     pinned (brute force loops, T=1 and q=0 closed forms,
                              a hand-evaluated two-row case, causal masking case)
* ``attend_absorbed``         pinned (agrees with the decompressed order to 1e-10)
* ``merge_splits``            pinned (softmax over a union equals the merge of the parts)
* ``heads_from_latent`` and
  ``output_projection``       pinned (through the order-swap check and brute force)
* cache-size formulas         pinned (every byte count the pages print)
* ``e4m3_value``              pinned (every one of the 256 codes against torch's
                              float8_e4m3fn)
* ``round_to_e4m3``           pinned (torch's fp32 -> float8_e4m3fn cast on fp32
                              values within +-448, ties, subnormals, saturation)
* ``fp8_row_quantize``        pinned (power-of-two scales, the smallest that fit 448,
                              the boundary case, every value within half a code step,
                              zero rows, code x scale exact in bf16)
"""

from .mla import (  # noqa: F401
    round_to_bf16,
    round_to_storage,
    rope,
    softmax_scale,
    latent_rows,
    latent_rows_exact,
    e4m3_value,
    e4m3_code,
    round_to_e4m3,
    fp8_row_quantize,
    queries,
    absorb_query,
    attend_decompressed,
    attend_absorbed,
    heads_from_latent,
    output_projection,
    merge_splits,
    decode_step,
    mla_cache_bytes_per_token,
    gqa_cache_bytes_per_token,
    mha_cache_bytes_per_token,
    to64,
)
