"""Per-token cache footprint measured on the real allocation.

[P5] section 4 asks to count the persistent tensors actually allocated and to
compare them with the formula; [P4] "Multi-head latent attention (MLA)" prints
the DeepSeek-V3 figure (61 layers x 576 values, 68.6 KiB per token in 16-bit
storage).  Here the pools are allocated exactly as the library's callers
allocate them (``mla_synth.build_pool`` for the host copy, the same shape and
dtype on the device), and their bytes are divided by their token slots.
"""

import pytest
import torch

from pathlib import Path

from mla_synth import WORKLOADS, generate, build_pool, reduced


def _golden():
    out = {}
    for line in (Path(__file__).parent / "golden" / "cache_sizes.txt").read_text().splitlines():
        if line.strip() and not line.startswith("#"):
            key, rest = line.split("=", 1)
            out[key.strip()] = float(rest.split(";")[0])
    return out


GOLDEN_KIB = _golden()["v3_kib_per_token"]     # printed to one decimal on the page
LAYERS = int(_golden()["v3_layers"])


def _bytes_per_slot(pool: torch.Tensor) -> float:
    slots = pool.shape[0] * pool.shape[1]
    return pool.numel() * pool.element_size() / slots


def test_host_pool_is_1152_bytes_per_token_and_layer():
    data = generate(reduced(WORKLOADS["v3_b64_ragged1k_8k"], lengths=[700, 130, 64]), with_weights=False)
    pool = build_pool(data)
    assert pool.dtype == torch.bfloat16 and pool.shape[1:] == (64, 576)
    per_layer = _bytes_per_slot(pool)
    assert per_layer == 1152
    per_token = LAYERS * per_layer
    assert per_token == 70272 and per_token / 1024 == 68.625
    assert round(per_token / 1024, 1) == GOLDEN_KIB


@pytest.mark.gpu
def test_device_pools_of_61_layers_allocate_68_625_kib_per_token():
    torch.cuda.synchronize()
    slots = 64 * 64          # 64 pages of 64 tokens per layer
    before = torch.cuda.memory_allocated()
    pools = [torch.empty(64, 64, 576, dtype=torch.bfloat16, device="cuda") for _ in range(LAYERS)]
    grown = torch.cuda.memory_allocated() - before
    assert grown == sum(p.numel() * p.element_size() for p in pools)
    per_token = grown / slots
    assert per_token == 70272 and per_token / 1024 == 68.625
    assert round(per_token / 1024, 1) == GOLDEN_KIB
    del pools
