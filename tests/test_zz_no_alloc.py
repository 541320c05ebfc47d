"""mla_cache_append_noalloc against mla_cache_append, through the C ABI.

Some callers cannot allocate device memory: an engine that has reserved all
device memory for its own pool and forbids further cudaMalloc, or a plain C
caller with no device allocator, cannot hand mla_cache_append the workspace
it asks for.  The no-allocation variant takes its scratch from a fixed array
built into the library instead.  Its cache rows must equal those of the
regular entry point, call after call, even though every call reuses the same
library-owned scratch.

This file is collected last on purpose (and works alone in a fresh process).
"""

import pytest
import torch

from mla_synth import WORKLOADS, device_inputs, generate, reduced
from mla_latent_kv_39_b200 import Cache, Config, MLAError, abi, check_device_error

pytestmark = pytest.mark.gpu

CASES = [
    reduced(WORKLOADS["v3_b64_ragged1k_8k"], lengths=[100, 300, 5, 64]),
    reduced(WORKLOADS["tiny_f32_b1_l128"], lengths=[40, 7]),
]


def _bits(t: torch.Tensor) -> torch.Tensor:
    """Integer view, so that NaN-filled empty slots compare equal bit for bit."""
    return t.view(torch.int16) if t.element_size() == 2 else t.view(torch.int32)


@pytest.mark.parametrize("wl", CASES, ids=[c.name for c in CASES])
def test_noalloc_append_matches_regular_append_on_two_calls_in_a_row(wl):
    torch.cuda.set_device(0)
    data = generate(wl)
    dev = device_inputs(data, "cuda")
    cfg = Config.from_shape(wl.shape)
    W = dev["weights"]
    pool_a, pool_b = dev["pool"].clone(), dev["pool"].clone()
    cache_a, cache_b = Cache(pool_a, dev["block_table"]), Cache(pool_b, dev["block_table"])
    g = torch.Generator().manual_seed(123)
    for call in range(2):
        if call == 0:   # the step's new tokens at their new positions
            x, seq, pos = dev["x_new"], dev["seq_idx"], dev["pos"]
        else:           # other tokens, rewriting the first rows of every sequence
            n = 3 * wl.batch
            x = torch.randn(n, wl.shape.hidden, generator=g).to(wl.shape.torch_dtype).cuda()
            seq = torch.arange(wl.batch, dtype=torch.int32).repeat_interleave(3).cuda()
            pos = torch.arange(3, dtype=torch.int32).repeat(wl.batch).cuda()
        ws = torch.empty(abi.mla_cache_append_workspace_size(cfg, x.shape[0]), dtype=torch.uint8,
                         device="cuda")
        abi.mla_cache_append(cfg, x, W["W_DKV"], W["W_KR"], seq, pos, cache_a, ws)
        abi.mla_cache_append_noalloc(cfg, x, W["W_DKV"], W["W_KR"], seq, pos, cache_b)
        torch.cuda.synchronize()
        check_device_error()
        assert torch.equal(_bits(pool_a), _bits(pool_b)), f"call {call}: pools differ"
        # the rows were really written (empty slots hold NaN)
        bs = wl.shape.block_size
        for t in range(x.shape[0]):
            b, p = int(seq[t]), int(pos[t])
            page = int(dev["block_table"][b, p // bs])
            assert not torch.isnan(pool_b[page, p % bs].float()).any()


def test_noalloc_append_rejects_more_tokens_than_its_scratch_holds():
    torch.cuda.set_device(0)
    wl = reduced(WORKLOADS["v3_b64_ragged1k_8k"], lengths=[10])
    cfg = Config.from_shape(wl.shape)
    n_max = 1
    while abi.mla_cache_append_workspace_size(cfg, n_max + 1) <= abi.MLA_APPEND_NOALLOC_SCRATCH_BYTES:
        n_max += 1
    assert n_max >= 256     # room for the multi-token workload's 256 new tokens
    data = generate(wl)
    dev = device_inputs(data, "cuda")
    n = n_max + 1
    x = torch.zeros(n, wl.shape.hidden, dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros(n, dtype=torch.int32, device="cuda")
    before = abi.mla_kernel_launches()
    with pytest.raises(MLAError) as e:
        abi.mla_cache_append_noalloc(cfg, x, dev["weights"]["W_DKV"], dev["weights"]["W_KR"], idx, idx,
                                     Cache(dev["pool"], dev["block_table"]))
    assert e.value.status == abi.MLA_ERR_WORKSPACE
    assert abi.mla_kernel_launches() == before      # rejected before any launch
