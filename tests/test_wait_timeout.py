"""The bounded-wait path of the tensor-core kernels, made to run out on purpose.

Every barrier wait in the decode and weight-GEMM kernels gives up after a time
limit, records MLA_ERR_TIMEOUT in the device error word and lets the kernel
return.  Here a one-warp kernel waits on a barrier whose second arrival never
comes, with a 1 ms limit: the status must come back as MLA_ERR_TIMEOUT, the
stream must finish, and the library must keep working afterwards.
"""

import time

import pytest
import torch

from mla_latent_kv_39_b200 import abi
from mla_synth import WORKLOADS, reduced

from mla_gpu_cases import run_gpu

pytestmark = pytest.mark.gpu


def test_a_wait_with_a_missing_arrival_times_out_and_returns():
    torch.cuda.synchronize()
    assert abi.mla_get_device_error()[0] == abi.MLA_OK
    t0 = time.perf_counter()
    abi.mla_check_wait_timeout(1_000_000)            # 1 ms
    status, detail = abi.mla_get_device_error()       # synchronises the stream
    elapsed = time.perf_counter() - t0
    assert status == abi.MLA_ERR_TIMEOUT and detail[0] == 1
    assert elapsed < 5.0
    assert abi.mla_get_device_error()[0] == abi.MLA_OK   # cleared by the first read
    # the context is still usable: a small decode step runs and checks clean
    run_gpu(reduced(WORKLOADS["v3_b64_ragged1k_8k"], lengths=[100, 7]))


def test_the_limit_is_checked_on_the_host():
    with pytest.raises(abi.MLAError) as e:
        abi.mla_check_wait_timeout(0)
    assert e.value.status == abi.MLA_ERR_INVALID_ARG
