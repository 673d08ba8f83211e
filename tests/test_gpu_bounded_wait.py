"""The bounded barrier wait that every kernel uses gives up at its deadline: no fault, no hang, the
timeout bit reaches the host and the context stays usable. The wait runs against a barrier nothing
ever arrives on (pa_selftest_bounded_wait), so the failure is made without breaking anything."""
import time

import numpy as np
import pytest
import torch

import paged_kv_cache_385_b200 as pa
import workloads as W
from tests import oracle_case
from tests.device_case import TOL, DeviceCase

pytestmark = pytest.mark.gpu


def test_wait_on_a_barrier_nobody_arrives_at_gives_up_and_reports():
    word = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    pa.pa_selftest_bounded_wait(20000, word)  # 20 ms
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert int(word.item()) & pa.PA_DEVERR_TIMEOUT
    assert 0.019 <= dt < 5.0, dt
    # The library's own word when none is given.
    pa.pa_read_device_error(clear=True)
    pa.pa_selftest_bounded_wait(1000)
    assert pa.pa_read_device_error(clear=True) & pa.PA_DEVERR_TIMEOUT
    # The context still works: a decode afterwards matches the oracle.
    w = W.ALL["tiny"]
    want = oracle_case.expected_out(oracle_case.build(w))
    dev = DeviceCase(w)
    dev.write_new_token()
    out = dev.decode(kernel=1)
    torch.cuda.synchronize()
    assert float(np.max(np.abs(out.double().cpu().numpy() - want))) <= TOL[w.kv_dtype]
    assert pa.pa_read_device_error(clear=True) == 0
