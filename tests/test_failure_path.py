"""The bounded-wait failure path, without a GPU fault: a kernel whose
mbarrier waits can never succeed (nothing arrives) gives up after the
library's limit, sets PA_DEV_TIMEOUT in the status word and returns; the
CUDA context stays usable for the next call."""
import time

import numpy as np
import pytest

import workloads
from pa_harness import assert_close, oracle_step, run_gpu

pytestmark = pytest.mark.gpu


def test_bounded_waits_time_out_and_the_context_survives():
    import torch
    import scatter_kv_b200 as pa
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    pa.pa_selftest_wait_timeout(st)
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    assert int(st.item()) == pa.PA_DEV_TIMEOUT
    assert 1.5 < waited < 30.0                    # the limit is 2 s per wait
    # The next calls run normally.
    spec = workloads.custom([1, 3, 40], [300, 20, 10], 8, 2, 64, 16, seed=5)
    x = workloads.generate(spec)
    got, _, status, _ = run_gpu(spec, x)
    want, _, _, _ = oracle_step(spec, x)
    assert status == 0
    assert_close(got, want, what="after a timed-out wait")
    assert np.isfinite(got.astype(np.float64)).all()
