"""Failure detection without a GPU fault: a bounded wait runs out and is reported."""
import time

import pytest
import torch

pytestmark = pytest.mark.gpu


def test_a_wait_that_nobody_satisfies_times_out_and_is_reported():
    import hierarchical_block_sparse_pyr_b200 as P

    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.time()
    P.selftest_wait(status)
    torch.cuda.synchronize()
    took = time.time() - t0
    assert int(status.item()) == P.PYR_ETIMEOUT
    assert took < 30.0
    # the context is still usable afterwards
    x = torch.arange(1024, device="cuda", dtype=torch.float32)
    assert float(x.sum().item()) == 1023 * 1024 / 2
