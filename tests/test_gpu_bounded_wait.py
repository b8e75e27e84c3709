"""The kernels' bounded wait made to run out on purpose (a barrier nothing
completes): the wait gives up after its 2 s limit, the status word reports
MOE_STATUS_TIMEOUT, the kernel ends normally and the context stays usable.
No GPU fault, trap or hang is involved."""
import numpy as np
import pytest
import torch

import mixture_experts_ffn_sort_b200 as moe
import oracle

pytestmark = pytest.mark.gpu


def test_expired_wait_sets_status_and_context_survives():
    status, elapsed = moe.moe_selftest_bounded_wait()
    assert status == moe.MOE_STATUS_TIMEOUT
    # The first wait expires at the limit; the second on the abort flag the
    # first raises (or its own limit), never much later.
    assert 1.9e9 <= elapsed[0] <= 3.0e9, elapsed
    assert 0 < elapsed[1] <= 3.0e9, elapsed
    # The context still runs kernels correctly.
    lg = np.random.default_rng(7).standard_normal((32, 16)).astype(np.float32)
    ids, _ = moe.moe_route(torch.from_numpy(lg).cuda(), 4)
    torch.cuda.synchronize()
    assert np.array_equal(ids.cpu().numpy(), oracle.route(lg, 4)[0])
