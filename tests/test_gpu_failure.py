"""The bounded-wait error path on the GPU, made to run out on purpose without a fault: a wait
on an mbarrier that nothing completes gives up after a short cycle limit, records the
wait-timeout code in the device error word and returns, and the context stays usable."""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_reports_and_leaves_the_context_usable(cuda):
    import looped_hybrid_attention_b200 as L
    L.device_error_status()                        # clear whatever an earlier test left
    L.wait_selftest(2_000_000)                     # about 1 ms of SM clock
    torch.cuda.synchronize()
    assert L.device_error_status() == 6            # LOOP_ERR_TIMEOUT, reported once
    assert L.device_error_status() == 0            # reading cleared it
    # the context still works: a projection afterwards is exact to fp32 rounding
    X = synth.normal((40, 256), 1.0, 90, "Xw").cuda()
    W = synth.normal((96, 256), 0.05, 90, "Ww").cuda()
    Y = torch.empty((40, 96), device=cuda)
    L.linear(X, W, Y, L.EPI_STORE)
    torch.cuda.synchronize()
    ref = X.double().cpu().numpy() @ W.double().cpu().numpy().T
    assert np.abs(Y.double().cpu().numpy() - ref).max() < 1e-4 * np.abs(ref).max()
    assert L.device_error_status() == 0
