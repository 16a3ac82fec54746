"""The bounded waits end with an error status, not a hang.

A debug kernel waits on something nothing will complete -- an mbarrier
phase, and a tagged word no CTA publishes -- with a budget of a few
microseconds.  The wait gives up, records the code in the device error word
and returns; tern_device_error reports it once and clears it; the context
stays usable (a streamed GEMV afterwards still matches the oracle)."""
import numpy as np
import pytest
import torch

import oracle
from ternary_weight_decode_b200 import synth, tern
from gpu_util import make_matrix, to_dev, tolerance

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kind", [0, 1])
def test_bounded_wait_runs_out_and_reports(kind):
    assert tern.tern_device_error() == 0
    tern.tern_debug_bounded_wait(kind, 20000)  # about 10 microseconds of SM clock
    code = tern.tern_device_error()
    assert code == 1, f"expected the timeout code, got {code}"
    assert tern.tern_device_error() == 0, "reading the error word clears it"
    # the context still works
    N, K = 300, 640
    w = synth.trits(45, 0, N, K)
    sw = synth.scales(45, 1, N, synth.groups(K))
    W = make_matrix(tern.TERN_FMT_BASE3, w, sw).retile_scales()
    xh = synth.activation_rows([800], K).astype(np.float32)
    y = torch.zeros((1, N), dtype=torch.float32, device="cuda")
    ws = tern.stream_workspace(tern.TERN_FMT_BASE3, N, 1, False)
    tern.tern_gemv_streamed(W, to_dev(xh), y, ws)
    q, s = oracle.act_quant(xh)
    ref = oracle.gemv(w, sw, q, s)
    assert np.max(np.abs(y.cpu().numpy() - ref)) <= tolerance(ref)
    assert tern.tern_device_error() == 0
