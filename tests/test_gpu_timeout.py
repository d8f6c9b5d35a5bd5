"""Failure detection without a GPU fault: the attention kernel's waits are bounded.

With the producer told to issue no loads (a test hook), nothing ever completes the K/V
barriers; each wait gives up after its time limit, the kernel records VDIT_ERR_TIMEOUT in the
device status word, frees its tensor memory and exits. The host reads the status and the
context stays usable: the next normal call succeeds and matches the oracle."""
import numpy as np
import pytest

import video_diffusion_transformer_vdit_b200 as vdit
from video_diffusion_transformer_vdit_b200.workloads import WORKLOADS

from _parity import assert_close, dev, f64, inputs, run_oracle, run_product

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    w = WORKLOADS[1]
    q, k, v = inputs(w)
    o, _, cache, plan = run_product(w, q, k, v, lse=False)
    assert vdit.get_status() == vdit.OK
    L = vdit.lib()
    L.vdit_debug_skip_loads(1)
    try:
        vdit.attn_forward(plan, dev(q), cache, scale=w.scale)
        status = vdit.get_status()  # synchronises: the kernel returns after its wait limit
    finally:
        L.vdit_debug_skip_loads(0)
    assert status == vdit.ERR_TIMEOUT
    assert vdit.get_status() == vdit.OK  # reading clears the word
    o2 = vdit.attn_forward(plan, dev(q), cache, scale=w.scale)
    ro, _ = run_oracle(w, q, k, v, np.arange(w.q_tokens), range(w.heads))
    assert_close(f64(o2), ro)
    assert vdit.get_status() == vdit.OK
