"""The bounded-wait path on the GPU, without a fault: the chunked prefill's prep kernel is told
to issue none of its tile loads (gdn_debug_set_wait with GDN_INJECT_SKIP_PREP_LOADS) and the wait
limit is lowered to 2 ms, so the prep CTA's wait on its tile barrier runs out with nothing in
flight. The call must come back, the device status word must read GDN_ERR_TIMEOUT (and be
cleared by reading it), and a normal call afterwards must give correct results on the same
context."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from helpers import TOL_SCAN, rel_err, to_np, upload_scan_inputs

pytestmark = pytest.mark.gpu

GDN_ERR_TIMEOUT = 4


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import gated_deltanet_03_b200 as lib
    return lib


def test_prep_wait_runs_out_and_context_survives(g):
    # one 64-token chunk of one head: a single prep CTA, no segments
    w = workloads.custom("timeout", (64,), 1, 1, 128, io="bf16", s0_std=0.1, seed=91)
    x = workloads.generate(w)
    d = upload_scan_inputs(x, True)
    assert g.gdn_get_device_status() == 0
    g.gdn_debug_set_wait(2_000_000, g.INJECT_SKIP_PREP_LOADS)
    try:
        g.gdn_prefill_chunked(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"],
                              initial_state=d["initial_state"], out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert g.gdn_get_device_status() == GDN_ERR_TIMEOUT
        assert g.gdn_get_device_status() == 0          # reading it cleared it
    finally:
        g.gdn_debug_set_wait(0, 0)
    o, S = g.gdn_prefill_chunked(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"],
                                 initial_state=d["initial_state"], out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert g.gdn_get_device_status() == 0
    o_ref, S_ref = oracle.gdn_scan(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"],
                                   initial_state=x["initial_state"])
    assert rel_err(to_np(o), o_ref) <= TOL_SCAN
    assert rel_err(to_np(S), S_ref) <= TOL_SCAN


def test_debug_switches_are_checked(g):
    with pytest.raises(Exception):
        g.gdn_debug_set_wait(2_000_000_000, 0)      # above the default limit
    with pytest.raises(Exception):
        g.gdn_debug_set_wait(0, 1 << 7)             # no such switch
    g.gdn_debug_set_wait(0, 0)
