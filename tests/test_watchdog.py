"""The bounded waits (the watchdog of every pipelined kernel here): a wait
whose arrival never comes gives up after its budget, records TQ_ERR_TIMEOUT
in the caller's status word and returns, leaving the context usable.

The failure is made on purpose but safely: one CTA, no cluster barrier, a
producer that withholds its arrival when the host says so, and a wait
budget of a few hundred microseconds.  Nothing faults, traps or hangs.
"""
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

TIMEOUT = 5
BUDGET = 1_000_000  # SM cycles: about half a millisecond


@pytest.fixture(scope="module")
def tq(cuda_ok):
    import rank_int4_gemm_b200 as m
    return m


def test_wait_that_is_served_reports_ok(tq):
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    ok = tq.tq_debug_watchdog(ws, withhold=False, budget_cycles=BUDGET)
    assert tq.tq_query_device_status(ws) == 0
    assert int(ok.item()) == 1


def test_withheld_arrival_times_out_and_context_survives(tq):
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    ok = tq.tq_debug_watchdog(ws, withhold=True, budget_cycles=BUDGET)
    assert tq.tq_query_device_status(ws) == TIMEOUT   # the wait gave up ...
    assert int(ok.item()) == 0                        # ... and the kernel returned
    assert tq.tq_query_device_status(ws) == 0         # the query cleared the word
    # the next normal call on the same workspace and context succeeds
    sh = synth.CONFIGS["tiny"]
    L = synth.make_layer(sh)
    X, L1t, L2t, Rt = (L[k].contiguous().cuda() for k in ("X", "L1t", "L2t", "Rt"))
    Wq, s_w = tq.tq_pack_weight(Rt, sh.had_block)
    Xq, s_x, XL1 = tq.tq_quantize_act(X, sh.had_block, L1t)
    Y = tq.tq_w4a4_lr_gemm(Xq, s_x, Wq, s_w, XL1, L2t, workspace=ws)
    torch.cuda.synchronize()
    assert torch.isfinite(Y.float()).all()
    assert tq.tq_query_device_status(ws) == 0


def test_watchdog_argument_checks(tq):
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(tq.TQError) as e:
        tq.tq_debug_watchdog(ws, withhold=True, budget_cycles=10)   # too short to be a wait
    assert e.value.status == 1
    with pytest.raises(tq.TQError) as e:
        tq.tq_debug_watchdog(ws[:128], withhold=True, budget_cycles=BUDGET)
    assert e.value.status == 6
