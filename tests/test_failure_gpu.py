"""Failure detection on the GPU without a GPU fault.

A host-side injected fault (kda_inject_fault(KDA_FAULT_DROP_READY)) launches
the overlapped chunked prefill's preparation kernel without its per-chunk ready
flags: the message the scan waits for is dropped.  The scan's bounded wait runs
out, every block drains its own copies and tensor-core work, frees its tensor
memory and returns; the device status word then reads KDA_ERR_TIMEOUT through
kda_check_async_status, and the context stays usable: the same call gives the
result it gave before the failure, bit for bit."""
import time

import pytest
import torch

import kda_inputs as ki
import linear_attention_sequence_kda_b200 as kda
from parity import run_prefill, to_dev

pytestmark = pytest.mark.gpu
BF = torch.bfloat16


def _call(inp, d, recurrent=False):
    """One prefill whose asynchronous status is returned, not asserted."""
    o, S, tail = kda.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["conv_w"], inp.cu_seqlens, d["cu_dev"],
                             d["init_state"], d["init_conv"], recurrent=recurrent)
    return kda.check_async_status(), (o, S, tail)


def test_dropped_ready_flags_time_out_and_context_recovers():
    # 2 segments x 4 heads = 8 scan chains: the overlapped mode
    inp = ki.make_prefill([300, 130], 4, BF, 91, state_std=0.02, conv_history=True)
    d = to_dev(inp)
    want = run_prefill(inp, dev_inputs=d)
    try:
        kda.inject_fault(kda.KDA_FAULT_DROP_READY)
        # a call that has no ready flags (the recurrent path) leaves the fault pending
        status, got = _call(inp, d, recurrent=True)
        assert status == 0
        t0 = time.monotonic()
        status, _ = _call(inp, d)
        elapsed = time.monotonic() - t0
    finally:
        kda.inject_fault(kda.KDA_FAULT_NONE)
    assert status == 6, kda.STATUS.get(status, status)  # KDA_ERR_TIMEOUT
    assert elapsed < 60.0  # bounded: the scan's waits give up well within two seconds
    assert kda.check_async_status() == 0  # the status word was read and cleared
    # the fault was taken by the call that applied it: the next call is whole
    for _ in range(2):
        status, got = _call(inp, d)
        assert status == 0
        assert all(torch.equal(a, b) for a, b in zip(got, want))
    # other entry points on the same context
    dec = ki.make_decode(3, 4, BF, 92)
    state = dec.state.cuda()
    kda.decode_step(state, dec.conv_cache.clone().cuda(), dec.q.cuda(), dec.k.cuda(), dec.v.cuda(), dec.g.cuda(),
                    dec.beta.cuda(), dec.conv_w.cuda())
    assert kda.check_async_status() == 0
    assert torch.isfinite(state).all()
