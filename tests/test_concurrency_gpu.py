"""Host-side concurrency and capture rules of the chunked prefill.

- Overlapped calls (at most 96 chains: the second kernel runs on the library's
  own stream, forked from and joined to the caller's) from two host threads on
  two streams at once give the single-threaded results bit for bit, call after
  call (the fork and join of each call are recorded and awaited under one lock).
- A chunked call on a capturing stream returns KDA_ERR_UNSUPPORTED and enqueues
  nothing: the chunk table it stages lives in host memory the call owns, which
  a replayed graph would read after it is gone."""
import threading

import numpy as np
import pytest
import torch

import kda_inputs as ki
import linear_attention_sequence_kda_b200 as kda
from parity import to_dev

pytestmark = pytest.mark.gpu


def _call(inp, d, ws, stream):
    with torch.cuda.stream(stream):
        out = kda.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["conv_w"], inp.cu_seqlens, d["cu_dev"],
                          d["init_state"], d["init_conv"], workspace=ws, stream=stream)
    return out


def test_two_threads_two_streams_overlapped_bitwise():
    problems = [ki.make_prefill([1500, 700], 8, torch.bfloat16, 71, state_std=0.02, conv_history=True),
                ki.make_prefill([2200], 16, torch.bfloat16, 72, state_std=0.02, conv_history=True)]
    devs = [to_dev(p) for p in problems]
    wss = [torch.empty(kda.workspace_size(p.num_seqs, p.total_tokens, p.num_heads,
                                          int(np.diff(p.cu_seqlens).max())), dtype=torch.uint8, device="cuda")
           for p in problems]
    assert all(p.num_seqs * p.num_heads <= 96 for p in problems)  # the overlapped schedule
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    refs = []
    for p, d, ws, s in zip(problems, devs, wss, streams):
        out = _call(p, d, ws, s)
        s.synchronize()
        refs.append([x.clone() for x in out])
    results = [[], []]
    errors = []

    def worker(i):
        try:
            for _ in range(6):
                out = _call(problems[i], devs[i], wss[i], streams[i])
                streams[i].synchronize()
                results[i].append([x.clone() for x in out])
        except Exception as e:  # reported below
            errors.append(e)

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    assert kda.check_async_status() == 0
    for i in range(2):
        assert len(results[i]) == 6
        for out in results[i]:
            for x, r in zip(out, refs[i]):
                assert torch.equal(x, r)


def test_capture_is_refused():
    inp = ki.make_prefill([300], 4, torch.bfloat16, 73)
    d = to_dev(inp)
    ws = torch.empty(kda.workspace_size(1, 300, 4, 300), dtype=torch.uint8, device="cuda")
    o = torch.zeros((300, 4, 128), dtype=torch.float32, device="cuda")
    S = torch.zeros((1, 4, 128, 128), dtype=torch.float32, device="cuda")
    tail = torch.zeros((1, 3, 3, 4 * 128), dtype=torch.bfloat16, device="cuda")
    cu_h = np.ascontiguousarray(inp.cu_seqlens.astype(np.int32))
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            rc = kda.lib.kda_prefill(d["q"].data_ptr(), d["k"].data_ptr(), d["v"].data_ptr(), d["g"].data_ptr(),
                                     d["beta"].data_ptr(), d["conv_w"].data_ptr(), None, None,
                                     d["cu_dev"].data_ptr(), cu_h.ctypes.data, 1, 4, kda.KDA_BF16,
                                     kda.KDA_CONV_NONE, kda.KDA_F32, kda.KDA_F32, o.data_ptr(), S.data_ptr(),
                                     tail.data_ptr(), ws.data_ptr(), ws.numel(), s.cuda_stream)
    assert rc == 2  # KDA_ERR_UNSUPPORTED
    graph.replay()  # the captured graph is empty: nothing was enqueued
    torch.cuda.synchronize()
    assert torch.count_nonzero(o) == 0 and torch.count_nonzero(S) == 0
    # the same call outside capture runs
    kda.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["conv_w"], inp.cu_seqlens, d["cu_dev"], o=o,
                final_state=S, conv_tail=tail, workspace=ws)
    torch.cuda.synchronize()
    assert torch.count_nonzero(o) > 0
