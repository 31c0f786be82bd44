"""kda_prefill_noalloc: the prefill entry point for callers that cannot
allocate device memory (a server whose memory is all pre-reserved in its own
pools, a plugin whose host owns every allocation).  It must give the same
results as kda_prefill with a caller workspace, call after call, although every
call reuses one static device scratch array."""
import numpy as np
import pytest
import torch

import kda_inputs as ki
import linear_attention_sequence_kda_b200 as kda
from parity import to_dev


def test_noalloc_rejects_problems_beyond_the_static_scratch():
    # host-side check before any launch: fake, aligned device addresses are
    # never dereferenced on this path
    H, T = 64, 1 << 20
    need = kda.workspace_size(1, T, H, T)
    assert need > kda.NOALLOC_SCRATCH_BYTES
    cu = np.array([0, T], dtype=np.int32)
    fake = [(i + 1) << 20 for i in range(10)]
    rc = kda.lib.kda_prefill_noalloc(fake[0], fake[1], fake[2], fake[3], fake[4], fake[5], None, None,
                                     fake[6], cu.ctypes.data, 1, H, kda.KDA_BF16, 0, kda.KDA_F32, kda.KDA_F32,
                                     fake[7], fake[8], fake[9], None)
    assert rc == 4  # KDA_ERR_WORKSPACE


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_on_two_calls_in_a_row():
    """Both entry points run the same kernels on the same inputs, and the
    chunked path is deterministic, so the results must be equal bit for bit.
    The cases cover both schedules of the chunked path: at most 96 (sequence,
    head) chains (the scan overlaps the preparation kernel) and more (the two
    run one after the other), all through the one static scratch array."""
    cases = [ki.make_prefill([200, 37], 4, torch.bfloat16, 31, state_std=0.02, conv_history=True),
             ki.make_prefill([65, 1, 300], 2, torch.bfloat16, 32, state_std=0.02, conv_history=True),
             ki.make_prefill([64, 200, 130, 77, 1, 128, 190, 65], 16, torch.bfloat16, 33, state_std=0.02,
                             conv_history=True)]
    assert cases[2].num_seqs * cases[2].num_heads > 96
    for inp in cases:  # different problems back to back through the same scratch
        assert kda.workspace_size(inp.num_seqs, inp.total_tokens, inp.num_heads,
                                  int(np.diff(inp.cu_seqlens).max())) <= kda.NOALLOC_SCRATCH_BYTES
        d = to_dev(inp)
        args = (d["q"], d["k"], d["v"], d["g"], d["beta"], d["conv_w"], inp.cu_seqlens, d["cu_dev"],
                d["init_state"], d["init_conv"])
        for _ in range(2):  # two calls in a row of each entry point
            o_ref, s_ref, t_ref = kda.prefill(*args)
            o_na, s_na, t_na = kda.prefill_noalloc(*args)
            torch.cuda.synchronize()
            assert kda.check_async_status() == 0
            assert torch.equal(o_na, o_ref)
            assert torch.equal(s_na, s_ref)
            assert torch.equal(t_na, t_ref)
