"""A bounded barrier wait of the attention kernel that runs out, on a valid
problem, without any fault.

Every barrier wait in the KV-block-outer attention kernel has a time limit
(2 s by default).  msa_debug_set_attn_wait_limit_ns lowers it; at 1 us the
pipeline's first waits (the epilogue's wait for the first output tile, the
MMA issuer's for the first K tile) run out while loads and tensor-core work
are in flight.  The kernel must then drain what it issued, free its tensor
memory, report MSA_DEVERR_TIMEOUT on the device flag and return; the call
after it, with the default limit, must run normally and give the oracle's
result -- the context is still usable.  No input is invalid and nothing
traps: the only change is the limit.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_32_b200 import capi, pipeline, workloads as wl

from _helpers import assert_rows_ok, bits, compare_rows

pytestmark = pytest.mark.gpu

CASES = [
    # R = 8: Q rows gathered by TMA boxes (one issuing warp)
    (wl.small("timeout_r8", 1, 1500, 1500, 0, 16, 2, 128, seed=41), False),
    (wl.small("timeout_r8_compact", 1, 1500, 1500, 0, 16, 2, 128, seed=41), True),
    # R = 4: Q rows gathered by cp.async (128 threads)
    (wl.small("timeout_r4", 1, 1500, 1500, 0, 8, 2, 64, seed=42), False),
]


@pytest.mark.parametrize("w,compact", CASES, ids=lambda c: getattr(c, "name", str(c)))
def test_attention_wait_timeout_is_reported_and_the_next_call_runs(w, compact):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    d = pipeline.dims_for(w)
    buf = pipeline.Buffers.allocate(d, compact=compact)
    inp = wl.make_inputs(w, "cuda")
    sel = wl.random_selection(w, "cpu")
    buf.sel.copy_(sel)
    fwd = capi.msa_sparse_attn_fwd_compact if compact else capi.msa_sparse_attn_fwd
    capi.msa_build_block_query_lists(d, buf.sel, buf.blk_offsets, buf.entries, buf.entry_pos,
                                     buf.ws, buf.dev_err)
    torch.cuda.synchronize()
    assert int(buf.dev_err[0]) == 0
    prev = capi.msa_debug_set_attn_wait_limit_ns(1000)
    try:
        fwd(d, inp["q"], inp["k"], inp["v"], buf.blk_offsets, buf.entries, buf.part_ml,
            buf.part_acc, buf.dev_err)
        torch.cuda.synchronize()
        code = int(buf.dev_err[0])
    finally:
        assert capi.msa_debug_set_attn_wait_limit_ns(prev) == 1000
    assert code == 1, code                                   # MSA_DEVERR_TIMEOUT
    # default limit again: the same problem runs through and matches the oracle
    buf.dev_err.zero_()
    pipeline.attend(buf, inp["q"], inp["k"], inp["v"])
    torch.cuda.synchronize()
    assert int(buf.dev_err[0]) == 0
    rows = np.arange(0, w.n_q, 37, dtype=np.int64)
    pos = w.q_pos0 + rows
    bat = np.zeros_like(rows)
    q_rows = bits(inp["q"])[0, rows]
    sel_rows = sel[0].permute(1, 0, 2)[torch.from_numpy(rows)].numpy()
    out, lse = oracle.attention(q_rows, pos, bat, bits(inp["k"]), bits(inp["v"]), sel_rows,
                                w.scale)
    res = compare_rows(buf.out[0, torch.from_numpy(rows).cuda()].float().cpu().numpy(),
                       buf.lse[0, torch.from_numpy(rows).cuda()].cpu().numpy(), out, lse)
    assert_rows_ok(res, w.name)
