"""The allocation-free block->query list builder against the workspace one.

msa_build_block_query_lists_noalloc exists for callers that cannot allocate
device memory where they build the lists (a plugin whose host process owns
all device memory through its own pool, a loop that must not allocate): its
scratch is a fixed device array inside the library.  This file checks,
through the C ABI, that it produces exactly the lists of the workspace
version (integer output: bit-exact), on two calls in a row -- the second one
finds the previous call's data in the shared scratch -- and that a problem
too large for the built-in scratch is refused before anything runs.

It is named to be collected last, so a run that stops at its first failure
has already run every other test.
"""
import pytest
import torch

from block_sparse_attention_32_b200 import build as msa_build
from block_sparse_attention_32_b200 import capi, pipeline, workloads as wl

pytestmark = pytest.mark.gpu


def _lists_with_workspace(d, sel):
    buf = pipeline.Buffers.allocate(d)
    capi.msa_build_block_query_lists(d, sel, buf.blk_offsets, buf.entries, buf.entry_pos,
                                     buf.ws, buf.dev_err)
    torch.cuda.synchronize()
    assert int(buf.dev_err[0]) == 0
    return buf.blk_offsets.clone(), buf.entries.clone(), buf.entry_pos.clone()


def _lists_without_workspace(d, sel):
    offsets = torch.full((capi.msa_num_segments(d) + 1,), -7, dtype=torch.int32, device="cuda")
    entries = torch.full((max(capi.msa_num_entries(d), 1),), -7, dtype=torch.int32, device="cuda")
    entry_pos = torch.full(tuple(sel.shape), -7, dtype=torch.int32, device="cuda")
    err = torch.zeros((4,), dtype=torch.int32, device="cuda")
    capi.msa_build_block_query_lists_noalloc(d, sel, offsets, entries, entry_pos, err)
    torch.cuda.synchronize()
    assert int(err[0]) == 0
    return offsets, entries, entry_pos


@pytest.mark.parametrize("w", [
    wl.small("ragged_r4", 1, 2500, 2500, 0, 8, 2, 128, seed=31),
    wl.small("chunk_unaligned", 2, 1600, 2600, 1000, 4, 2, 64, seed=32),
    wl.small("decode_like", 16, 1, 40000, 39999, 64, 8, 128, seed=33),
    wl.small("windows_of_256", 1, 2000, 2000, 0, 16, 2, 128, seed=34, q_window=256),
], ids=lambda w: w.name)
def test_noalloc_lists_match_the_workspace_version_twice(w):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    msa_build.build()
    d = pipeline.dims_for(w)
    assert capi.msa_block_query_lists_workspace(d) <= (32 << 20)
    # two different selections, one call each, in a row
    for offset in (11, 12):
        sel = wl.random_selection(w, "cpu", seed_offset=offset).cuda()
        want = _lists_with_workspace(d, sel)
        got = _lists_without_workspace(d, sel)
        for g_, w_ in zip(got, want):
            assert torch.equal(g_, w_)


def test_noalloc_refuses_problems_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    msa_build.build()
    d = pipeline.dims_for(wl.P128)                 # 128K prefill: ~34 MB of scratch
    assert capi.msa_block_query_lists_workspace(d) > (32 << 20)
    dummy = torch.zeros((16,), dtype=torch.int32, device="cuda")
    with pytest.raises(capi.MSAError) as ei:
        capi.msa_build_block_query_lists_noalloc(d, dummy, dummy, dummy, dummy)
    assert ei.value.status == 6                    # MSA_ERR_SCRATCH_LIMIT
