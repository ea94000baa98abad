"""Host-only checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/msa.h declares, sizes work out, and argument
validation rejects bad input before anything reaches the device."""
import ctypes
import os
import re

import pytest

from block_sparse_attention_32_b200 import build as msa_build
from block_sparse_attention_32_b200 import capi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    msa_build.build()
    return capi.lib()


def _declared():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"MSA_API\s+[\w\s\*]+?\b(msa_\w+)\s*\(", txt)
    return names


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n


def test_block_and_entry_counts(lib):
    d = capi.make_dims(1, 4096, 4096, 0, 4, 1, 64)
    assert capi.msa_num_blocks(d) == 32
    # queries t < 1920 keep own+1 blocks, later ones 16
    want = sum(min(16, t // 128 + 1) for t in range(4096))
    assert capi.msa_num_entries(d) == want
    d = capi.make_dims(64, 1, 262144, 262143, 64, 8, 128)
    assert capi.msa_num_blocks(d) == 2048
    assert capi.msa_num_entries(d) == 64 * 8 * 16
    d = capi.make_dims(1, 8192, 1056768, 1048576, 64, 8, 128)
    assert capi.msa_num_blocks(d) == 8256
    assert capi.msa_num_entries(d) == 8 * 8192 * 16
    d = capi.make_dims(1, 1000, 2600, 1000, 4, 2, 64)   # unaligned chunk start
    want = sum(min(16, t // 128 + 1) for t in range(1000, 2000)) * 2
    assert capi.msa_num_entries(d) == want


def test_workspace_size(lib):
    d = capi.make_dims(2, 300, 1000, 700, 8, 2, 64)
    nblk, ntiles = 8, 3
    nseg = 2 * 2 * nblk
    nchunks = (nseg + 4095) // 4096
    assert capi.msa_num_segments(d) == nseg
    assert capi.msa_block_query_lists_workspace(d) == 4 * (nseg * (ntiles + 1) + nchunks)
    # 3 query windows of 128: tile histograms + per-(window, block) totals
    d = capi.make_dims(2, 300, 1000, 700, 8, 2, 64, q_window=128)
    nseg = 2 * 2 * 3 * nblk
    assert capi.msa_num_segments(d) == nseg
    assert capi.msa_block_query_lists_workspace(d) == 4 * (2 * 2 * ntiles * nblk + nseg + 1)


def test_query_window(lib):
    """The default window follows the rule the header states (the same rule
    the oracle writes out); an explicit window must be a positive multiple of
    128."""
    import oracle
    for h_q, h_kv in ((64, 8), (32, 8), (32, 2), (8, 8), (4, 1)):
        d = capi.make_dims(1, 131072, 131072, 0, h_q, h_kv, 128)
        assert capi.msa_query_window(d) == oracle.query_window(h_q, h_kv)
    d = capi.make_dims(1, 131072, 131072, 0, 64, 8, 128)
    assert capi.msa_query_window(d) == 16384
    assert capi.msa_num_segments(d) == 8 * 8 * 1024
    assert capi.msa_query_window(capi.make_dims(1, 1000, 1000, 0, 8, 2, 64, q_window=256)) == 256
    t = capi.Tensor(0x100000, 0, 256, 128)
    for qw in (100, -128, 1):
        d = capi.make_dims(1, 1000, 4096, 0, 8, 2, 128, q_window=qw)
        assert capi.msa_query_window(d) == 0
        assert lib.msa_index_score_maxpool(ctypes.byref(d), t, t, ctypes.c_void_p(0x200000), 32,
                                           None, None) == 1


BAD_DIMS = [
    dict(batch=0), dict(n_q=0), dict(n_kv=0), dict(q_pos0=-1), dict(q_pos0=5000),
    dict(h_q=6), dict(h_kv=3), dict(h_kidx=3), dict(scale=0.0), dict(scale=float("nan")),
]


@pytest.mark.parametrize("bad", BAD_DIMS, ids=lambda b: ",".join(f"{k}={v}" for k, v in b.items()))
def test_invalid_dims_are_rejected(lib, bad):
    args = dict(batch=1, n_q=1000, n_kv=4096, q_pos0=0, h_q=8, h_kv=2, d_idx=128, h_kidx=1,
                scale=0.088)
    args.update(bad)
    d = capi.Dims(args["batch"], args["n_q"], args["n_kv"], args["q_pos0"], args["h_q"],
                  args["h_kv"], args["h_kidx"], args["d_idx"], args["scale"], 0)
    t = capi.Tensor(0x100000, 0, 256, 128)
    st = lib.msa_index_score_maxpool(ctypes.byref(d), t, t, ctypes.c_void_p(0x200000), 32, None,
                                     None)
    assert st in (1, 2)          # INVALID_ARG or UNSUPPORTED, nothing enqueued


def test_unsupported_sizes(lib):
    for d in (capi.make_dims(1, 100, 100, 0, 8, 2, 96),          # d_idx 96
              capi.make_dims(1, 100, 100, 0, 12, 4, 64),         # R = 3
              capi.make_dims(1, 100, 100, 0, 64, 2, 64)):        # R = 32
        t = capi.Tensor(0x100000, 0, 256, 128)
        assert lib.msa_index_score_maxpool(ctypes.byref(d), t, t, ctypes.c_void_p(0x200000),
                                           4, None, None) == 2


def test_pointer_and_stride_checks(lib):
    d = capi.make_dims(1, 1000, 4096, 0, 8, 2, 128)
    good = capi.Tensor(0x100000, 0, 256, 128)
    null = capi.Tensor(0, 0, 256, 128)
    mis = capi.Tensor(0x100008, 0, 256, 128)
    odd = capi.Tensor(0x100000, 0, 260, 128)
    P = ctypes.c_void_p
    f = lib.msa_index_score_maxpool
    assert f(ctypes.byref(d), null, good, P(0x200000), 32, None, None) == 1
    assert f(ctypes.byref(d), mis, good, P(0x200000), 32, None, None) == 3
    assert f(ctypes.byref(d), good, odd, P(0x200000), 32, None, None) == 3
    assert f(ctypes.byref(d), good, good, P(0x200004), 32, None, None) == 3
    assert f(ctypes.byref(d), good, good, P(0x200000), 30, None, None) == 1   # stride < nblk
    assert f(ctypes.byref(d), good, good, P(0x200000), 33, None, None) == 1   # not a multiple of 4
    assert f(None, good, good, P(0x200000), 32, None, None) == 1
    ws = capi.msa_block_query_lists_workspace(d)
    g = lib.msa_build_block_query_lists
    assert g(ctypes.byref(d), P(0x1000), P(0x2000), P(0x3000), P(0x5000), P(0x4000), ws - 4,
             None, None) == 4
    assert g(ctypes.byref(d), P(0x1000), None, P(0x3000), P(0x5000), P(0x4000), ws,
             None, None) == 1
    assert g(ctypes.byref(d), P(0x1000), P(0x2000), P(0x3000), None, P(0x4000), ws,
             None, None) == 1                                       # no entry_pos
    h = lib.msa_sparse_attn_fwd
    assert h(ctypes.byref(d), good, good, mis, P(0x1000), P(0x2000), P(0x3000), P(0x4000),
             None, None) == 3
    m = lib.msa_merge_partials
    assert m(ctypes.byref(d), P(0x1000), P(0x2000), P(0x3000), None, P(0x5000), None, None) == 1
    assert lib.msa_status_string(4) == b"MSA_ERR_WORKSPACE_TOO_SMALL"


def test_noalloc_builder_returns_the_workspace_builders_statuses(lib):
    """On rejected arguments the allocation-free list builder returns the same
    status as the workspace one (both stop before any CUDA call)."""
    P = ctypes.c_void_p
    ws_fn, na_fn = lib.msa_build_block_query_lists, lib.msa_build_block_query_lists_noalloc
    cases = [capi.make_dims(1, 100, 100, 0, 64, 2, 64),       # R = 32: unsupported
             capi.make_dims(1, 100, 100, 0, 8, 2, 96),        # d_idx 96: unsupported
             capi.make_dims(1, 100, 100, 0, 12, 4, 64),       # R = 3: unsupported
             capi.make_dims(0, 100, 100, 0, 8, 2, 64),        # batch 0: invalid
             capi.make_dims(1, 100, 100, 50, 8, 2, 64)]       # q_pos0 + n_q > n_kv: invalid
    for d in cases:
        want = ws_fn(ctypes.byref(d), P(0x1000), P(0x2000), P(0x3000), P(0x5000), P(0x4000),
                     1 << 30, None, None)
        got = na_fn(ctypes.byref(d), P(0x1000), P(0x2000), P(0x3000), P(0x5000), None, None)
        assert want in (1, 2) and got == want, (want, got)
    assert na_fn(None, P(0x1000), P(0x2000), P(0x3000), P(0x5000), None, None) == 1
    d = capi.make_dims(1, 1000, 4096, 0, 8, 2, 128)
    assert na_fn(ctypes.byref(d), P(0x1000), None, P(0x3000), P(0x5000), None, None) == 1
    assert na_fn(ctypes.byref(d), P(0x1000), P(0x2000), P(0x3000), None, None, None) == 1
    assert na_fn(ctypes.byref(d), P(0x1004), P(0x2000), P(0x3000), P(0x5000), None, None) == 3


def test_token_select_and_backward_validation(lib):
    """The token-level and backward entry points reject bad arguments on the
    host, before anything is enqueued."""
    P = ctypes.c_void_p
    d = capi.make_dims(1, 1000, 4096, 0, 8, 2, 128)
    good = capi.Tensor(0x100000, 0, 256, 128)
    mis = capi.Tensor(0x100008, 0, 256, 128)
    # workspace: one fp32 score row per (sampled row, group)
    assert capi.msa_token_select_workspace(d, 3) == 3 * 2 * 4096 * 4
    ws = capi.msa_token_select_workspace(d, 3)
    t = lib.msa_token_select_attention
    args = lambda budget, out, wsb, rows=P(0x1000): (ctypes.byref(d), good, good, good, good, good,
                                                     rows, 3, budget, P(0x2000), out, P(0x4000),
                                                     P(0x5000), wsb, None, None)
    assert t(*args(0, P(0x3000), ws)) == 1                 # budget < 1
    assert t(*args(2048, P(0x3000), ws - 4)) == 4          # workspace too small
    assert t(*args(2048, P(0x3004), ws)) == 3              # misaligned out
    assert t(*args(2048, P(0x3000), ws, rows=None)) == 1   # no rows
    d16 = capi.make_dims(1, 1000, 4096, 0, 32, 2, 128)    # R = 16: heads exceed the 8-wide tiles
    assert t(ctypes.byref(d16), good, good, good, good, good, P(0x1000), 3, 2048, P(0x2000),
             P(0x3000), P(0x4000), P(0x5000), capi.msa_token_select_workspace(d16, 3), None,
             None) == 2
    b = lib.msa_sparse_attn_bwd
    ptrs = [P(0x1000 * (i + 1)) for i in range(8)]      # lse, offsets, entries, delta, part, dq, dk, dv
    bad = list(ptrs)
    bad[5] = None
    assert b(ctypes.byref(d), good, good, good, good, good, *bad, None, None) == 1
    bad = list(ptrs)
    bad[6] = P(0x7008)
    assert b(ctypes.byref(d), good, good, good, good, good, *bad, None, None) == 3
    bad = list(ptrs)
    bad[6] = P(0x7010)                                   # dk 16- but not 32-byte aligned
    assert b(ctypes.byref(d), good, good, good, good, good, *bad, None, None) == 3
    bad = list(ptrs)
    bad[4] = P(0x5010)                                   # dq pieces likewise
    assert b(ctypes.byref(d), good, good, good, good, good, *bad, None, None) == 3
    assert b(ctypes.byref(d), good, good, good, mis, good, *ptrs, None, None) == 3
    assert b(None, good, good, good, good, good, *ptrs, None, None) == 1


def test_header_is_plain_c(tmp_path):
    """include/msa.h compiles as C99 on its own (no C++ or CUDA types in the ABI)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc") or shutil.which("cc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_msa.c"
    src.write_text('#include "msa.h"\nint main(void) { msa_dims d; (void)d; '
                   'return (int)msa_num_blocks((const msa_dims*)0) * 0; }\n')
    subprocess.check_call([gcc, "-std=c99", "-Wall", "-Werror", "-pedantic", "-fsyntax-only",
                           "-I", os.path.join(ROOT, "include"), str(src)])
