"""Backward of the sparse attention on the GPU against the oracle.

The gradients a model trained through MSA needs ("MSA 稀疏注意力三国杀" page,
section "MSA 能力不掉：3T token 对照实验"; the selection is a fixed input, section
"索引分支训练：KL 对齐").  The selection fed to both sides is a seeded random
valid one (own block + up to 15 earlier blocks), so the comparison does not
hinge on index-score near-ties; the GPU's backward uses the GPU forward's
bf16 output and fp32 lse, the oracle its own fp64 forward.

Bars (bf16 operands; each output element sums >= 128 products, each carrying
one bf16-rounded factor -- P for dV, dS for dK and dQ, and o inside D -- that
is, <= 2^-9 relative per term, accumulated in fp32):
  * max-abs error <= 2e-2 x max |oracle| of the tensor;
  * mean-abs error <= 5e-3 x mean |oracle| of the tensor.
At the full 128K prefill size (the real selection), sampled rows' dq against
the oracle with the same bars, and two identities that hold at any size:
sum_j dk_j = 0 (each row's dS sums to zero) and sum_j dv_j = sum of dO over
the group's heads and queries (each row's weights sum to one), per (batch,
group), within 1e-3 of the sum of magnitudes.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_32_b200 import capi, pipeline, workloads as wl
from _helpers import bits, compare_sets

pytestmark = pytest.mark.gpu

MAX_REL = 2e-2
MEAN_REL = 5e-3

CASES = [
    wl.small("bwd_tiny_r4", 1, 1500, 1500, 0, 4, 1, 64, seed=71),
    wl.small("bwd_r8_batch2_chunk", 2, 700, 3100, 2400, 16, 2, 128, seed=72),
    wl.small("bwd_r1", 1, 1800, 1800, 0, 4, 4, 64, seed=73),
    wl.small("bwd_r16_chunk", 1, 600, 2600, 2000, 32, 2, 64, seed=74),
    wl.small("bwd_r2_decode", 3, 1, 4000, 3999, 8, 4, 128, seed=75),
    wl.small("bwd_r4_ragged", 1, 333, 2222, 1889, 8, 2, 64, seed=76),
    # block->query lists in query windows of 256: a block's gradient gathers
    # from several windows' segments
    wl.small("bwd_r8_windows", 1, 1700, 1700, 0, 16, 2, 128, seed=77, q_window=256),
    # 2 x 2 x 80 = 320 (batch, group, block) items, more than there are SMs: the
    # items are dealt largest first (the work order the call sorts on the device)
    wl.small("bwd_r8_sorted_items", 2, 600, 10240, 9640, 16, 2, 128, seed=78),
]


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _check(name, gpu, ref):
    err = np.abs(gpu.astype(np.float64) - ref)
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= MAX_REL * np.abs(ref).max(), (name, mx, np.abs(ref).max())
    assert mean <= MEAN_REL * np.abs(ref).mean(), (name, mean, np.abs(ref).mean())


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_backward_matches_oracle(w):
    _need_gpu()
    d = pipeline.dims_for(w)
    buf = pipeline.Buffers.allocate(d)
    grads = pipeline.Grads.allocate(d)
    inp = wl.make_inputs(w, "cuda")
    sel = wl.random_selection(w, "cuda")
    d_out = wl.upstream_grad(w, "cuda")
    pipeline.attend(buf, inp["q"], inp["k"], inp["v"], sel=sel)
    dq, dk, dv = pipeline.backward(buf, grads, inp["q"], inp["k"], inp["v"], d_out)
    torch.cuda.synchronize()
    assert int(buf.dev_err[0]) == 0
    e_dq, e_dk, e_dv, _, e_delta = oracle.attention_bwd(
        bits(inp["q"]), bits(inp["k"]), bits(inp["v"]), bits(d_out), sel.cpu().numpy(), w.scale,
        w.q_pos0)
    _check("dq", dq.cpu().numpy(), e_dq)
    _check("dk", dk.cpu().numpy(), e_dk)
    _check("dv", dv.cpu().numpy(), e_dv)
    _check("delta", grads.delta.cpu().numpy(), e_delta)


@pytest.mark.parametrize("wi", [1, 6, 7], ids=["chunk_after_cache", "query_windows",
                                               "sorted_items"])
def test_backward_deterministic_and_unselected_blocks_zero(wi):
    """dq is summed in slot order and every KV block's dk, dv come from the one
    CTA that owns the block: two runs give identical bits for all three, also
    when a block's queries span several query windows; the keys of a cache
    block that no query selected get exactly zero dk and dv."""
    _need_gpu()
    w = CASES[wi]              # a chunk after cached tokens / windows of 256 / 320 items
    d = pipeline.dims_for(w)
    buf = pipeline.Buffers.allocate(d)
    inp = wl.make_inputs(w, "cuda")
    s_np = wl.random_selection(w, "cpu").numpy()
    drop3 = w.q_pos0 >= 4 * 128          # block 3 is nobody's own block
    if drop3:
        # a full selection in which cache block 3 never appears: where a row
        # holds it, the lowest block the row lacks takes its place
        for b, g, i in zip(*np.nonzero((s_np == 3).any(axis=-1))):
            row = set(int(c) for c in s_np[b, g, i] if c >= 0)
            spare = next(c for c in range(4, (w.q_pos0 + i) // 128) if c not in row)
            row.discard(3)
            row.add(spare)
            s_np[b, g, i] = sorted(row)
        assert not (s_np == 3).any()
    sel = torch.from_numpy(s_np).cuda()
    d_out = wl.upstream_grad(w, "cuda")
    res = []
    for _ in range(2):
        grads = pipeline.Grads.allocate(d)
        pipeline.attend(buf, inp["q"], inp["k"], inp["v"], sel=sel)
        dq, dk, dv = pipeline.backward(buf, grads, inp["q"], inp["k"], inp["v"], d_out)
        res.append((dq.clone(), dk.clone(), dv.clone()))
    torch.cuda.synchronize()
    assert int(buf.dev_err[0]) == 0
    for x, y in zip(res[0], res[1]):
        assert torch.equal(x, y)
    if drop3:
        assert not res[0][1][:, :, 3 * 128:4 * 128].any()
        assert not res[0][2][:, :, 3 * 128:4 * 128].any()
    e_dq, e_dk, e_dv, _, _ = oracle.attention_bwd(
        bits(inp["q"]), bits(inp["k"]), bits(inp["v"]), bits(d_out), sel.cpu().numpy(), w.scale,
        w.q_pos0)
    _check("dq", res[0][0].cpu().numpy(), e_dq)
    _check("dk", res[0][1].cpu().numpy(), e_dk)
    _check("dv", res[0][2].cpu().numpy(), e_dv)


def test_backward_rejects_bad_arguments():
    _need_gpu()
    w = CASES[0]
    d = pipeline.dims_for(w)
    buf = pipeline.Buffers.allocate(d)
    grads = pipeline.Grads.allocate(d)
    inp = wl.make_inputs(w, "cuda")
    d_out = wl.upstream_grad(w, "cuda")
    bad = torch.empty(grads.dq.numel() + 1, dtype=torch.float32, device="cuda")[1:]
    with pytest.raises(capi.MSAError):                       # misaligned dq
        capi.msa_sparse_attn_bwd(d, inp["q"], inp["k"], inp["v"], buf.out, d_out, buf.lse,
                                 buf.blk_offsets, buf.entries, grads.delta, buf.part_acc, bad,
                                 grads.dk, grads.dv)


def test_backward_full_size_rows_and_identities():
    """The 128K prefill (64 heads, 8 groups) with the real selection: dq of
    sampled rows against the oracle (rows whose selection matches the
    oracle's), and the two sum identities over all keys."""
    _need_gpu()
    w = wl.P128
    d = pipeline.dims_for(w)
    buf = pipeline.Buffers.allocate(d)
    grads = pipeline.Grads.allocate(d)
    inp = wl.make_inputs(w, "cuda")
    d_out = wl.upstream_grad(w, "cuda")
    pipeline.forward(buf, inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"])
    dq, dk, dv = pipeline.backward(buf, grads, inp["q"], inp["k"], inp["v"], d_out)
    torch.cuda.synchronize()
    assert int(buf.dev_err[0]) == 0
    # identities, per (batch, group), in float64 on the device
    R = w.h_q // w.h_kv
    sk = dk.double().sum(dim=2)                                   # [B, G, 128]
    ak = dk.double().abs().sum(dim=2)
    assert float((sk.abs() / ak.clamp_min(1e-30)).max()) <= 1e-3
    sdv = dv.double().sum(dim=2)
    sdo = d_out.double().view(w.batch, w.n_q, w.h_kv, R, 128).sum(dim=(1, 3))
    ado = d_out.double().abs().view(w.batch, w.n_q, w.h_kv, R, 128).sum(dim=(1, 3))
    assert float(((sdv - sdo).abs() / ado).max()) <= 1e-3
    # sampled rows: the oracle's own selection, then each row as a one-query problem
    rows = np.array([3, 40000, 99999, w.n_q - 1], np.int64)
    pos = w.q_pos0 + rows
    b = np.zeros_like(rows)
    kb, vb, kib = bits(inp["k"]), bits(inp["v"]), bits(inp["k_idx"])
    q_rows = bits(inp["q"])[0, rows]
    qi_rows = bits(inp["q_idx"])[0, rows]
    do_rows = bits(d_out)[0, rows]
    g_dq = dq[0, torch.from_numpy(rows).cuda()].cpu().numpy()
    gpu_sel = buf.sel[0, :, torch.from_numpy(rows).cuda()].permute(1, 0, 2).cpu().numpy()
    del inp, buf, grads
    torch.cuda.empty_cache()
    pooled = oracle.index_pooled(qi_rows, pos, b, kib)
    sel = oracle.topk(pooled, pos)
    bad, ties, bad_tie, eval_sel = compare_sets(gpu_sel, sel, pooled, pos)
    assert bad == 0 and bad_tie == 0, (bad, ties, bad_tie)
    kf, vf = oracle.bits_to_f64(kb), oracle.bits_to_f64(vb)
    for r in range(len(rows)):
        e_dq, _, _, _, _ = oracle.attention_bwd(
            q_rows[r][None, None], kf, vf, do_rows[r][None, None],
            eval_sel[r][None, :, None, :].astype(np.int32), w.scale, int(pos[r]))
        _check(f"dq row {rows[r]}", g_dq[r], e_dq[0, 0])


def test_backward_reports_short_selection():
    """A selection with fewer entries than the sizes imply (a query keeping 15
    of its 16 blocks) is reported by the backward on the device flag
    (MSA_DEVERR_BAD_ENTRY), after which the call returns."""
    _need_gpu()
    w = CASES[5]                                  # 333 queries after 1889 cached tokens
    d = pipeline.dims_for(w)
    buf = pipeline.Buffers.allocate(d)
    grads = pipeline.Grads.allocate(d)
    inp = wl.make_inputs(w, "cuda")
    s_np = wl.random_selection(w, "cpu").numpy()
    keep = s_np[0, 0, 300][s_np[0, 0, 300] >= 0][1:]      # query 300 of group 0 drops one block
    s_np[0, 0, 300] = np.concatenate([keep, np.full(16 - len(keep), -1)])
    sel = torch.from_numpy(s_np).cuda()
    d_out = wl.upstream_grad(w, "cuda")
    pipeline.attend(buf, inp["q"], inp["k"], inp["v"], sel=sel)
    torch.cuda.synchronize()
    buf.dev_err.zero_()
    pipeline.backward(buf, grads, inp["q"], inp["k"], inp["v"], d_out)
    torch.cuda.synchronize()
    assert int(buf.dev_err[0]) == 3                          # MSA_DEVERR_BAD_ENTRY
