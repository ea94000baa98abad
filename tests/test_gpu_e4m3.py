"""8-bit (e4m3) index branch on the GPU against the oracle.

Quantisation (per-tensor amax / 448, nearest code, ties to even, saturation)
must give the oracle's codes and scale bit for bit.  The pooled scores come
from exact e4m3 x e4m3 products summed in fp32, so they are held to the
bf16 path's bound: |gpu - oracle| <= 1e-5 * s_q s_k max_j sum_k |q_k k_jk|.
The selection on them must match the oracle's selection on its own pooled
scores bit for bit, near-ties (< 1e-5 relative) counted as in the bf16 path.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_32_b200 import pipeline, workloads as wl

from _helpers import compare_pooled, compare_sets

pytestmark = pytest.mark.gpu

CASES = [
    wl.small("e4m3_r4", 1, 2500, 2500, 0, 8, 2, 128, seed=61, plants_per_group=3,
             plant_targets=128),
    wl.small("e4m3_batch2_hk2", 2, 700, 3100, 2400, 8, 2, 128, seed=62, h_kidx=2),
    wl.small("e4m3_decode", 3, 1, 4000, 3999, 32, 4, 128, seed=63),
]


def _tolerance(qv, kv, pos, bat, h_kidx, s):
    """1e-5 * s * max over each block's keys of sum_k |q_k k_jk| (decoded codes)."""
    n, G, _ = qv.shape
    n_kv = kv.shape[2]
    nblk = (n_kv + 127) // 128
    pad = nblk * 128 - n_kv
    out = np.zeros((n, G, nblk))
    for r in range(n):
        for g in range(G):
            kk = np.abs(kv[bat[r], 0 if h_kidx == 1 else g])
            v = np.concatenate([kk @ np.abs(qv[r, g]), np.zeros(pad)])
            out[r, g] = v.reshape(nblk, 128).max(axis=1)
    return 1e-5 * s * out


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_e4m3_codes_pooled_and_selection(w):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    d = pipeline.dims_for(w)
    buf = pipeline.Buffers.allocate(d)
    inp = wl.make_inputs(w, "cuda", with_qkv=False)
    buf.pooled.fill_(float("nan"))
    q8, k8, sq, sk = pipeline.select_e4m3(buf, inp["q_idx"], inp["k_idx"])
    torch.cuda.synchronize()
    assert int(buf.dev_err[0]) == 0
    # codes and scales, bit for bit
    qb, kb = oracle.bf16_bits(inp["q_idx"]), oracle.bf16_bits(inp["k_idx"])
    oq, osq = oracle.quantize_e4m3(qb)
    ok, osk = oracle.quantize_e4m3(kb)
    assert float(sq[0]) == osq and float(sk[0]) == osk
    np.testing.assert_array_equal(q8.cpu().numpy(), oq)
    np.testing.assert_array_equal(k8.cpu().numpy(), ok)
    # pooled scores from the oracle's codes
    rows = np.arange(w.n_q, dtype=np.int64)
    pos = np.tile(w.q_pos0 + rows, w.batch)
    bat = np.repeat(np.arange(w.batch, dtype=np.int64), w.n_q)
    q_rows = oq.reshape(-1, w.h_kv, w.d_idx)
    ora = oracle.index_pooled_e4m3(q_rows, pos, bat, ok, osq, osk, out_stride=buf.pooled_stride)
    gpu = buf.pooled.permute(0, 2, 1, 3).reshape(-1, w.h_kv, buf.pooled_stride).cpu().numpy()
    dec = np.vectorize(oracle.e4m3_value)
    lut = dec(np.arange(256)).astype(np.float64)
    lut[np.isnan(lut)] = 0.0
    tol = _tolerance(lut[q_rows], lut[ok], pos, bat, w.h_kidx, osq * osk)
    assert compare_pooled(gpu, ora[:, :, :tol.shape[2]], tol, pos) <= 1.0
    # selection on the 8-bit scores
    ora_sel = oracle.topk(ora, pos)
    gpu_sel = buf.sel.permute(0, 2, 1, 3).reshape(-1, w.h_kv, 16).cpu().numpy()
    bad, ties, bad_cert, _ = compare_sets(gpu_sel, ora_sel, ora, pos)
    assert bad == 0 and bad_cert == 0, (bad, ties, bad_cert)


def test_e4m3_full_size_rows():
    """The 128K prefill's index branch (8 groups, d_idx 128): every code and both
    scales bit for bit, pooled scores and selections of sampled rows against the
    oracle."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    w = wl.P128
    d = pipeline.dims_for(w)
    buf = pipeline.Buffers.allocate(d)
    inp = wl.make_inputs(w, "cuda", with_qkv=False)
    q8, k8, sq, sk = pipeline.select_e4m3(buf, inp["q_idx"], inp["k_idx"])
    torch.cuda.synchronize()
    assert int(buf.dev_err[0]) == 0
    qb, kb = oracle.bf16_bits(inp["q_idx"]), oracle.bf16_bits(inp["k_idx"])
    oq, osq = oracle.quantize_e4m3(qb)
    ok, osk = oracle.quantize_e4m3(kb)
    assert float(sq[0]) == osq and float(sk[0]) == osk
    np.testing.assert_array_equal(q8.cpu().numpy(), oq)
    np.testing.assert_array_equal(k8.cpu().numpy(), ok)
    rows = np.array([1000, 70000, w.n_q - 1], np.int64)
    pos = w.q_pos0 + rows
    bat = np.zeros_like(rows)
    q_rows = oq[0, rows]
    ora = oracle.index_pooled_e4m3(q_rows, pos, bat, ok, osq, osk, out_stride=buf.pooled_stride)
    gpu = buf.pooled[0, :, torch.from_numpy(rows).cuda()].permute(1, 0, 2).cpu().numpy()
    dec = np.vectorize(oracle.e4m3_value)
    lut = dec(np.arange(256)).astype(np.float64)
    lut[np.isnan(lut)] = 0.0
    tol = _tolerance(lut[q_rows], lut[ok], pos, bat, w.h_kidx, osq * osk)
    assert compare_pooled(gpu, ora[:, :, :tol.shape[2]], tol, pos) <= 1.0
    ora_sel = oracle.topk(ora, pos)
    gpu_sel = buf.sel[0, :, torch.from_numpy(rows).cuda()].permute(1, 0, 2).cpu().numpy()
    bad, ties, bad_cert, _ = compare_sets(gpu_sel, ora_sel, ora, pos)
    assert bad == 0 and bad_cert == 0, (bad, ties, bad_cert)
