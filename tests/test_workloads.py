"""Host checks of the seeded input generators that both the CUDA path and the
oracle consume (no GPU): shapes, determinism, and the validity of the random
selections the attention and backward parity tests feed to both sides."""
import numpy as np
import torch

from block_sparse_attention_32_b200 import workloads as wl

SHAPES = [
    wl.small("prefill", 1, 1500, 1500, 0, 4, 1, 64, seed=1),
    wl.small("chunk_unaligned", 2, 333, 2222, 1889, 8, 2, 64, seed=2),
    wl.small("decode", 3, 1, 4000, 3999, 8, 4, 128, seed=3),
    wl.small("tiny_context", 1, 200, 200, 0, 4, 2, 64, seed=4),
]


def test_random_selection_is_valid():
    """Each (batch, group, query) row holds its own block, min(16, own + 1)
    distinct blocks in [0, own], ascending, then -1."""
    for w in SHAPES:
        sel = wl.random_selection(w).numpy()
        assert sel.shape == (w.batch, w.h_kv, w.n_q, 16) and sel.dtype == np.int32
        for i in range(w.n_q):
            own = (w.q_pos0 + i) // 128
            n = min(16, own + 1)
            rows = sel[:, :, i].reshape(-1, 16)
            assert (rows[:, n:] == -1).all()
            v = rows[:, :n]
            assert (v >= 0).all() and (v <= own).all()
            assert (np.diff(v, axis=1) > 0).all()
            assert (v == own).any(axis=1).all()


def test_random_selection_draws_uniformly_and_deterministically():
    w = wl.small("long", 1, 64, 64 * 128, 63 * 128, 8, 2, 64, seed=5)
    a = wl.random_selection(w).numpy()
    b = wl.random_selection(w).numpy()
    np.testing.assert_array_equal(a, b)
    # 62 candidates below the own block, 15 drawn per row: every candidate shows up
    counts = np.bincount(a[a >= 0].ravel(), minlength=w.nblk)
    assert (counts[:62] > 0).all()
    other = wl.random_selection(w, seed_offset=999).numpy()
    assert not np.array_equal(a, other)


def test_upstream_grad_and_inputs_are_seeded():
    w = SHAPES[1]
    g1, g2 = wl.upstream_grad(w), wl.upstream_grad(w)
    assert g1.shape == (w.batch, w.n_q, w.h_q, 128) and g1.dtype == torch.bfloat16
    assert torch.equal(g1, g2)
    x1, x2 = wl.make_inputs(w), wl.make_inputs(w)
    for k in ("q", "k", "v", "q_idx", "k_idx"):
        assert torch.equal(x1[k], x2[k]), k
    assert x1["k_idx"].shape == (w.batch, w.h_kidx, w.n_kv, w.d_idx)
