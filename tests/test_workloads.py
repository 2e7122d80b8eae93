"""Host-side checks of the seeded workload generators (no GPU)."""
import numpy as np

from kv_cache_decode_index_b200 import workloads as W


def test_workloads_shapes_and_determinism():
    wl = W.scaled(W.WORKLOADS["group_1m_b4"], ctx=20000, needles=16)
    q1, w1 = W.index_query(wl, 0)
    q2, w2 = W.index_query(wl, 0)
    assert q1.shape == (4, 32, 128) and w1.shape == (4, 32)
    assert np.array_equal(q1, q2) and np.array_equal(w1, w2)
    assert not np.array_equal(q1, W.index_query(wl, 1)[0])
    assert (w1 >= 0).all() and (w1 < 1).all()
    k = W.request_rows(wl, 1, which="ik")
    assert k.shape == (20000, 128) and k.dtype == np.float32
    # any row regenerates on its own
    pos = np.array([0, 4095, 4096, 19999])
    assert np.array_equal(W.rows_at(wl, 1, pos, "ik"), k[pos])
    kv = W.request_rows(wl, 1, which="kv")
    assert np.array_equal(W.rows_at(wl, 1, pos, "kv"), kv[pos])


def test_needles_are_query_aligned():
    wl = W.scaled(W.WORKLOADS["group_1m_b4"], ctx=50000)
    pos = W.needle_positions(wl, 2)
    assert len(pos) == 64 and len(np.unique(pos)) == 64 and pos.max() < 50000
    u = W.needle_direction(wl, 2)
    k = W.request_rows(wl, 2, which="ik")
    proj = k.astype(np.float64) @ u
    mask = np.zeros(50000, bool)
    mask[pos] = True
    # projection along u: N(0,1) for ordinary keys, N(4,1) for needles
    assert abs(proj[~mask].mean()) < 0.05 and abs(proj[~mask].std() - 1) < 0.05
    assert abs(proj[mask].mean() - 4) < 0.5


def test_ragged_page_table():
    wl = W.WORKLOADS["ragged_b64"]
    n = W.ctx_lengths(wl)
    assert n.min() >= 4096 and n.max() <= 1048576 and len(n) == 64
    table, num_pages = W.page_layout(wl)
    used = table[table >= 0]
    assert len(used) == num_pages and len(np.unique(used)) == num_pages
    assert (used < num_pages).all()
    assert not np.array_equal(used, np.sort(used))          # shuffled
    for b in range(64):
        assert (table[b] >= 0).sum() == -(-n[b] // 4096)


def test_channel_scale_outliers():
    c = W.channel_scale(W.WORKLOADS["full_4k_b1"])
    assert c.shape == (512,) and (c > 0).all()
    assert (c > 8 * np.exp(-1.5)).sum() >= 5
