"""End-to-end parity of one CSA2 layer-group decode step (DecodeGroup through
the C ABI) against the float64 oracle: pool, every layer's Top-k, and the
attention outputs.  Needs a B200 and libcsa2.so."""
import numpy as np
import pytest
import torch

from kv_cache_decode_index_b200 import workloads as W
from oracle import csa2 as C
from tests import gpu_util as U

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def csa2():
    from kv_cache_decode_index_b200 import csa2 as lib
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return lib


def _queries(wl, dev):
    q_idx, w_idx, q_main = [], [], []
    for layer, m in enumerate(wl.modes):
        if m == "Ru":
            q_idx.append(None)
            w_idx.append(None)
        else:
            q, w = W.index_query(wl, layer)
            q_idx.append(q)
            w_idx.append(w)
        q_main.append(W.main_query(wl, layer))
    tq = [None if q is None else torch.from_numpy(q).to(dev) for q in q_idx]
    tw = [None if w is None else torch.from_numpy(w).to(dev) for w in w_idx]
    tm = [m.to(dev) for m in q_main]
    return q_idx, w_idx, q_main, tq, tw, tm


def _run_gpu(csa2, wl, cache, dev, append_rows=None):
    q_idx, w_idx, q_main, tq, tw, tm = _queries(wl, dev)
    group = csa2.DecodeGroup(cache, wl.modes, wl.heads, wl.topk, wl.pool_blocks, wl.scale)
    out = [torch.empty_like(m) for m in tm]
    if append_rows is not None:
        kv, ik, pos = append_rows
        csa2.append_kv(cache, kv, ik, pos)
    group.step(tq, tw, tm, out)
    torch.cuda.synchronize()
    return group, q_idx, w_idx, q_main, out


def _check_request(csa2, wl, cache, group, b, n, q_idx, w_idx, q_main, out, dev):
    """Full oracle of request b and comparison under the parity rules."""
    codes, exp = U.oracle_request(wl, b, n)
    ora = C.decode_group(wl.modes, [None if q is None else q[b] for q in q_idx],
                         [None if w is None else w[b] for w in w_idx], codes, exp, n, wl.pool_blocks, wl.topk)
    s64 = ora["scores"]
    excused = lambda t: False
    if wl.pool_blocks:
        gp = group.pool[b].cpu().numpy()
        U.assert_sorted_padded(gp, f"pool b={b}")
        bm64 = ora["blockmax"]
        diff = U.assert_set_parity(gp, ora["pool"], lambda j: bm64[j], U.threshold(bm64, wl.pool_blocks),
                                   what=f"pool b={b}")
        pool_diff = set(gp[gp >= 0].tolist()) ^ set(ora["pool"][ora["pool"] >= 0].tolist())
        excused = lambda t: (t // 8) in pool_diff
        gpu_pool_pos = set(C.pool_positions(gp, n).tolist())
    layer_scores = {}
    for layer, m in enumerate(wl.modes):
        gt = group.topk[layer][b].cpu().numpy()
        U.assert_sorted_padded(gt, f"topk layer {layer} b={b}")
        if m == "Ru":
            np.testing.assert_array_equal(gt, group.topk[layer - 1][b].cpu().numpy())
            layer_scores[layer] = layer_scores[layer - 1]
            continue
        if wl.pool_blocks:
            assert set(gt[gt >= 0].tolist()) <= gpu_pool_pos, f"layer {layer} selects outside the pool"
        if m == "F":
            sc = s64
        else:
            sc = C.indexer_scores(q_idx[layer][b], w_idx[layer][b], codes, exp)
        layer_scores[layer] = sc
        ot = ora["topk"][layer]
        cand = np.arange(n) if not wl.pool_blocks else C.pool_positions(ora["pool"], n)
        U.assert_set_parity(gt, ot, lambda t: sc[t], U.threshold(sc[cand], wl.topk), excused,
                            what=f"topk layer {layer} ({m}) b={b}")
    # attention: GPU kernel fed the oracle's indices vs the oracle
    sel = np.unique(np.concatenate([t[t >= 0] for t in ora["topk"]]))
    kvc, kvs = U.oracle_kv_rows(wl, b, sel)
    full_c = np.zeros((n, 256), np.uint8)
    full_s = np.zeros((n, 32), np.uint8)
    full_c[sel], full_s[sel] = kvc, kvs
    worst = 0.0
    for layer in range(len(wl.modes)):
        ot = ora["topk"][layer].astype(np.int32)
        ref = C.sparse_attention(q_main[layer][b].float().numpy(), full_c, full_s, ot, wl.scale)
        # as many queries as the group's launch (all of them request b's): the
        # number of queries per launch decides the key split, and with it the
        # rounding of the merge
        nq = wl.batch
        qi = torch.full((nq,), b, dtype=torch.int32, device=dev)
        g = csa2.sparse_attn(cache, torch.from_numpy(np.repeat(ot[None], nq, axis=0)).to(dev),
                             q_main[layer][b:b + 1].repeat(nq, 1, 1).to(dev), wl.scale,
                             q_req=qi).float().cpu().numpy()[0]
        worst = max(worst, U.assert_attention_close(g, ref, f"attention layer {layer} b={b}"))
        if np.array_equal(group.topk[layer][b].cpu().numpy(), ot):
            np.testing.assert_array_equal(out[layer][b].float().cpu().numpy(), g)
    return ora, worst


def test_group_full_4k_b1(csa2):
    wl = W.WORKLOADS["full_4k_b1"]
    cache = U.build_cache(wl, csa2)
    dev = cache.device
    group, q_idx, w_idx, q_main, out = _run_gpu(csa2, wl, cache, dev)
    _, worst = _check_request(csa2, wl, cache, group, 0, 4096, q_idx, w_idx, q_main, out, dev)
    print(f"max attention rel err {worst:.2e}")
    assert csa2.get_error(cache)[0] == csa2.OK


def test_group_64k_b8(csa2):
    wl = W.WORKLOADS["group_64k_b8"]
    cache = U.build_cache(wl, csa2)
    dev = cache.device
    group, q_idx, w_idx, q_main, out = _run_gpu(csa2, wl, cache, dev)
    for b in range(wl.batch):
        _check_request(csa2, wl, cache, group, b, 65536, q_idx, w_idx, q_main, out, dev)
    assert csa2.get_error(cache)[0] == csa2.OK


def test_group_ragged_paged_with_append(csa2):
    """Ragged contexts behind a shuffled page table; one FP4 append per request
    precedes the step (1 Full + 4 Reindex + 1 Reuse)."""
    wl = W.scaled(W.WORKLOADS["ragged_b64"], batch=12, ctx_range=(4096, 300000))
    n = W.ctx_lengths(wl)
    cache = U.build_cache(wl, csa2, append_last=True)
    dev = cache.device
    last = n - 1
    kv = np.stack([W.rows_at(wl, b, [last[b]], "kv")[0] for b in range(wl.batch)])
    ik = np.stack([W.rows_at(wl, b, [last[b]], "ik")[0] for b in range(wl.batch)])
    rows = (torch.from_numpy(kv).to(dev), torch.from_numpy(ik).to(dev),
            torch.from_numpy(last.astype(np.int32)).to(dev))
    group, q_idx, w_idx, q_main, out = _run_gpu(csa2, wl, cache, dev, append_rows=rows)
    from oracle import formats as F
    ikc, ike = F.quantize_indexer(ik)
    for b in range(wl.batch):
        row = int(cache.rows_of(b, [last[b]])[0])
        np.testing.assert_array_equal(cache.ik_codes[row].cpu().numpy(), ikc[b])
        assert int(cache.ik_exp[row]) == int(ike[b])
        _check_request(csa2, wl, cache, group, b, int(n[b]), q_idx, w_idx, q_main, out, dev)
    assert csa2.get_error(cache)[0] == csa2.OK


def test_group_1m_b4_full_size(csa2):
    """The 1M-context workload at full size, in the bench's launch
    configuration: every request against the full oracle (pool, every layer's
    Top-k, attention), the pool also against the exact top blocks of the GPU's
    own block maxima, and the planted needles' pool recall and score margin
    reported per request."""
    wl = W.WORKLOADS["group_1m_b4"]
    cache = U.build_cache(wl, csa2)
    dev = cache.device
    group, q_idx, w_idx, q_main, out = _run_gpu(csa2, wl, cache, dev)
    n = wl.ctx
    bm_all = group.blockmax.cpu().numpy()
    for b in range(wl.batch):
        ora, worst = _check_request(csa2, wl, cache, group, b, n, q_idx, w_idx, q_main, out, dev)
        gp = group.pool[b].cpu().numpy()
        bm = bm_all[b, :n // 8].astype(np.float64)
        order = np.lexsort((np.arange(len(bm)), -bm))
        np.testing.assert_array_equal(gp, np.sort(order[:2048]), err_msg=f"pool b={b}")
        needles = W.needle_positions(wl, b)
        s64 = ora["scores"]
        sd = s64.std()
        theta = np.sort(ora["blockmax"])[::-1][wl.pool_blocks - 1]   # the pool's threshold block max
        z = (s64[needles] - s64.mean()) / sd
        margin = (s64[needles] - theta) / sd
        ora_recall = int(np.isin(needles // 8, ora["pool"]).sum())
        gpu_recall = int(np.isin(needles // 8, gp).sum())
        print(f"request {b}: needle pool recall oracle {ora_recall}/64, gpu {gpu_recall}/64; needle score "
              f"z = {np.median(z):.2f} median ({z.min():.2f} min) standard deviations above the mean score; "
              f"{np.median(margin):+.2f} median sd from the pool threshold; attention rel err {worst:.2e}")
        assert ora_recall == gpu_recall
    assert csa2.get_error(cache)[0] == csa2.OK


def test_group_ragged_b64_full_size(csa2):
    """The 64-request ragged workload at full size (log-uniform contexts from
    4,096 to 1,048,576 positions behind a shuffled page table, one append per
    request, 1 Full + 4 Reindex + 1 Reuse): every appended row bit-exact; the
    two shortest requests against the full oracle; every request on sampled
    block maxima and on properties that hold at any size."""
    wl = W.WORKLOADS["ragged_b64"]
    n = W.ctx_lengths(wl)
    cache = U.build_cache(wl, csa2, append_last=True)
    dev = cache.device
    last = n - 1
    kv = np.stack([W.rows_at(wl, b, [last[b]], "kv")[0] for b in range(wl.batch)])
    ik = np.stack([W.rows_at(wl, b, [last[b]], "ik")[0] for b in range(wl.batch)])
    rows = (torch.from_numpy(kv).to(dev), torch.from_numpy(ik).to(dev),
            torch.from_numpy(last.astype(np.int32)).to(dev))
    group, q_idx, w_idx, q_main, out = _run_gpu(csa2, wl, cache, dev, append_rows=rows)
    assert csa2.get_error(cache)[0] == csa2.OK
    from oracle import formats as F
    ikc, ike = F.quantize_indexer(ik)
    kvc, kvs = F.quantize_main_kv(kv)
    for b in range(wl.batch):
        row = int(cache.rows_of(b, [last[b]])[0])
        np.testing.assert_array_equal(cache.ik_codes[row].cpu().numpy(), ikc[b])
        assert int(cache.ik_exp[row]) == int(ike[b])
        np.testing.assert_array_equal(cache.kv_codes[row].cpu().numpy(), kvc[b])
        np.testing.assert_array_equal(cache.kv_scales[row].cpu().numpy(), kvs[b])
    for b in np.argsort(n)[:2]:
        _check_request(csa2, wl, cache, group, int(b), int(n[b]), q_idx, w_idx, q_main, out, dev)
    rng = np.random.default_rng(1)
    bm_all = group.blockmax.cpu().numpy()
    pools = group.pool.cpu().numpy()
    for b in range(wl.batch):
        nb = -(-int(n[b]) // 8)
        bm = bm_all[b, :nb].astype(np.float64)
        gp = pools[b]
        order = np.lexsort((np.arange(nb), -bm))
        want = np.full(wl.pool_blocks, -1, np.int64)
        want[:min(nb, wl.pool_blocks)] = np.sort(order[:wl.pool_blocks])
        np.testing.assert_array_equal(gp, want, err_msg=f"pool b={b}: not the top blocks of the GPU's maxima")
        blocks = rng.choice(nb, min(nb, 64), replace=False)
        pos = (blocks[:, None] * 8 + np.arange(8)).reshape(-1)
        keep = pos < n[b]
        codes, exp = F.quantize_indexer(W.rows_at(wl, b, pos[keep], "ik"))
        s64 = np.full(len(pos), -np.inf)
        s64[keep] = C.indexer_scores(q_idx[0][b], w_idx[0][b], codes, exp)
        bm64 = s64.reshape(-1, 8).max(axis=1)
        assert np.all(np.abs(bm[blocks] - bm64) <= 1e-5 * np.abs(bm64)), f"block maxima b={b}"
        pool_pos = set(C.pool_positions(gp, int(n[b])).tolist())
        for layer, m in enumerate(wl.modes):
            t = group.topk[layer][b].cpu().numpy()
            U.assert_sorted_padded(t, f"topk layer {layer} b={b}")
            assert (t >= 0).sum() == min(wl.topk, int(n[b])) and set(t[t >= 0].tolist()) <= pool_pos
            if m == "Ru":
                np.testing.assert_array_equal(t, group.topk[layer - 1][b].cpu().numpy())


def test_group_graph_replay_matches_eager(csa2):
    """The bench times CUDA-graph replays of the step (programmatic dependent
    launch inside the graph); a replay must give the eager step's indices and
    outputs exactly, twice in a row."""
    wl = W.WORKLOADS["group_64k_b8"]
    cache = U.build_cache(wl, csa2)
    dev = cache.device
    group, q_idx, w_idx, q_main, out = _run_gpu(csa2, wl, cache, dev)
    ref_topk = [t.clone() for t in group.topk]
    ref_pool = group.pool.clone()
    ref_out = [o.clone() for o in out]
    _, _, _, tq, tw, tm = _queries(wl, dev)
    g_out = [torch.empty_like(m) for m in tm]
    group.step(tq, tw, tm, g_out)   # warm-up outside capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        group.step(tq, tw, tm, g_out)
    for _ in range(2):
        for t in g_out:
            t.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(group.pool, ref_pool)
        for layer in range(len(wl.modes)):
            assert torch.equal(group.topk[layer], ref_topk[layer]), f"topk layer {layer}"
            assert torch.equal(g_out[layer], ref_out[layer]), f"attention layer {layer}"
    del graph
    assert csa2.get_error(cache)[0] == csa2.OK
