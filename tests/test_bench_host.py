"""Host-side logic of bench.py, on CPU: algorithmic bytes, I/O bytes, clock
parsing, per-rank workloads, the max-over-ranks reduction across 2 gloo ranks,
the reference arm's JSON line on a small workload, and the keying of the
reported DRAM traffic to the scan's source."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from kv_cache_decode_index_b200 import workloads as W


def test_alg_bytes_of_the_1m_group():
    step, scan = bench.alg_bytes(W.WORKLOADS["group_1m_b4"])
    assert scan == 4 * 1048576 * 129                        # 541.1 MB of indexer K
    reindex = 2 * 4 * 16384 * 129                            # two Reindex layers over the pool
    kv = 6 * 4 * 512 * 288                                   # six layers gather Top-512 FP4 rows
    pool = 4 * 2048 * 4 * 3                                  # pool read by 3 selecting layers
    assert step == scan + reindex + kv + pool
    assert abs(step / 1e6 - 561.6) < 0.1


def test_alg_bytes_short_context_and_no_pool():
    step, scan = bench.alg_bytes(W.WORKLOADS["full_4k_b1"])
    assert scan == 4096 * 129 and step == scan + 512 * 288


def test_io_bytes():
    h2d, d2h = bench.io_bytes(W.WORKLOADS["group_1m_b4"])
    assert h2d == 3 * 4 * (32 * 128 * 4 + 32 * 4) + 6 * 4 * 64 * 512 * 2
    assert d2h == 6 * 4 * 64 * 512 * 2


def test_clock_parsing():
    text = ("0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n"
            "0, 1800, 1965, 998.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n"
            "0, 1900, 1965, 990.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n")
    c = bench.parse_clock_samples(text)
    assert c == {"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}


def test_rank_workloads_differ_only_in_data():
    wl = W.WORKLOADS["group_1m_b4"]
    w1 = bench.rank_workload(wl, 1)
    assert bench.rank_workload(wl, 0) is wl
    assert (w1.batch, w1.ctx, w1.modes) == (wl.batch, wl.ctx, wl.modes) and w1.seed != wl.seed
    assert not np.array_equal(W.index_query(w1, 0)[0], W.index_query(wl, 0)[0])


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        t = [3.5, 7.25][rank]
        out[rank] = bench.max_over_ranks(t, torch.device("cpu"), world)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(2, _free_port(), out), nprocs=2, start_method="spawn", join=True)
        assert dict(out) == {0: 7.25, 1: 7.25}


def test_reference_arm_json_small(monkeypatch):
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.main(["--impl", "reference", "--workload", "full_4k_b1", "--steps", "2", "--warmup", "3"])
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "queries/s"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["cpu_baseline"]["cores"] >= 1
    assert line["timed_steps"] == 2


def test_reference_arm_is_time_boxed(monkeypatch):
    """Past the time box the reference arm stops after the query in progress,
    so a large --steps still ends within minutes; the line says how many
    steps it timed."""
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setattr(bench, "REFERENCE_TIME_BOX_S", 0)
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.main(["--impl", "reference", "--workload", "full_4k_b1", "--steps", "500", "--warmup", "20"])
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert line["timed_steps"] == 1 and line["steps"] == 500 and line["value"] > 0
    assert "1 of the 500 steps" in line["cpu_baseline"]["sample"]


def test_reference_arm_other_ranks_do_nothing(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.main(["--impl", "reference", "--workload", "full_4k_b1", "--steps", "2", "--warmup", "3"])
    assert buf.getvalue() == ""


def test_prefill_flops_closed_form():
    # queries at tokens 516096 + j (j < 8192) see 258048 + floor((j + 1) / 2)
    # m=2 entries: sum = 8192 * 258048 + 4096 * 4096
    import bench
    wl = W.WORKLOADS["prefill_256k_q8192"]
    assert bench.prefill_flops(wl) == 2 * 32 * 128 * (8192 * 258048 + 4096 * 4096)


def _shard_rank_main(rank, world, port, out):
    """Rank g holds slice g of two requests' block maxima; the candidates are
    exchanged with the product's all-gather and merged with the oracle."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import numpy as np
        from kv_cache_decode_index_b200 import sharded
        from oracle import csa2 as C
        rng = np.random.default_rng(5)
        nb, P = 5000, 512
        bm = np.round(rng.standard_normal((2, nb)) * 4) / 4          # ties across the slices
        cut = [0, 2100, nb]
        v = np.zeros((2, P), np.float32)
        i = np.zeros((2, P), np.int32)
        for b in range(2):
            vb, ib = C.slice_candidates(bm[b, cut[rank]:cut[rank + 1]], cut[rank], P)
            v[b], i[b] = vb, ib
        all_v, all_i = sharded.exchange_candidates(torch.from_numpy(v), torch.from_numpy(i))
        assert tuple(all_v.shape) == (world, 2, P) and tuple(all_i.shape) == (world, 2, P)
        merged = [C.pool_merge(all_v[:, b].numpy(), all_i[:, b].numpy(), P) for b in range(2)]
        whole = [C.pool_select(bm[b].astype(np.float32).astype(np.float64), P) for b in range(2)]
        out[rank] = all(np.array_equal(m, w) for m, w in zip(merged, whole)) and \
            bool((all_i[rank].numpy() == i).all())
    finally:
        dist.destroy_process_group()


def test_sharded_pool_exchange_gloo_two_ranks():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_shard_rank_main, args=(2, _free_port(), out), nprocs=2, start_method="spawn", join=True)
        assert dict(out) == {0: True, 1: True}


def test_slice_pages_cover_the_table():
    from kv_cache_decode_index_b200 import sharded
    for pages, g in [(256, 2), (256, 8), (10, 3), (7, 7), (5, 1)]:
        s = sharded.slice_pages(pages, g)
        assert len(s) == g and s[0][0] == 0 and sum(n for _, n in s) == pages
        assert all(s[k][0] + s[k][1] == s[k + 1][0] for k in range(g - 1))
        assert max(n for _, n in s) - min(n for _, n in s) <= 1


def test_fp4_oracle_sample_runs_small():
    from kv_cache_decode_index_b200 import workloads as W
    wl = W.scaled(W.WORKLOADS["group_1m_b4"], ctx=8192, pool_blocks=64, needles=0)
    assert bench.oracle_sample_fp4(wl, 0) > 0
    step, scan = bench.alg_bytes(wl, ik_row_bytes=bench.IK4_ROW_BYTES)
    assert scan == 72 * 8192 * wl.batch


def _fake_tree(root, fp4):
    """A copy of the scan's source files under `root` (for the source hash)."""
    src = os.path.join(os.path.dirname(bench.__file__), "kv_cache_decode_index_b200", "csrc")
    dst = os.path.join(root, "kv_cache_decode_index_b200", "csrc")
    os.makedirs(dst, exist_ok=True)
    names = ("k_index_fp4.cu", "fp4.cuh") if fp4 else ("k_index.cu", "index_common.cuh")
    for name in names + ("scan_units.cuh", "common.cuh"):
        with open(os.path.join(src, name), "rb") as f, open(os.path.join(dst, name), "wb") as g:
            g.write(f.read())
    os.makedirs(os.path.join(root, "profiles"), exist_ok=True)


def test_scan_traffic_is_keyed_to_the_kernel_source(monkeypatch, tmp_path):
    """The reported DRAM traffic comes from the committed ncu summary only
    while the scan's sources hash to the value it was captured on, and only
    for its workload: any edit of those sources (a comment too) drops it."""
    for fp4 in (False, True):
        root = str(tmp_path / ("fp4" if fp4 else "fp8"))
        _fake_tree(root, fp4)
        monkeypatch.setattr(bench, "ROOT", root)
        name = "index_full_fp4_traffic.txt" if fp4 else "index_full_traffic.txt"
        path = os.path.join(root, "profiles", name)
        with open(path, "w") as f:
            f.write(f"kernel_source_hash: {bench.scan_kernel_hash(fp4)}\nworkload: group_1m_b4\n"
                    "dram_bytes_per_launch: 123456\n")
        assert bench.scan_traffic_per_launch("group_1m_b4", fp4) == 123456.0
        assert bench.scan_traffic_per_launch("group_64k_b8", fp4) is None
        src = os.path.join(root, "kv_cache_decode_index_b200", "csrc", "scan_units.cuh")
        with open(src, "a") as f:
            f.write("// edited\n")
        assert bench.scan_traffic_per_launch("group_1m_b4", fp4) is None
        os.remove(path)
        assert bench.scan_traffic_per_launch("group_1m_b4", fp4) is None
