"""The C-ABI library loads, exports every symbol include/csa2.h declares, and
rejects bad arguments on the host before touching a GPU (no device needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "csa2.h")


@pytest.fixture(scope="module")
def lib():
    from kv_cache_decode_index_b200 import build
    build.build()
    from kv_cache_decode_index_b200 import csa2
    return csa2


def declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"CSA2_API\s+[\w\s\*]+?\b(csa2_\w+)\s*\(", text)


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert len(names) == 24, names
    so = ctypes.CDLL(lib.LIB_PATH)
    for n in names:
        assert hasattr(so, n), f"{n} missing from libcsa2.so"


def _cache(lib, **over):
    buf = (ctypes.c_uint8 * 4096)()
    base = (ctypes.addressof(buf) + 255) & ~255
    f = dict(kv_codes=base, kv_scales=base, ik_codes=base, ik_exp=base, page_table=base, ctx_len=base,
             num_pages=4, page_size=128, max_pages_per_req=2, batch=2, err_word=base)
    f.update(over)
    c = lib.CacheStruct(**f)
    c._keep = buf
    return c, base


def test_host_side_validation(lib):
    L = lib._lib
    c, p = _cache(lib)
    P = ctypes.c_void_p(p)
    assert L.csa2_index_full(None, P, P, P, None, None, None) == lib.ERR_ARG
    bad, _ = _cache(lib, batch=0)
    assert L.csa2_index_full(ctypes.byref(bad), P, P, P, None, None, None) == lib.ERR_SHAPE
    bad, _ = _cache(lib, page_size=100)
    assert L.csa2_pool_select(ctypes.byref(bad), P, None, 2048, P, None) == lib.ERR_SHAPE
    bad, _ = _cache(lib, ik_codes=p + 4)
    assert L.csa2_index_full(ctypes.byref(bad), P, P, P, None, None, None) == lib.ERR_ARG
    assert b"16-byte" in L.csa2_last_error_message()
    assert L.csa2_pool_select(ctypes.byref(c), P, None, 0, P, None) == lib.ERR_SHAPE
    assert L.csa2_pool_select(ctypes.byref(c), P, ctypes.c_void_p(p + 4), 2048, P, None) == lib.ERR_ARG
    assert L.csa2_index_full(ctypes.byref(c), P, P, P, None, ctypes.c_void_p(p + 4), None) == lib.ERR_ARG
    # multi-layer Top-k over a pool: layer count, k, pointers and workspace are checked on the host
    rw = L.csa2_reindex_layers_workspace_bytes
    assert rw(2, 3, 2048) == 2 * 3 * (2048 * 8 + 4096) * 4 and rw(0, 3, 2048) == 0
    rl = L.csa2_reindex_layers
    pa = (ctypes.c_void_p * 3)(p, p, p)
    rneed = rw(2, 3, 2048)
    assert rl(ctypes.byref(c), 9, P, 2048, pa, pa, 512, pa, P, rneed, None) == lib.ERR_SHAPE
    assert rl(ctypes.byref(c), 3, P, 2048, pa, pa, 0, pa, P, rneed, None) == lib.ERR_SHAPE
    assert rl(ctypes.byref(c), 3, None, 2048, pa, pa, 512, pa, P, rneed, None) == lib.ERR_ARG
    assert rl(ctypes.byref(c), 3, P, 2048, pa, pa, 512, pa, P, rneed - 4, None) == lib.ERR_SHAPE
    assert b"csa2_reindex_layers_workspace_bytes" in L.csa2_last_error_message()
    assert rl(ctypes.byref(c), 3, P, 2048, pa, pa, 512, pa, None, rneed, None) == lib.ERR_ARG
    pz = (ctypes.c_void_p * 3)(p, None, p)
    assert rl(ctypes.byref(c), 3, P, 2048, pa, pz, 512, pa, P, rneed, None) == lib.ERR_ARG
    assert L.csa2_reindex(ctypes.byref(c), lib.REINDEX, P, 2048, P, P, None, None, 0, P, None) == lib.ERR_SHAPE
    assert L.csa2_reindex(ctypes.byref(c), 7, P, 2048, P, P, None, None, 512, P, None) == lib.ERR_ARG
    assert L.csa2_reindex(ctypes.byref(c), lib.REUSE, None, 0, None, None, None, None, 512, P, None) == lib.ERR_ARG
    assert L.csa2_sparse_attn(ctypes.byref(c), 2, None, P, 512, P, 48, ctypes.c_float(0.1), P, None) == lib.ERR_SHAPE
    assert L.csa2_sparse_attn(ctypes.byref(c), 3, None, P, 512, P, 64, ctypes.c_float(0.1), P, None) == lib.ERR_SHAPE
    assert L.csa2_append_kv(ctypes.byref(c), -1, P, P, None, P, None) == lib.ERR_SHAPE
    assert L.csa2_append_kv(ctypes.byref(c), 0, P, P, None, P, None) == lib.OK   # nothing to do
    big, _ = _cache(lib, max_pages_per_req=2048, page_size=4096)
    assert L.csa2_reindex(ctypes.byref(big), lib.FULL, None, 0, P, P, None, None, 512, P, None) == lib.ERR_SHAPE
    assert L.csa2_status_string(lib.ERR_TIMEOUT) == b"a pipeline wait on the device gave up"
    # prefill: req, k, ratio, workspace size and alignment are checked on the host
    need = L.csa2_prefill_workspace_bytes(8)
    assert need == 8 * 4096 * 8 + 32 and L.csa2_prefill_workspace_bytes(0) == 0
    pf = L.csa2_prefill_index
    assert pf(ctypes.byref(c), 2, 8, P, 2, P, P, 512, P, P, need, None) == lib.ERR_SHAPE      # req >= batch
    assert pf(ctypes.byref(c), 0, 8, P, 2, P, P, 1025, P, P, need, None) == lib.ERR_SHAPE     # k > 1024
    assert pf(ctypes.byref(c), 0, 8, P, 0, P, P, 512, P, P, need, None) == lib.ERR_SHAPE      # ratio < 1
    assert pf(ctypes.byref(c), 0, 8, P, 2, P, P, 512, P, P, need - 16, None) == lib.ERR_SHAPE
    assert b"needed" in L.csa2_last_error_message()
    assert pf(ctypes.byref(c), 0, 8, P, 2, P, P, 512, P, ctypes.c_void_p(p + 8), need, None) == lib.ERR_ARG
    assert pf(ctypes.byref(c), 0, 8, None, 2, P, P, 512, P, P, need, None) == lib.ERR_ARG
    assert pf(ctypes.byref(c), 0, 0, None, 2, None, None, 512, None, None, 0, None) == lib.OK   # nothing to do
    ca = L.csa2_compress_append
    assert ca(ctypes.byref(c), 4, 3, P, P, None, P, None) == lib.ERR_SHAPE      # m not a power of two <= 8
    assert ca(ctypes.byref(c), -1, 2, P, P, None, P, None) == lib.ERR_SHAPE
    assert ca(ctypes.byref(c), 4, 2, None, P, None, P, None) == lib.ERR_ARG
    assert ca(ctypes.byref(c), 0, 2, None, None, None, None, None) == lib.OK
    # multi-layer attention: the optional exchange workspace is checked on the host
    aw = L.csa2_attn_workspace_bytes
    assert aw(2, 3, 64) == 2 * 3 * 4 * (64 * 512 + 2 * 64) * 4 and aw(-1, 3, 64) == 0
    al = L.csa2_sparse_attn_layers
    qa = (ctypes.c_void_p * 2)(p, p)
    wneed = aw(2, 2, 64)
    assert al(ctypes.byref(c), 2, 2, None, qa, 512, qa, 64, ctypes.c_float(0.1), qa, P, wneed - 4, None) == lib.ERR_SHAPE
    assert b"csa2_attn_workspace_bytes" in L.csa2_last_error_message()
    assert al(ctypes.byref(c), 2, 2, None, qa, 512, qa, 64, ctypes.c_float(0.1), qa, ctypes.c_void_p(p + 4), wneed,
              None) == lib.ERR_ARG
    assert al(ctypes.byref(c), 9, 2, None, qa, 512, qa, 64, ctypes.c_float(0.1), qa, None, 0, None) == lib.ERR_SHAPE
    tz = (ctypes.c_void_p * 2)(p, None)
    assert al(ctypes.byref(c), 2, 2, None, tz, 512, qa, 64, ctypes.c_float(0.1), qa, None, 0, None) == lib.ERR_ARG
    # sharded pool: shard count, sizes and pointers are checked on the host
    pm = L.csa2_pool_merge
    assert pm(0, 2, 2048, P, P, P, None) == lib.ERR_SHAPE
    assert pm(17, 2, 2048, P, P, P, None) == lib.ERR_SHAPE
    assert pm(16, 2, 4096, P, P, P, None) == lib.ERR_SHAPE        # more than 32768 candidates
    assert pm(2, 2, 2048, None, P, P, None) == lib.ERR_ARG
    pc = L.csa2_pool_candidates
    assert pc(ctypes.byref(c), P, P, 0, 0, P, P, None) == lib.ERR_SHAPE
    assert pc(ctypes.byref(c), P, P, 2048, -1, P, P, None) == lib.ERR_SHAPE
    assert pc(ctypes.byref(c), P, None, 2048, 0, P, P, None) == lib.ERR_ARG
    ps = L.csa2_prefill_index_static
    assert ps(ctypes.byref(c), 0, 257, P, 2, P, P, 512, P, None) == lib.ERR_SHAPE   # above the static limit
    assert b"static scratch" in L.csa2_last_error_message()
    assert ps(ctypes.byref(c), 0, 8, P, 2, P, P, 1025, P, None) == lib.ERR_SHAPE
    assert ps(ctypes.byref(c), 0, 0, None, 2, None, None, 512, None, None) == lib.OK


def test_binding_rejects_wrong_tensors(lib):
    import torch
    c = lib.Cache.__new__(lib.Cache)
    with pytest.raises(ValueError):
        lib._need(torch.zeros(3, dtype=torch.float32), torch.int32, (3,), "x")
