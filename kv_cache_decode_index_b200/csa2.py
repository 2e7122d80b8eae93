"""ctypes binding of libcsa2.so (include/csa2.h).

Argument marshalling only: every step of the decode path runs in the library's
CUDA kernels.  PyTorch supplies device memory and the current stream.  There is
no fallback: importing this module raises if the library has not been built,
and every call raises ``Csa2Error`` when the library reports a failure.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa2.so")
if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m kv_cache_decode_index_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)

FULL, REINDEX, REUSE = 0, 1, 2
MODE = {"F": FULL, "Ri": REINDEX, "Ru": REUSE}
OK, ERR_ARG, ERR_SHAPE, ERR_CUDA, ERR_DEVICE_BOUNDS, ERR_TIMEOUT, ERR_UNSUPPORTED = range(7)
BLOCK, INDEX_HEADS, INDEX_DIM, KV_DIM, KV_CODE_BYTES, KV_SCALE_BYTES = 8, 32, 128, 512, 256, 32
PREFILL_MAX_K, PREFILL_CANDIDATES, PREFILL_STATIC_MAX_QUERIES = 1024, 4096, 256
POOL_HIST_BINS, RESCORE_HIST_BINS, MAX_SCORE_LAYERS = 4096, 4096, 8
IK4_CODE_BYTES, IK4_TILE_SCALE_BYTES, MAX_FP4_SCORE_LAYERS = 64, 1024, 4


class CacheStruct(ctypes.Structure):
    _fields_ = [("kv_codes", ctypes.c_void_p), ("kv_scales", ctypes.c_void_p), ("ik_codes", ctypes.c_void_p),
                ("ik_exp", ctypes.c_void_p), ("page_table", ctypes.c_void_p), ("ctx_len", ctypes.c_void_p),
                ("num_pages", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("max_pages_per_req", ctypes.c_int32), ("batch", ctypes.c_int32), ("err_word", ctypes.c_void_p)]


class Ik4Struct(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


_P = ctypes.c_void_p
_I = ctypes.c_int32
_CP = ctypes.POINTER(CacheStruct)
_KP = ctypes.POINTER(Ik4Struct)
_sig = {
    "csa2_append_kv": [_CP, _I, _P, _P, _P, _P, _P],
    "csa2_compress_append": [_CP, _I, _I, _P, _P, _P, _P, _P],
    "csa2_index_full": [_CP, _P, _P, _P, _P, _P, _P],
    "csa2_pool_select": [_CP, _P, _P, _I, _P, _P],
    "csa2_reindex": [_CP, _I, _P, _I, _P, _P, _P, _P, _I, _P, _P],
    "csa2_reindex_layers": [_CP, _I, _P, _I, _P, _P, _I, _P, _P, ctypes.c_size_t, _P],
    "csa2_pool_candidates": [_CP, _P, _P, _I, _I, _P, _P, _P],
    "csa2_append_ik4": [_CP, _KP, _I, _P, _P, _P, _P],
    "csa2_index_full_fp4": [_CP, _KP, _P, _P, _P, _P, _P, _P],
    "csa2_reindex_layers_fp4": [_CP, _KP, _I, _P, _I, _P, _P, _I, _P, _P, ctypes.c_size_t, _P],
    "csa2_pool_merge": [_I, _I, _I, _P, _P, _P, _P],
    "csa2_sparse_attn": [_CP, _I, _P, _P, _I, _P, _I, ctypes.c_float, _P, _P],
    "csa2_sparse_attn_layers": [_CP, _I, _I, _P, _P, _I, _P, _I, ctypes.c_float, _P, _P, ctypes.c_size_t, _P],
    "csa2_swa_append": [_CP, _I, _P, _P, _I, _P, _P, _P, _P],
    "csa2_sparse_attn_swa": [_CP, _I, _P, _P, _I, _P, _P, _I, _P, _P, _I, ctypes.c_float, _P, _P],
    "csa2_prefill_index": [_CP, _I, _I, _P, _I, _P, _P, _I, _P, _P, ctypes.c_size_t, _P],
    "csa2_prefill_index_static": [_CP, _I, _I, _P, _I, _P, _P, _I, _P, _P],
    "csa2_get_error": [_CP, ctypes.POINTER(ctypes.c_int32), _P],
}
for _name, _args in _sig.items():
    getattr(_lib, _name).argtypes = _args
    getattr(_lib, _name).restype = ctypes.c_int
_lib.csa2_status_string.argtypes = [ctypes.c_int]
_lib.csa2_status_string.restype = ctypes.c_char_p
_lib.csa2_last_error_message.argtypes = []
_lib.csa2_last_error_message.restype = ctypes.c_char_p
_lib.csa2_prefill_workspace_bytes.argtypes = [_I]
_lib.csa2_prefill_workspace_bytes.restype = ctypes.c_size_t
_lib.csa2_attn_workspace_bytes.argtypes = [_I, _I, _I]
_lib.csa2_attn_workspace_bytes.restype = ctypes.c_size_t
_lib.csa2_reindex_layers_workspace_bytes.argtypes = [_I, _I, _I]
_lib.csa2_reindex_layers_workspace_bytes.restype = ctypes.c_size_t
_lib.csa2_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
_lib.csa2_set_wait_limit_ns.restype = None


class Csa2Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.csa2_last_error_message().decode()
        super().__init__(f"{where}: {_lib.csa2_status_string(status).decode()} ({status}): {msg}")


def _check(status: int, where: str):
    if status != OK:
        raise Csa2Error(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(dev):
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _need(t, dtype, shape, name):
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous() or t.device.type != "cuda":
        raise ValueError(f"{name}: expected contiguous cuda {dtype} {tuple(shape)}, "
                         f"got {t.device} {t.dtype} {tuple(t.shape)}")


def set_wait_limit_ns(ns: int):
    """Bound of every pipeline wait in the tensor-core kernels (default 2 s)."""
    _lib.csa2_set_wait_limit_ns(int(ns))


class Cache:
    """The paged cache of one layer group (device memory owned by torch).

    Rows: num_pages * page_size; request b's position t lives in row
    page_table[b, t // page_size] * page_size + t % page_size.
    """

    def __init__(self, num_pages: int, page_size: int, page_table, ctx_len, device="cuda"):
        self.device = torch.device(device)
        rows = num_pages * page_size
        self.num_pages, self.page_size = int(num_pages), int(page_size)
        self.kv_codes = torch.zeros(rows, KV_CODE_BYTES, dtype=torch.uint8, device=self.device)
        self.kv_scales = torch.zeros(rows, KV_SCALE_BYTES, dtype=torch.uint8, device=self.device)
        self.ik_codes = torch.zeros(rows, INDEX_DIM, dtype=torch.uint8, device=self.device)
        self.ik_exp = torch.zeros(rows, dtype=torch.uint8, device=self.device)
        self.page_table = torch.as_tensor(page_table, dtype=torch.int32).to(self.device).contiguous()
        self.ctx_len = torch.as_tensor(ctx_len, dtype=torch.int32).to(self.device).contiguous()
        self.batch, self.max_pages_per_req = self.page_table.shape
        self.err_word = torch.zeros(4, dtype=torch.int32, device=self.device)
        self._struct = None

    @property
    def capacity(self) -> int:
        return self.max_pages_per_req * self.page_size

    @property
    def struct(self) -> CacheStruct:
        s = CacheStruct(self.kv_codes.data_ptr(), self.kv_scales.data_ptr(), self.ik_codes.data_ptr(),
                        self.ik_exp.data_ptr(), self.page_table.data_ptr(), self.ctx_len.data_ptr(),
                        self.num_pages, self.page_size, self.max_pages_per_req, self.batch,
                        self.err_word.data_ptr())
        self._struct = s   # keep alive while a call is in flight
        return s

    def rows_of(self, b: int, positions):
        """Cache row numbers of request b's positions (host helper for tests)."""
        pt = self.page_table[b].cpu()
        positions = torch.as_tensor(positions, dtype=torch.int64)
        return pt[positions // self.page_size].to(torch.int64) * self.page_size + positions % self.page_size


class Ik4:
    """FP4 indexer keys of a cache (same rows and page table as `cache`):
    codes uint8 [rows, 64] (element 2i in the low nibble of byte i) and the
    block scales uint8 [rows / 128, 1024] of every 128-row tile in the
    tensor-core order (ik4_scale_offset)."""

    def __init__(self, cache: Cache):
        rows = cache.num_pages * cache.page_size
        self.codes = torch.zeros(rows, IK4_CODE_BYTES, dtype=torch.uint8, device=cache.device)
        self.scales = torch.zeros(rows // 128, IK4_TILE_SCALE_BYTES, dtype=torch.uint8, device=cache.device)
        self._struct = None

    @property
    def struct(self) -> Ik4Struct:
        s = Ik4Struct(self.codes.data_ptr(), self.scales.data_ptr())
        self._struct = s
        return s


def ik4_scale_offset(m, g):
    """Byte of the scale of tile row m (0..127), element group g (0..7) inside
    a tile's 1 KB scale block (host helper)."""
    return (g // 4) * 512 + (m % 32) * 16 + (m // 32) * 4 + g % 4


def append_ik4(cache: Cache, ik4: Ik4, ik_new, pos, req=None):
    """Quantise indexer keys ik_new float32 [n, 128] to the FP4 indexer format."""
    n = ik_new.shape[0]
    _need(ik_new, torch.float32, (n, INDEX_DIM), "ik_new")
    _need(pos, torch.int32, (n,), "pos")
    if req is not None:
        _need(req, torch.int32, (n,), "req")
    _check(_lib.csa2_append_ik4(ctypes.byref(cache.struct), ctypes.byref(ik4.struct), n, _ptr(ik_new), _ptr(req),
                                _ptr(pos), _stream(cache.device)), "csa2_append_ik4")


def index_full_fp4(cache: Cache, ik4: Ik4, q, w, blockmax=None, scores=None, hist=None):
    """Full scan over the FP4 indexer keys (as index_full)."""
    B = cache.batch
    _need(q, torch.float32, (B, INDEX_HEADS, INDEX_DIM), "q")
    _need(w, torch.float32, (B, INDEX_HEADS), "w")
    if blockmax is None:
        blockmax = torch.empty(B, cache.capacity // BLOCK, dtype=torch.float32, device=cache.device)
    _need(blockmax, torch.float32, (B, cache.capacity // BLOCK), "blockmax")
    if scores is not None:
        _need(scores, torch.float32, (B, cache.capacity), "scores")
    if hist is not None:
        _need(hist, torch.int32, (B, POOL_HIST_BINS), "hist")
    _check(_lib.csa2_index_full_fp4(ctypes.byref(cache.struct), ctypes.byref(ik4.struct), _ptr(q), _ptr(w),
                                    _ptr(blockmax), _ptr(scores), _ptr(hist), _stream(cache.device)),
           "csa2_index_full_fp4")
    return blockmax


def append_kv(cache: Cache, kv_new, ik_new, pos, req=None):
    n = kv_new.shape[0]
    _need(kv_new, torch.float32, (n, KV_DIM), "kv_new")
    _need(ik_new, torch.float32, (n, INDEX_DIM), "ik_new")
    _need(pos, torch.int32, (n,), "pos")
    if req is not None:
        _need(req, torch.int32, (n,), "req")
    _check(_lib.csa2_append_kv(ctypes.byref(cache.struct), n, _ptr(kv_new), _ptr(ik_new), _ptr(req), _ptr(pos),
                               _stream(cache.device)), "csa2_append_kv")


def compress_append(cache: Cache, kv_tok, ik_tok, pos, m: int = 2, req=None):
    """Sequence compressor + quantise-on-append: entry i = mean of token rows
    m*i .. m*i+m-1 of kv_tok [n*m,512] / ik_tok [n*m,128], stored at pos[i]."""
    n = pos.shape[0]
    _need(kv_tok, torch.float32, (n * m, KV_DIM), "kv_tok")
    _need(ik_tok, torch.float32, (n * m, INDEX_DIM), "ik_tok")
    _need(pos, torch.int32, (n,), "pos")
    if req is not None:
        _need(req, torch.int32, (n,), "req")
    _check(_lib.csa2_compress_append(ctypes.byref(cache.struct), n, int(m), _ptr(kv_tok), _ptr(ik_tok), _ptr(req),
                                     _ptr(pos), _stream(cache.device)), "csa2_compress_append")


def pool_hist(cache: Cache):
    """A zeroed block-max histogram buffer (uint32 bit patterns in an int32
    tensor [batch, POOL_HIST_BINS]) for index_full / pool_select."""
    return torch.zeros(cache.batch, POOL_HIST_BINS, dtype=torch.int32, device=cache.device)


def index_full(cache: Cache, q, w, blockmax=None, scores=None, hist=None):
    """Full scan: returns blockmax float32 [batch, capacity/8] (and fills scores
    if given; adds the block maxima's histogram into hist if given)."""
    B = cache.batch
    _need(q, torch.float32, (B, INDEX_HEADS, INDEX_DIM), "q")
    _need(w, torch.float32, (B, INDEX_HEADS), "w")
    if blockmax is None:
        blockmax = torch.empty(B, cache.capacity // BLOCK, dtype=torch.float32, device=cache.device)
    _need(blockmax, torch.float32, (B, cache.capacity // BLOCK), "blockmax")
    if scores is not None:
        _need(scores, torch.float32, (B, cache.capacity), "scores")
    if hist is not None:
        _need(hist, torch.int32, (B, POOL_HIST_BINS), "hist")
    _check(_lib.csa2_index_full(ctypes.byref(cache.struct), _ptr(q), _ptr(w), _ptr(blockmax), _ptr(scores),
                                _ptr(hist), _stream(cache.device)), "csa2_index_full")
    return blockmax


def pool_select(cache: Cache, blockmax, pool_blocks: int = 2048, pool=None, hist=None):
    """The pool (int32 [batch, pool_blocks]); hist: the scan's block-max
    histogram (read, then zeroed), or None."""
    B = cache.batch
    _need(blockmax, torch.float32, (B, cache.capacity // BLOCK), "blockmax")
    if pool is None:
        pool = torch.empty(B, pool_blocks, dtype=torch.int32, device=cache.device)
    _need(pool, torch.int32, (B, pool_blocks), "pool")
    if hist is not None:
        _need(hist, torch.int32, (B, POOL_HIST_BINS), "hist")
    _check(_lib.csa2_pool_select(ctypes.byref(cache.struct), _ptr(blockmax), _ptr(hist), pool_blocks, _ptr(pool),
                                 _stream(cache.device)), "csa2_pool_select")
    return pool


def reindex_layers_workspace_bytes(batch: int, n_layers: int, pool_blocks: int) -> int:
    return int(_lib.csa2_reindex_layers_workspace_bytes(int(batch), int(n_layers), int(pool_blocks)))


def reindex_layers(cache: Cache, pool, q_layers, w_layers, k: int = 512, topk_layers=None, workspace=None,
                   ik4: Ik4 | None = None):
    """Top-k over the pool of several Full / Reindex layers in one pass
    (csa2_reindex_layers, or csa2_reindex_layers_fp4 over the FP4 indexer keys
    `ik4`); returns the list of int32 [batch, k] Top-k.
    workspace: a zeroed uint8 device tensor of reindex_layers_workspace_bytes
    bytes, kept between calls (allocated and zeroed here when None)."""
    B, P = pool.shape
    L = len(q_layers)
    _need(pool, torch.int32, (B, P), "pool")
    for i, (q, w) in enumerate(zip(q_layers, w_layers)):
        _need(q, torch.float32, (B, INDEX_HEADS, INDEX_DIM), f"q_layers[{i}]")
        _need(w, torch.float32, (B, INDEX_HEADS), f"w_layers[{i}]")
    if topk_layers is None:
        topk_layers = [torch.empty(B, k, dtype=torch.int32, device=cache.device) for _ in range(L)]
    for i, t in enumerate(topk_layers):
        _need(t, torch.int32, (B, k), f"topk_layers[{i}]")
    need = reindex_layers_workspace_bytes(B, L, P)
    if workspace is None:
        workspace = torch.zeros(need, dtype=torch.uint8, device=cache.device)
    if workspace.dtype != torch.uint8 or not workspace.is_contiguous() or workspace.device.type != "cuda":
        raise ValueError("workspace: expected a contiguous cuda uint8 tensor")
    qa = (ctypes.c_void_p * L)(*[q.data_ptr() for q in q_layers])
    wa = (ctypes.c_void_p * L)(*[w.data_ptr() for w in w_layers])
    ta = (ctypes.c_void_p * L)(*[t.data_ptr() for t in topk_layers])
    if ik4 is None:
        _check(_lib.csa2_reindex_layers(ctypes.byref(cache.struct), L, _ptr(pool), P, qa, wa, int(k), ta,
                                        _ptr(workspace), workspace.numel(), _stream(cache.device)),
               "csa2_reindex_layers")
    else:
        _check(_lib.csa2_reindex_layers_fp4(ctypes.byref(cache.struct), ctypes.byref(ik4.struct), L, _ptr(pool), P,
                                            qa, wa, int(k), ta, _ptr(workspace), workspace.numel(),
                                            _stream(cache.device)), "csa2_reindex_layers_fp4")
    return topk_layers


def reindex(cache: Cache, mode: int, k: int = 512, pool=None, q=None, w=None, full_scores=None,
            prev_topk=None, topk=None):
    """Top-k of one layer (mode FULL / REINDEX / REUSE); returns topk int32 [batch, k]."""
    B = cache.batch
    P = 0
    if pool is not None:
        P = pool.shape[1]
        _need(pool, torch.int32, (B, P), "pool")
    if q is not None:
        _need(q, torch.float32, (B, INDEX_HEADS, INDEX_DIM), "q")
        _need(w, torch.float32, (B, INDEX_HEADS), "w")
    if full_scores is not None:
        _need(full_scores, torch.float32, (B, cache.capacity), "full_scores")
    if prev_topk is not None:
        _need(prev_topk, torch.int32, (B, k), "prev_topk")
    if topk is None:
        topk = torch.empty(B, k, dtype=torch.int32, device=cache.device)
    _need(topk, torch.int32, (B, k), "topk")
    _check(_lib.csa2_reindex(ctypes.byref(cache.struct), mode, _ptr(pool), P, _ptr(q), _ptr(w), _ptr(full_scores),
                             _ptr(prev_topk), k, _ptr(topk), _stream(cache.device)), "csa2_reindex")
    return topk


def sparse_attn(cache: Cache, topk, q, scale: float | None = None, out=None, q_req=None):
    """Sparse attention; q bf16 [n, H, 512] -> out bf16 [n, H, 512]."""
    n, k = topk.shape
    H = q.shape[1]
    _need(topk, torch.int32, (n, k), "topk")
    _need(q, torch.bfloat16, (n, H, KV_DIM), "q")
    if q_req is not None:
        _need(q_req, torch.int32, (n,), "q_req")
    if out is None:
        out = torch.empty_like(q)
    _need(out, torch.bfloat16, (n, H, KV_DIM), "out")
    scale = 1.0 / math.sqrt(KV_DIM) if scale is None else scale
    _check(_lib.csa2_sparse_attn(ctypes.byref(cache.struct), n, _ptr(q_req), _ptr(topk), k, _ptr(q), H,
                                 ctypes.c_float(scale), _ptr(out), _stream(cache.device)), "csa2_sparse_attn")
    return out


def prefill_workspace_bytes(n_queries: int) -> int:
    return int(_lib.csa2_prefill_workspace_bytes(int(n_queries)))


def prefill_index(cache: Cache, req: int, q_pos, q, w, k: int = 512, ratio: int = 2, topk=None, workspace=None):
    """Causal prefill Top-k of n queries of request `req`: q_pos int32 [n]
    (token positions), q float32 [n,32,128], w float32 [n,32]; returns topk
    int32 [n, k] (entries ascending, -1 padded)."""
    n = q_pos.shape[0]
    _need(q_pos, torch.int32, (n,), "q_pos")
    _need(q, torch.float32, (n, INDEX_HEADS, INDEX_DIM), "q")
    _need(w, torch.float32, (n, INDEX_HEADS), "w")
    if topk is None:
        topk = torch.empty(n, k, dtype=torch.int32, device=cache.device)
    _need(topk, torch.int32, (n, k), "topk")
    if workspace is None:
        workspace = torch.empty(max(prefill_workspace_bytes(n), 16), dtype=torch.uint8, device=cache.device)
    if workspace.dtype != torch.uint8 or not workspace.is_contiguous() or workspace.device.type != "cuda":
        raise ValueError("workspace: expected a contiguous cuda uint8 tensor")
    _check(_lib.csa2_prefill_index(ctypes.byref(cache.struct), int(req), n, _ptr(q_pos), int(ratio), _ptr(q), _ptr(w),
                                   int(k), _ptr(topk), _ptr(workspace), workspace.numel(), _stream(cache.device)),
           "csa2_prefill_index")
    return topk


def prefill_index_static(cache: Cache, req: int, q_pos, q, w, k: int = 512, ratio: int = 2, topk=None):
    """csa2_prefill_index_static: prefill_index with the library's static
    scratch instead of a workspace (at most 256 queries per call; calls on one
    device must not overlap)."""
    n = q_pos.shape[0]
    _need(q_pos, torch.int32, (n,), "q_pos")
    _need(q, torch.float32, (n, INDEX_HEADS, INDEX_DIM), "q")
    _need(w, torch.float32, (n, INDEX_HEADS), "w")
    if topk is None:
        topk = torch.empty(n, k, dtype=torch.int32, device=cache.device)
    _need(topk, torch.int32, (n, k), "topk")
    _check(_lib.csa2_prefill_index_static(ctypes.byref(cache.struct), int(req), n, _ptr(q_pos), int(ratio), _ptr(q),
                                          _ptr(w), int(k), _ptr(topk), _stream(cache.device)),
           "csa2_prefill_index_static")
    return topk


def attn_workspace_bytes(n_layers: int, n_queries: int, heads: int) -> int:
    return int(_lib.csa2_attn_workspace_bytes(int(n_layers), int(n_queries), int(heads)))


def sparse_attn_layers(cache: Cache, topk, q_layers, scale: float | None = None, out_layers=None, q_req=None,
                       workspace=None):
    """Sparse attention of several layers in one launch; topk: one int32
    [n, k] tensor shared by every layer, or a list with one per layer;
    q_layers: list of bf16 [n, H, 512] -> list of outputs of the same shape.
    workspace: optional uint8 device tensor of attn_workspace_bytes(...) bytes
    (the key splits then merge through it instead of shared memory)."""
    L = len(q_layers)
    topk_layers = list(topk) if isinstance(topk, (list, tuple)) else [topk] * L
    n, k = topk_layers[0].shape
    H = q_layers[0].shape[1]
    if len(topk_layers) != L:
        raise ValueError(f"{len(topk_layers)} Top-k tensors for {L} layers")
    for i, t in enumerate(topk_layers):
        _need(t, torch.int32, (n, k), f"topk[{i}]")
    for i, q in enumerate(q_layers):
        _need(q, torch.bfloat16, (n, H, KV_DIM), f"q_layers[{i}]")
    if q_req is not None:
        _need(q_req, torch.int32, (n,), "q_req")
    if out_layers is None:
        out_layers = [torch.empty_like(q) for q in q_layers]
    for i, o in enumerate(out_layers):
        _need(o, torch.bfloat16, (n, H, KV_DIM), f"out_layers[{i}]")
    scale = 1.0 / math.sqrt(KV_DIM) if scale is None else scale
    qa = (ctypes.c_void_p * L)(*[q.data_ptr() for q in q_layers])
    oa = (ctypes.c_void_p * L)(*[o.data_ptr() for o in out_layers])
    ta = (ctypes.c_void_p * L)(*[t.data_ptr() for t in topk_layers])
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.csa2_sparse_attn_layers(ctypes.byref(cache.struct), L, n, _ptr(q_req), ta, k, qa, H,
                                        ctypes.c_float(scale), oa, _ptr(workspace), ws_bytes,
                                        _stream(cache.device)), "csa2_sparse_attn_layers")
    return out_layers


class SwaKV:
    """One layer's sliding-window KV: FP8 rows in a ring of `window` slots per
    request (codes uint8 [batch, window, 512], exponent bytes [batch, window])."""

    def __init__(self, cache: Cache, window: int):
        self.window = int(window)
        self.codes = torch.zeros(cache.batch, self.window, KV_DIM, dtype=torch.uint8, device=cache.device)
        self.exp = torch.zeros(cache.batch, self.window, dtype=torch.uint8, device=cache.device)


def swa_append(cache: Cache, swa: SwaKV, x, pos, req=None):
    """Quantise SWA rows x float32 [n, 512] and store token pos[i] in slot pos[i] % window."""
    n = pos.shape[0]
    _need(x, torch.float32, (n, KV_DIM), "x")
    _need(pos, torch.int32, (n,), "pos")
    if req is not None:
        _need(req, torch.int32, (n,), "req")
    _check(_lib.csa2_swa_append(ctypes.byref(cache.struct), swa.window, _ptr(swa.codes), _ptr(swa.exp), n, _ptr(x),
                                _ptr(req), _ptr(pos), _stream(cache.device)), "csa2_swa_append")


def sparse_attn_swa(cache: Cache, topk, swa: SwaKV, q_pos, q, scale: float | None = None, out=None, q_req=None):
    """Sparse attention with the query's window (tokens q_pos-window+1 .. q_pos) merged in."""
    n, k = topk.shape
    H = q.shape[1]
    _need(topk, torch.int32, (n, k), "topk")
    _need(q_pos, torch.int32, (n,), "q_pos")
    _need(q, torch.bfloat16, (n, H, KV_DIM), "q")
    if q_req is not None:
        _need(q_req, torch.int32, (n,), "q_req")
    if out is None:
        out = torch.empty_like(q)
    _need(out, torch.bfloat16, (n, H, KV_DIM), "out")
    scale = 1.0 / math.sqrt(KV_DIM) if scale is None else scale
    _check(_lib.csa2_sparse_attn_swa(ctypes.byref(cache.struct), n, _ptr(q_req), _ptr(topk), k, _ptr(swa.codes),
                                     _ptr(swa.exp), swa.window, _ptr(q_pos), _ptr(q), H, ctypes.c_float(scale),
                                     _ptr(out), _stream(cache.device)), "csa2_sparse_attn_swa")
    return out


def get_error(cache: Cache):
    """Synchronise the current stream and return (status, err_word list)."""
    out = (ctypes.c_int32 * 4)()
    st = _lib.csa2_get_error(ctypes.byref(cache.struct), out, _stream(cache.device))
    return st, list(out)


def layer_sources(modes):
    """Group the layers of a layer group by the Top-k they attend over: each
    Full or Reindex layer starts a group, and the Reuse layers that follow it
    join that group (a Reuse layer takes the most recent Full/Reindex layer's
    indices).  Returns a list of lists of layer indices."""
    modes = tuple(modes)
    if not modes or modes[0] == "Ru":
        raise ValueError("a layer group starts with a Full or Reindex layer")
    bad = [m for m in modes if m not in ("F", "Ri", "Ru")]
    if bad:
        raise ValueError(f"unknown layer modes {bad}")
    sources = []
    for layer, m in enumerate(modes):
        if m != "Ru":
            sources.append([layer])
        else:
            sources[-1].append(layer)
    return sources


class DecodeGroup:
    """One decode step of a CSA2 layer group over `cache`, through the C ABI.

    modes: e.g. ("F", "Ri", "Ri", "Ru", "Ru", "Ru").  The first Full layer
    scans the context and (with pool_blocks) builds the pool; Reindex layers
    re-score the pool with their own query; Reuse layers take the previous
    layer's Top-k.  Every layer attends with its own main query.

    With a pool the step is five kernels on the calling stream, each linked
    to the one before by programmatic dependent launch (so it can be captured
    in a CUDA graph): the scan (which also fills the block maxima's
    histogram), the pool selection (which starts from that histogram), the
    Top-k of every Full / Reindex layer (csa2_reindex_layers: one scoring and
    one select launch for all of them), and one attention launch for all
    layers.  Without a pool each Full / Reindex layer takes its flat Top-k
    with csa2_reindex, then the same single attention launch follows.
    """

    def __init__(self, cache: Cache, modes, heads: int, k: int = 512, pool_blocks: int | None = 2048,
                 scale: float | None = None, ik4: Ik4 | None = None):
        if modes[0] != "F":
            raise ValueError("a layer group starts with a Full layer")
        if ik4 is not None and not pool_blocks:
            raise ValueError("the FP4 indexer path needs a pool")
        self.ik4 = ik4
        self.cache, self.modes, self.heads, self.k = cache, tuple(modes), heads, k
        self.pool_blocks = pool_blocks
        self.scale = 1.0 / math.sqrt(KV_DIM) if scale is None else scale
        dev, B = cache.device, cache.batch
        self.blockmax = torch.empty(B, cache.capacity // BLOCK, dtype=torch.float32, device=dev)
        self.pool = torch.empty(B, pool_blocks, dtype=torch.int32, device=dev) if pool_blocks else None
        self.hist = pool_hist(cache) if pool_blocks else None
        # Reuse layers alias the Top-k buffer of the layer they reuse
        self.topk, src = [], None
        for m in self.modes:
            if m == "Ru":
                self.topk.append(src)
            else:
                src = torch.empty(B, k, dtype=torch.int32, device=dev)
                self.topk.append(src)
        self.sources = layer_sources(self.modes)
        self.index_layers = [layers[0] for layers in self.sources]
        if pool_blocks:
            self.rs_ws = torch.zeros(reindex_layers_workspace_bytes(B, len(self.index_layers), pool_blocks),
                                     dtype=torch.uint8, device=dev)
            # one workspace part per Top-k launch pair
            step = MAX_FP4_SCORE_LAYERS if ik4 is not None else len(self.index_layers)
            n_parts = -(-len(self.index_layers) // step)
            self.rs_ws_parts, off = [], 0
            for i in range(n_parts):
                nl = min(step, len(self.index_layers) - i * step)
                nb = reindex_layers_workspace_bytes(B, nl, pool_blocks)
                self.rs_ws_parts.append(self.rs_ws[off:off + nb])
                off += nb
        self.attn_ws = torch.empty(attn_workspace_bytes(len(self.modes), B, heads), dtype=torch.uint8, device=dev)
        # kernels per step: scan, pool, score + select, attention (with a
        # pool); scan, one Top-k per index layer, attention (without)
        self.launches_per_step = (3 + 2 * len(self.rs_ws_parts)) if pool_blocks else 2 + len(self.index_layers)

    def step(self, q_idx, w_idx, q_main, out, timing=None, append=None):
        """q_idx / w_idx: per layer ([B,32,128] / [B,32], None for Reuse);
        q_main / out: per layer bf16 [B, H, 512].  append: optional (kv_new
        [B,512], ik_new [B,128], pos [B]) float32 / int32 rows that each
        request appends (quantise-on-append) before the scan, one per request
        (ctx_len already counts them).  timing: optional dict name -> (start,
        end) CUDA events, recorded on the calling stream around the launches of
        that name ("append", "scan", "pool", "topk", "attn"; an event between
        two launches cuts their programmatic link, so time a separate graph
        with it)."""
        c = self.cache

        def timed(name, fn):
            ev = None if timing is None else timing.get(name)
            if ev is not None:
                ev[0].record()
            torch.cuda.nvtx.range_push(f"csa2 {name}")   # profiler range around the launches
            try:
                r = fn()
            finally:
                torch.cuda.nvtx.range_pop()
            if ev is not None:
                ev[1].record()
            return r

        if append is not None:
            kv_new, ik_new, pos = append

            def do_append():
                append_kv(c, kv_new, ik_new, pos)
                if self.ik4 is not None:
                    append_ik4(c, self.ik4, ik_new, pos)
            timed("append", do_append)
        if self.ik4 is None:
            timed("scan", lambda: index_full(c, q_idx[0], w_idx[0], self.blockmax, hist=self.hist))
        else:
            timed("scan", lambda: index_full_fp4(c, self.ik4, q_idx[0], w_idx[0], self.blockmax, hist=self.hist))
        if self.pool is not None:
            timed("pool", lambda: pool_select(c, self.blockmax, self.pool_blocks, self.pool, hist=self.hist))
            L = self.index_layers
            timed("topk", lambda: self._pool_topk(q_idx, w_idx))
        else:
            def flat():
                for l in self.index_layers:
                    mode = FULL if self.modes[l] == "F" else REINDEX
                    reindex(c, mode, self.k, None, q_idx[l], w_idx[l], topk=self.topk[l])
            timed("topk", flat)
        timed("attn", lambda: sparse_attn_layers(c, self.topk, q_main, self.scale, out, workspace=self.attn_ws))
        return out

    def _pool_topk(self, q_idx, w_idx):
        """Top-k of every index layer over the pool; the FP4 path scores at
        most four layers per launch pair (one block of query scales)."""
        L = self.index_layers
        step = MAX_FP4_SCORE_LAYERS if self.ik4 is not None else len(L)
        for i, ws in zip(range(0, len(L), step), self.rs_ws_parts):
            part = L[i:i + step]
            reindex_layers(self.cache, self.pool, [q_idx[l] for l in part], [w_idx[l] for l in part], self.k,
                           [self.topk[l] for l in part], ws, ik4=self.ik4)

    def launch_names(self, append: bool = False):
        return (["append"] if append else []) + ["scan"] + (["pool"] if self.pool is not None else []) + \
            ["topk", "attn"]


class PrefillGroup:
    """One encoder-style prefill chunk of a CSA2 layer group over request
    `req` of `cache`: every Full (or Reindex) layer runs the causal prefill
    indexer with its own query, Reuse layers take the previous layer's Top-k,
    and every layer attends with its own main query (H heads of 512)."""

    def __init__(self, cache: Cache, req: int, modes, heads: int, n_queries: int, k: int = 512, ratio: int = 2,
                 scale: float | None = None):
        if modes[0] == "Ru":
            raise ValueError("a layer group starts with a Full layer")
        self.cache, self.req, self.modes, self.heads, self.k, self.ratio = cache, req, tuple(modes), heads, k, ratio
        self.scale = 1.0 / math.sqrt(KV_DIM) if scale is None else scale
        dev = cache.device
        self.n = n_queries
        self.workspace = torch.empty(max(prefill_workspace_bytes(n_queries), 16), dtype=torch.uint8, device=dev)
        self.q_req = torch.full((n_queries,), req, dtype=torch.int32, device=dev)
        self.sources = layer_sources(self.modes)
        self.topk = [None] * len(self.modes)
        for layers in self.sources:
            src = torch.empty(n_queries, k, dtype=torch.int32, device=dev)
            for layer in layers:
                self.topk[layer] = src
        self.launches_per_step = 3 * len(self.sources)   # indexer (2 kernels) + one attention launch per source

    def step(self, q_pos, q_idx, w_idx, q_main, out, timing=None):
        """q_pos int32 [n]; q_idx / w_idx per layer (None for Reuse); q_main /
        out per layer bf16 [n, H, 512].  timing: optional dict name -> (start,
        end) CUDA events around "topk<l>" and "attn<l>" (l a Full/Reindex
        layer; its attention launch covers the Reuse layers that follow it)."""
        c = self.cache

        def timed(name, fn):
            ev = None if timing is None else timing.get(name)
            if ev is not None:
                ev[0].record()
            torch.cuda.nvtx.range_push(f"csa2 {name}")
            try:
                fn()
            finally:
                torch.cuda.nvtx.range_pop()
            if ev is not None:
                ev[1].record()

        for layers in self.sources:
            src = layers[0]
            timed(f"topk{src}", lambda: prefill_index(c, self.req, q_pos, q_idx[src], w_idx[src], self.k,
                                                      self.ratio, self.topk[src], self.workspace))
            timed(f"attn{src}", lambda: sparse_attn_layers(c, self.topk[src], [q_main[l] for l in layers],
                                                           self.scale, [out[l] for l in layers], q_req=self.q_req))
        return out

    def launch_names(self):
        names = []
        for layers in self.sources:
            names += [f"topk{layers[0]}", f"attn{layers[0]}"]
        return names
