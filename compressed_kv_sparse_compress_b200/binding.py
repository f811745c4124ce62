"""ctypes binding of libckv (include/ckv.h).

Argument marshalling only: every step of the decode path runs in the library's CUDA kernels.
PyTorch provides device memory and the current stream. There is no fallback: if libckv.so is
missing or a call fails, an exception is raised.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libckv.so")

CKV_OK = 0
CKV_ERR_INVALID_ARG = -1
CKV_ERR_UNSUPPORTED = -2
CKV_ERR_OUT_OF_BLOCKS = -3
CKV_ERR_WORKSPACE = -4
CKV_ERR_CUDA = -5

CKV_DEV_BAD_BLOCK = 0x1
CKV_DEV_BAD_LENGTH = 0x2
CKV_DEV_BAD_INDEX = 0x4
CKV_DEV_TIMEOUT = 0x8

CKV_F32, CKV_BF16, CKV_FP8_E4M3, CKV_NVFP4 = 0, 1, 2, 3
DTYPES = {"f32": CKV_F32, "bf16": CKV_BF16, "fp8": CKV_FP8_E4M3, "nvfp4": CKV_NVFP4}

# every symbol include/ckv.h declares
EXPORTS = (
    "kv_block_pool_create", "kv_block_pool_destroy", "kv_block_alloc", "kv_block_free",
    "kv_block_pool_num_free", "ckv_cache_row_bytes", "ckv_score_stride",
    "ckv_indexer_workspace_bytes", "ckv_attention_workspace_bytes", "kv_compress_append",
    "sparse_indexer_topk", "compressed_window_attention", "ckv_status_str", "ckv_launch_count",
    "ckv_profile_events", "sparse_indexer_topk_noalloc", "ckv_decode_step_workspace_bytes",
    "ckv_decode_step", "kv_index_append", "ckv_mh_indexer_workspace_bytes", "sparse_mh_indexer_topk",
    "kv_window_replay", "ckv_debug_force_timeout",
)
CKV_PROF_SCORE, CKV_PROF_ATTENTION = 0, 1


class CkvError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {status_str(status)} ({status})")
        self.status = status


class LayerCfgC(ctypes.Structure):
    _fields_ = [("num_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("rope_dim", ctypes.c_int32), ("ratio", ctypes.c_int32),
                ("window", ctypes.c_int32), ("comp_dtype", ctypes.c_int32),
                ("win_dtype", ctypes.c_int32), ("sm_scale", ctypes.c_float),
                ("rope_base", ctypes.c_float)]


class LayerCacheC(ctypes.Structure):
    _fields_ = [("comp_codes", ctypes.c_void_p), ("comp_scales", ctypes.c_void_p),
                ("win_codes", ctypes.c_void_p), ("win_scales", ctypes.c_void_p),
                ("residue_kv", ctypes.c_void_p), ("residue_logit", ctypes.c_void_p),
                ("comp_table", ctypes.c_void_p), ("win_table", ctypes.c_void_p),
                ("table_stride", ctypes.c_int32), ("comp_blocks", ctypes.c_int32),
                ("win_blocks", ctypes.c_int32)]


class IndexCfgC(ctypes.Structure):
    _fields_ = [("index_heads", ctypes.c_int32), ("index_dim", ctypes.c_int32)]


class IndexCacheC(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("residue_k", ctypes.c_void_p), ("residue_logit", ctypes.c_void_p)]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads libckv.so once; raises when it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libckv.so not found at {path}: build it with "
                           "`python -m compressed_kv_sparse_compress_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    P = ctypes.POINTER
    lib.kv_block_pool_create.argtypes = [i32, P(vp)]
    lib.kv_block_pool_destroy.argtypes = [vp]
    lib.kv_block_alloc.argtypes = [vp, i32, P(i32)]
    lib.kv_block_free.argtypes = [vp, P(i32), i32]
    lib.kv_block_pool_num_free.argtypes = [vp]
    lib.kv_block_pool_num_free.restype = i32
    lib.ckv_cache_row_bytes.argtypes = [P(LayerCfgC), P(sz), P(sz), P(sz), P(sz)]
    lib.ckv_score_stride.argtypes = [P(LayerCfgC), i32]
    lib.ckv_score_stride.restype = i64
    lib.ckv_indexer_workspace_bytes.argtypes = [P(LayerCfgC), i32, i32, i32]
    lib.ckv_indexer_workspace_bytes.restype = sz
    lib.ckv_attention_workspace_bytes.argtypes = [P(LayerCfgC), i32, i32, i32]
    lib.ckv_attention_workspace_bytes.restype = sz
    lib.kv_compress_append.argtypes = [P(LayerCfgC), P(LayerCacheC), i32, vp, vp, i32, i32, vp,
                                       vp, vp, vp]
    lib.kv_window_replay.argtypes = [P(LayerCfgC), P(LayerCacheC), i32, vp, i32, vp, vp, vp, vp]
    lib.kv_window_replay.restype = ctypes.c_int
    lib.sparse_indexer_topk.argtypes = [P(LayerCfgC), P(LayerCacheC), i32, vp, i32, vp, i32, vp,
                                        vp, vp, vp, sz, vp, vp]
    lib.compressed_window_attention.argtypes = [P(LayerCfgC), P(LayerCacheC), i32, vp, i32, vp,
                                                vp, vp, i32, vp, vp, sz, vp, vp]
    lib.sparse_indexer_topk_noalloc.argtypes = [P(LayerCfgC), P(LayerCacheC), i32, vp, i32, vp, i32,
                                                vp, vp, vp, vp, vp]
    lib.sparse_indexer_topk_noalloc.restype = ctypes.c_int
    lib.ckv_decode_step_workspace_bytes.argtypes = [P(LayerCfgC), i32, i32, i32]
    lib.ckv_decode_step_workspace_bytes.restype = sz
    lib.ckv_decode_step.argtypes = [P(LayerCfgC), P(LayerCacheC), i32, vp, i32, vp, vp, vp, i32, vp,
                                    vp, vp, vp, sz, vp, vp]
    lib.ckv_decode_step.restype = ctypes.c_int
    lib.kv_index_append.argtypes = [P(LayerCfgC), P(LayerCacheC), P(IndexCfgC), P(IndexCacheC), i32, vp,
                                    vp, i32, i32, vp, vp, vp, vp]
    lib.kv_index_append.restype = ctypes.c_int
    lib.ckv_mh_indexer_workspace_bytes.argtypes = [P(LayerCfgC), P(IndexCfgC), i32, i32, i32]
    lib.ckv_mh_indexer_workspace_bytes.restype = sz
    lib.sparse_mh_indexer_topk.argtypes = [P(LayerCfgC), P(LayerCacheC), P(IndexCfgC), P(IndexCacheC), i32,
                                           vp, i32, vp, vp, i32, vp, vp, vp, vp, sz, vp, vp]
    lib.sparse_mh_indexer_topk.restype = ctypes.c_int
    lib.ckv_status_str.argtypes = [ctypes.c_int]
    lib.ckv_status_str.restype = ctypes.c_char_p
    lib.ckv_profile_events.argtypes = [ctypes.c_int, vp, vp]
    lib.ckv_profile_events.restype = ctypes.c_int
    lib.ckv_debug_force_timeout.argtypes = [i32]
    lib.ckv_debug_force_timeout.restype = ctypes.c_int
    lib.ckv_launch_count.argtypes = []
    lib.ckv_launch_count.restype = ctypes.c_uint64
    for name in ("kv_block_pool_create", "kv_block_pool_destroy", "kv_block_alloc",
                 "kv_block_free", "ckv_cache_row_bytes", "kv_compress_append",
                 "sparse_indexer_topk", "compressed_window_attention"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def status_str(status: int) -> str:
    return load_library().ckv_status_str(status).decode()


def launch_count() -> int:
    return int(load_library().ckv_launch_count())


def debug_force_timeout(request: int) -> None:
    """Test hook of the device failure path (ckv_debug_force_timeout); -1 turns it off."""
    _check("ckv_debug_force_timeout", load_library().ckv_debug_force_timeout(request))


def profile_events(which: int, begin=None, end=None) -> None:
    """Records torch.cuda.Event pair (begin, end) around one kernel of later calls (diagnostic)."""
    b = begin.cuda_event if begin is not None else None
    e = end.cuda_event if end is not None else None
    _check("ckv_profile_events", load_library().ckv_profile_events(which, b, e))


def _check(fn: str, st: int) -> None:
    if st != CKV_OK:
        raise CkvError(fn, st)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("device tensor expected")
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


# ------------------------------------------------------------------------------------------ pools


class BlockPool:
    """Host free list of physical block ids (kv_block_pool_*)."""

    def __init__(self, num_blocks: int):
        lib = load_library()
        self._h = ctypes.c_void_p()
        _check("kv_block_pool_create", lib.kv_block_pool_create(num_blocks, ctypes.byref(self._h)))
        self.num_blocks = num_blocks

    def alloc(self, n: int):
        """n ids, or None when the pool has fewer than n free (nothing allocated)."""
        arr = (ctypes.c_int32 * max(n, 1))()
        st = load_library().kv_block_alloc(self._h, n, arr)
        if st == CKV_ERR_OUT_OF_BLOCKS:
            return None
        _check("kv_block_alloc", st)
        return [int(arr[i]) for i in range(n)]

    def free(self, ids) -> None:
        ids = list(ids)
        arr = (ctypes.c_int32 * max(len(ids), 1))(*ids)
        _check("kv_block_free", load_library().kv_block_free(self._h, arr, len(ids)))

    @property
    def num_free(self) -> int:
        n = load_library().kv_block_pool_num_free(self._h)
        if n < 0:
            raise CkvError("kv_block_pool_num_free", n)
        return n

    def close(self) -> None:
        if self._h:
            load_library().kv_block_pool_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ------------------------------------------------------------------------------------------ layer


@dataclass
class LayerConfig:
    num_heads: int
    head_dim: int
    rope_dim: int
    ratio: int
    window: int
    comp_dtype: str      # 'f32' | 'bf16' | 'nvfp4'
    win_dtype: str       # 'f32' | 'fp8'
    sm_scale: float = 0.0
    rope_base: float = 0.0

    def c(self) -> LayerCfgC:
        return LayerCfgC(self.num_heads, self.head_dim, self.rope_dim, self.ratio, self.window,
                         DTYPES[self.comp_dtype], DTYPES[self.win_dtype], self.sm_scale,
                         self.rope_base)

    def row_bytes(self):
        a, b, c, d = (ctypes.c_size_t() for _ in range(4))
        _check("ckv_cache_row_bytes", load_library().ckv_cache_row_bytes(
            ctypes.byref(self.c()), ctypes.byref(a), ctypes.byref(b), ctypes.byref(c), ctypes.byref(d)))
        return a.value, b.value, c.value, d.value


@dataclass
class LayerCache:
    """Device tensors of one layer's caches (caller-owned; see ckv_layer_cache)."""
    comp_codes: torch.Tensor
    comp_scales: torch.Tensor | None
    win_codes: torch.Tensor
    win_scales: torch.Tensor | None
    residue_kv: torch.Tensor
    residue_logit: torch.Tensor
    comp_table: torch.Tensor
    win_table: torch.Tensor

    def c(self) -> LayerCacheC:
        return LayerCacheC(_ptr(self.comp_codes), _ptr(self.comp_scales), _ptr(self.win_codes),
                           _ptr(self.win_scales), _ptr(self.residue_kv), _ptr(self.residue_logit),
                           _ptr(self.comp_table), _ptr(self.win_table),
                           int(self.comp_table.shape[1]), int(self.comp_codes.shape[0]),
                           int(self.win_codes.shape[0]))


def score_stride(cfg: LayerConfig, max_seq_len: int) -> int:
    return int(load_library().ckv_score_stride(ctypes.byref(cfg.c()), max_seq_len))


def indexer_workspace_bytes(cfg: LayerConfig, batch: int, max_seq_len: int, top_k: int) -> int:
    return int(load_library().ckv_indexer_workspace_bytes(ctypes.byref(cfg.c()), batch,
                                                          max_seq_len, top_k))


def attention_workspace_bytes(cfg: LayerConfig, batch: int, max_seq_len: int,
                              max_selected: int) -> int:
    return int(load_library().ckv_attention_workspace_bytes(ctypes.byref(cfg.c()), batch,
                                                            max_seq_len, max_selected))


def kv_compress_append(cfg: LayerConfig, cache: LayerCache, prev_len: torch.Tensor,
                       kv_new: torch.Tensor, logit_new: torch.Tensor, status: torch.Tensor,
                       cu_new: torch.Tensor | None = None, max_new: int = 1,
                       max_seq_len: int | None = None, stream=None) -> None:
    batch = int(prev_len.shape[0])
    if max_seq_len is None:
        max_seq_len = int(cache.comp_table.shape[1]) * 256
    _check("kv_compress_append", load_library().kv_compress_append(
        ctypes.byref(cfg.c()), ctypes.byref(cache.c()), batch, _ptr(prev_len), _ptr(cu_new),
        max_new if cu_new is not None else 1, max_seq_len, _ptr(kv_new), _ptr(logit_new),
        _ptr(status), _stream(stream)))


def kv_window_replay(cfg: LayerConfig, cache: LayerCache, seq_len: torch.Tensor, kv: torch.Tensor,
                     logit: torch.Tensor, status: torch.Tensor, max_seq_len: int | None = None,
                     stream=None) -> None:
    """SWA bounded replay: kv [batch][W][D] / logit [batch][W] hold the recomputed raw tokens of
    positions L - min(W, L) .. L - 1 (row i = position L - n_w + i)."""
    batch = int(seq_len.shape[0])
    if max_seq_len is None:
        max_seq_len = int(cache.comp_table.shape[1]) * 256
    _check("kv_window_replay", load_library().kv_window_replay(
        ctypes.byref(cfg.c()), ctypes.byref(cache.c()), batch, _ptr(seq_len), max_seq_len, _ptr(kv),
        _ptr(logit), _ptr(status), _stream(stream)))


def sparse_indexer_topk(cfg: LayerConfig, cache: LayerCache, seq_len: torch.Tensor,
                        max_seq_len: int, q: torch.Tensor, top_k: int, idx: torch.Tensor,
                        cnt: torch.Tensor, workspace: torch.Tensor, status: torch.Tensor,
                        scores: torch.Tensor | None = None, stream=None) -> None:
    batch = int(seq_len.shape[0])
    _check("sparse_indexer_topk", load_library().sparse_indexer_topk(
        ctypes.byref(cfg.c()), ctypes.byref(cache.c()), batch, _ptr(seq_len), max_seq_len, _ptr(q),
        top_k, _ptr(idx), _ptr(cnt), _ptr(scores), _ptr(workspace), workspace.numel(),
        _ptr(status), _stream(stream)))


def sparse_indexer_topk_noalloc(cfg: LayerConfig, cache: LayerCache, seq_len: torch.Tensor,
                                max_seq_len: int, q: torch.Tensor, top_k: int, idx: torch.Tensor,
                                cnt: torch.Tensor, status: torch.Tensor,
                                scores: torch.Tensor | None = None, stream=None) -> None:
    """sparse_indexer_topk with the library's own fixed scratch (no workspace, no allocation)."""
    batch = int(seq_len.shape[0])
    _check("sparse_indexer_topk_noalloc", load_library().sparse_indexer_topk_noalloc(
        ctypes.byref(cfg.c()), ctypes.byref(cache.c()), batch, _ptr(seq_len), max_seq_len, _ptr(q),
        top_k, _ptr(idx), _ptr(cnt), _ptr(scores), _ptr(status), _stream(stream)))


def compressed_window_attention(cfg: LayerConfig, cache: LayerCache, seq_len: torch.Tensor,
                                max_seq_len: int, q: torch.Tensor, idx: torch.Tensor | None,
                                cnt: torch.Tensor | None, out: torch.Tensor,
                                workspace: torch.Tensor, status: torch.Tensor,
                                stream=None) -> None:
    batch = int(seq_len.shape[0])
    stride = int(idx.shape[1]) if idx is not None else 0
    _check("compressed_window_attention", load_library().compressed_window_attention(
        ctypes.byref(cfg.c()), ctypes.byref(cache.c()), batch, _ptr(seq_len), max_seq_len,
        _ptr(q), _ptr(idx), _ptr(cnt), stride, _ptr(out), _ptr(workspace), workspace.numel(),
        _ptr(status), _stream(stream)))


def decode_step_workspace_bytes(cfg: LayerConfig, batch: int, max_seq_len: int, top_k: int) -> int:
    return int(load_library().ckv_decode_step_workspace_bytes(ctypes.byref(cfg.c()), batch,
                                                              max_seq_len, top_k))


def decode_step(cfg: LayerConfig, cache: LayerCache, seq_len: torch.Tensor, max_seq_len: int,
                q: torch.Tensor, kv_new: torch.Tensor, logit_new: torch.Tensor, top_k: int,
                idx: torch.Tensor | None, cnt: torch.Tensor | None, out: torch.Tensor,
                workspace: torch.Tensor, status: torch.Tensor, stream=None) -> None:
    """ckv_decode_step: append the token at seq_len-1, select (top_k > 0) and attend, one call."""
    batch = int(seq_len.shape[0])
    _check("ckv_decode_step", load_library().ckv_decode_step(
        ctypes.byref(cfg.c()), ctypes.byref(cache.c()), batch, _ptr(seq_len), max_seq_len, _ptr(q),
        _ptr(kv_new), _ptr(logit_new), top_k, _ptr(idx), _ptr(cnt), _ptr(out), _ptr(workspace),
        workspace.numel(), _ptr(status), _stream(stream)))


# ------------------------------------------------------------------------------ multi-head indexer


@dataclass
class IndexConfig:
    index_heads: int = 64
    index_dim: int = 128

    def c(self) -> IndexCfgC:
        return IndexCfgC(self.index_heads, self.index_dim)


@dataclass
class IndexCache:
    """Device tensors of a layer's index plane (see ckv_index_cache); the rings may be None for
    scoring only."""
    codes: torch.Tensor
    scales: torch.Tensor
    residue_k: torch.Tensor | None = None
    residue_logit: torch.Tensor | None = None

    def c(self) -> IndexCacheC:
        return IndexCacheC(_ptr(self.codes), _ptr(self.scales), _ptr(self.residue_k),
                           _ptr(self.residue_logit))


def kv_index_append(cfg: LayerConfig, cache: LayerCache, icfg: IndexConfig, icache: IndexCache,
                    prev_len: torch.Tensor, k_new: torch.Tensor, logit_new: torch.Tensor,
                    status: torch.Tensor, cu_new: torch.Tensor | None = None, max_new: int = 1,
                    max_seq_len: int | None = None, stream=None) -> None:
    batch = int(prev_len.shape[0])
    if max_seq_len is None:
        max_seq_len = int(cache.comp_table.shape[1]) * 256
    _check("kv_index_append", load_library().kv_index_append(
        ctypes.byref(cfg.c()), ctypes.byref(cache.c()), ctypes.byref(icfg.c()), ctypes.byref(icache.c()),
        batch, _ptr(prev_len), _ptr(cu_new), max_new if cu_new is not None else 1, max_seq_len, _ptr(k_new),
        _ptr(logit_new), _ptr(status), _stream(stream)))


def mh_indexer_workspace_bytes(cfg: LayerConfig, icfg: IndexConfig, batch: int, max_seq_len: int,
                               top_k: int) -> int:
    return int(load_library().ckv_mh_indexer_workspace_bytes(ctypes.byref(cfg.c()), ctypes.byref(icfg.c()),
                                                             batch, max_seq_len, top_k))


def sparse_mh_indexer_topk(cfg: LayerConfig, cache: LayerCache, icfg: IndexConfig, icache: IndexCache,
                           seq_len: torch.Tensor, max_seq_len: int, q_index: torch.Tensor,
                           weights: torch.Tensor, top_k: int, idx: torch.Tensor, cnt: torch.Tensor,
                           workspace: torch.Tensor, status: torch.Tensor,
                           scores: torch.Tensor | None = None, stream=None) -> None:
    batch = int(seq_len.shape[0])
    _check("sparse_mh_indexer_topk", load_library().sparse_mh_indexer_topk(
        ctypes.byref(cfg.c()), ctypes.byref(cache.c()), ctypes.byref(icfg.c()), ctypes.byref(icache.c()),
        batch, _ptr(seq_len), max_seq_len, _ptr(q_index), _ptr(weights), top_k, _ptr(idx), _ptr(cnt),
        _ptr(scores), _ptr(workspace), workspace.numel(), _ptr(status), _stream(stream)))
