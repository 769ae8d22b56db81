"""Thin ctypes binding over libpariskv.so (the C ABI declared in include/pariskv.h,
include/pariskv_cache.h, include/pariskv_dense.h, include/pariskv_learned.h and
include/pariskv_debug.h).

Only argument marshalling happens here: tensors become data pointers and strides become the
library's slab strides; every step of the retrieval path runs in the library's CUDA kernels.
Importing this module loads the library and raises if it is missing (there is no fallback).
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
# PARISKV_LIBRARY=check loads the checked build (extra device-side bounds checks; see
# build.py); the default is the product library.
LIB_PATH = os.path.join(_PKG, "_lib", "libpariskv_check.so" if os.environ.get(
    "PARISKV_LIBRARY") == "check" else "libpariskv.so")
HEADERS = [os.path.join(os.path.dirname(_PKG), "include", h)
           for h in ("pariskv.h", "pariskv_cache.h", "pariskv_dense.h", "pariskv_learned.h",
                     "pariskv_debug.h")]

OK, EINVAL, ENOMEM, ECUDA, ECAPACITY, ETIMEOUT = range(6)
F32, BF16 = 0, 1
LEVELS_UNIFORM, LEVELS_PRIOR, LEVELS_TABLE = range(3)


class PariskvError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        super().__init__(f"{where}: status {status} ({_status_name(status)}): {message}")
        self.status = status


def _status_name(s: int) -> str:
    return ["OK", "EINVAL", "ENOMEM", "ECUDA", "ECAPACITY", "ETIMEOUT"][s] if 0 <= s < 6 else "?"


class Config(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("B", ctypes.c_int32), ("m", ctypes.c_int32),
                ("rho", ctypes.c_int32), ("w_rank1", ctypes.c_int32), ("w_rest", ctypes.c_int32),
                ("cand_bp", ctypes.c_int32), ("batch", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("group", ctypes.c_int32),
                ("capacity", ctypes.c_int64), ("dtype", ctypes.c_int32),
                ("levels", ctypes.c_int32), ("level_table", ctypes.c_float * 8)]

    @property
    def num_q_heads(self) -> int:
        return self.num_kv_heads * self.group


class CacheConfig(ctypes.Structure):
    _fields_ = [("n_sink", ctypes.c_int32), ("n_local", ctypes.c_int32),
                ("n_buffer", ctypes.c_int32), ("k", ctypes.c_int32),
                ("retrieval_capacity", ctypes.c_int64)]


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python -m long_context_kv_srht_b200.build`")
lib = ctypes.CDLL(LIB_PATH)

_P = ctypes.c_void_p
_I32, _I64 = ctypes.c_int32, ctypes.c_int64
_S = ctypes.c_int
_SIGS = {
    "pariskv_config_default": (_S, [ctypes.POINTER(Config)]),
    "pariskv_build_index": (_S, [ctypes.POINTER(Config), _P, _P, _I64, _I64, _P, ctypes.POINTER(_P)]),
    "pariskv_append": (_S, [_P, _P, _I64, _I64, _P]),
    "pariskv_search": (_S, [_P, _P, _I32, _P, _P, _P]),
    "pariskv_sparse_attend": (_S, [ctypes.POINTER(Config), _P, _P, _P, _I64, _I64, _P, _I32,
                                   ctypes.c_float, _P, _I32, _P]),
    "pariskv_sparse_attend_noalloc": (_S, [ctypes.POINTER(Config), _P, _P, _P, _I64, _I64, _P,
                                           _I32, ctypes.c_float, _P, _I32, _P]),
    "pariskv_export_bytes": (_S, [_P, ctypes.POINTER(ctypes.c_size_t)]),
    "pariskv_export": (_S, [_P, _P, ctypes.c_size_t, _P]),
    "pariskv_import": (_S, [_P, ctypes.c_size_t, _I64, _P, ctypes.POINTER(_P)]),
    "pariskv_dense_attend": (_S, [ctypes.POINTER(Config), _P, _P, _P, _I64, _I64, ctypes.c_float,
                                  _P, _I32, _P]),
    "pariskv_prior_levels": (_S, [ctypes.POINTER(ctypes.c_float)]),
    "pariskv_train_centroids": (_S, [ctypes.POINTER(Config), _P, _P, _I64, _I64, _I32, _P, _P]),
    "pariskv_set_centroids": (_S, [_P, _P, _P]),
    "pariskv_sync": (_S, [_P, _P]),
    "pariskv_destroy": (_S, [_P]),
    "pariskv_size": (_I64, [_P]),
    "pariskv_last_launch_count": (_I32, []),
    "pariskv_status_string": (ctypes.c_char_p, [_S]),
    "pariskv_last_error": (ctypes.c_char_p, []),
    "pariskv_debug_rotate": (_S, [ctypes.POINTER(Config), _P, _P, _I64, _P, _P, _P]),
    "pariskv_debug_build_index_rotated": (_S, [ctypes.POINTER(Config), _P, _P, _P, _I64, _I64, _P,
                                               ctypes.POINTER(_P)]),
    "pariskv_debug_append_rotated": (_S, [_P, _P, _P, _I64, _I64, _P]),
    "pariskv_debug_search_rotated": (_S, [_P, _P, _P, _I32, _P, _P, _P]),
    "pariskv_debug_export_index": (_S, [_P, _P, _P, _P]),
    "pariskv_debug_export_search": (_S, [_P, _P, _P, ctypes.POINTER(_I64), _P, _P]),
    "pariskv_debug_profile": (_S, [_P, _I32]),
    "pariskv_debug_stage_ms": (_S, [_P, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(_I32)]),
    "pariskv_debug_read_stream": (_S, [_P, _I64, _P, _P]),
    "pariskv_debug_gather_candidates": (_S, [_P, _P, _P]),
    "pariskv_debug_inject_bad_candidate": (_S, [_P, _I32, _I64, _I32]),
    "pariskv_debug_set_launch": (_S, [_P, _I32, _I32, _I32]),
    "pariskv_debug_inject_wait_timeout": (_S, [_P]),
    "pariskv_debug_check_guards": (_S, []),
    "pariskv_debug_union_rows": (_S, [ctypes.POINTER(_I64)]),
    "pariskv_cache_create": (_S, [ctypes.POINTER(Config), ctypes.POINTER(CacheConfig), _P, _P,
                                  ctypes.POINTER(_P)]),
    "pariskv_cache_prefill": (_S, [_P, _P, _P, _I64, _I64, _P]),
    "pariskv_cache_step": (_S, [_P, _P, _P, _P, ctypes.c_float, _P, _I32, _P, _P]),
    "pariskv_cache_counts": (_S, [_P, ctypes.POINTER(_I64)]),
    "pariskv_cache_index": (_P, [_P]),
    "pariskv_cache_destroy": (_S, [_P]),
}

STAGES = ("query_prep", "vote", "threshold", "compact", "rerank", "topk")
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(lib, _name)
    _f.restype = _res
    _f.argtypes = _args


def declared_symbols() -> list:
    """Every function declared in the public and test-only headers."""
    names = []
    for h in HEADERS:
        with open(h) as f:
            names += re.findall(r"PARISKV_API\s+[\w\s\*]+?\b(pariskv_\w+)\s*\(", f.read())
    return names


def last_error() -> str:
    return lib.pariskv_last_error().decode()


def _check(status: int, where: str) -> None:
    if status != OK:
        raise PariskvError(status, where, last_error())


def config(**kw) -> Config:
    c = Config()
    _check(lib.pariskv_config_default(ctypes.byref(c)), "pariskv_config_default")
    for k, v in kw.items():
        if k == "dtype" and isinstance(v, str):
            v = BF16 if v == "bf16" else F32
        if k == "levels" and isinstance(v, str):
            v = {"uniform": LEVELS_UNIFORM, "prior": LEVELS_PRIOR, "table": LEVELS_TABLE}[v]
        if k == "level_table":
            v = (ctypes.c_float * 8)(*[float(x) for x in v])
        setattr(c, k, v)
    return c


def prior_levels() -> np.ndarray:
    """pariskv_prior_levels: the 8 magnitude levels of PARISKV_LEVELS_PRIOR."""
    out = (ctypes.c_float * 8)()
    _check(lib.pariskv_prior_levels(out), "pariskv_prior_levels")
    return np.array(out, dtype=np.float32)


def _stream(stream) -> int:
    import torch
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _signs_ptr(signs) -> tuple:
    a = np.ascontiguousarray(np.asarray(signs.cpu() if hasattr(signs, "cpu") else signs,
                                        dtype=np.int8))
    return a, a.ctypes.data


def _slab(t, d: int = 128) -> int:
    """Token slab stride of a [units..., tokens, d] view (rows contiguous, d elements each)."""
    assert t.stride(-1) == 1 and t.stride(-2) == d, "rows must be contiguous d-vectors"
    if t.dim() <= 2:
        return t.shape[-2] if t.dim() == 2 else 1
    return t.stride(-3) // d


class Index:
    """Owner of a ``pariskv_index*``; methods map one-to-one onto the C calls."""

    def __init__(self, handle: int, cfg: Config, owned: bool = True):
        self.handle = ctypes.c_void_p(handle)
        self.cfg = cfg
        self.owned = owned          # False for a view of an index some other object owns

    # -- product calls ------------------------------------------------------------------
    def append(self, keys, t: Optional[int] = None, stream=None) -> None:
        t = keys.shape[-2] if t is None else t
        _check(lib.pariskv_append(self.handle, keys.data_ptr(), _slab(keys), t, _stream(stream)),
               "pariskv_append")

    def search(self, q, k: int, topk_idx=None, topk_est=None, want_est: bool = True,
               stream=None):
        import torch
        H = self.cfg.batch * self.cfg.num_q_heads
        if topk_idx is None:
            topk_idx = torch.empty((H, k), dtype=torch.int32, device=q.device)
        if topk_est is None and want_est:
            topk_est = torch.empty((H, k), dtype=torch.float32, device=q.device)
        _check(lib.pariskv_search(self.handle, q.data_ptr(), k, topk_idx.data_ptr(),
                                  topk_est.data_ptr() if topk_est is not None else None,
                                  _stream(stream)), "pariskv_search")
        return topk_idx, topk_est

    def sync(self, stream=None) -> None:
        _check(lib.pariskv_sync(self.handle, _stream(stream)), "pariskv_sync")

    def set_centroids(self, centroids, stream=None) -> None:
        """pariskv_set_centroids: learned centroids [units, 16, 256, 8] fp32 (empty index)."""
        _check(lib.pariskv_set_centroids(self.handle, centroids.data_ptr(), _stream(stream)),
               "pariskv_set_centroids")

    def export_image(self, stream=None) -> np.ndarray:
        """pariskv_export: the index image as a uint8 array (host memory)."""
        nb = ctypes.c_size_t(0)
        _check(lib.pariskv_export_bytes(self.handle, ctypes.byref(nb)), "pariskv_export_bytes")
        buf = np.empty((nb.value,), np.uint8)
        _check(lib.pariskv_export(self.handle, buf.ctypes.data, nb.value, _stream(stream)),
               "pariskv_export")
        return buf

    @property
    def size(self) -> int:
        return int(lib.pariskv_size(self.handle))

    def destroy(self) -> None:
        if self.handle and self.owned:
            lib.pariskv_destroy(self.handle)
        self.handle = ctypes.c_void_p(0)

    def __del__(self):
        try:
            self.destroy()
        except Exception:
            pass

    # -- test-only calls ----------------------------------------------------------------
    def append_rotated(self, y, knorm, stream=None) -> None:
        _check(lib.pariskv_debug_append_rotated(self.handle, y.data_ptr(), knorm.data_ptr(),
                                                _slab(y), y.shape[-2], _stream(stream)),
               "pariskv_debug_append_rotated")

    def search_rotated(self, qt, qnorm, k: int, stream=None):
        import torch
        H = self.cfg.batch * self.cfg.num_q_heads
        idx = torch.empty((H, k), dtype=torch.int32, device=qt.device)
        est = torch.empty((H, k), dtype=torch.float32, device=qt.device)
        _check(lib.pariskv_debug_search_rotated(self.handle, qt.data_ptr(), qnorm.data_ptr(), k,
                                                idx.data_ptr(), est.data_ptr(), _stream(stream)),
               "pariskv_debug_search_rotated")
        return idx, est

    def inject_bad_candidate(self, head: int, pos: int, value: int) -> None:
        """pariskv_debug_inject_bad_candidate (test hook, consumed by the next search)."""
        _check(lib.pariskv_debug_inject_bad_candidate(self.handle, head, pos, value),
               "pariskv_debug_inject_bad_candidate")

    def set_launch(self, vote_ctas: int = 0, rerank_ctas: int = 0, topk_mode: int = 0) -> None:
        """pariskv_debug_set_launch: force the launch shapes of later searches (0: automatic)."""
        _check(lib.pariskv_debug_set_launch(self.handle, vote_ctas, rerank_ctas, topk_mode),
               "pariskv_debug_set_launch")

    def inject_wait_timeout(self) -> None:
        """pariskv_debug_inject_wait_timeout: the next search's top-k copy wait runs out."""
        _check(lib.pariskv_debug_inject_wait_timeout(self.handle),
               "pariskv_debug_inject_wait_timeout")

    def gather_candidates(self, sink, stream=None) -> None:
        """pariskv_debug_gather_candidates: the last search's candidate records read once,
        without arithmetic (the rerank's gathers alone); ``sink`` a device tensor (4 bytes)."""
        _check(lib.pariskv_debug_gather_candidates(self.handle, sink.data_ptr(), _stream(stream)),
               "pariskv_debug_gather_candidates")

    def profile(self, enable: bool = True) -> None:
        _check(lib.pariskv_debug_profile(self.handle, int(enable)), "pariskv_debug_profile")

    def stage_ms(self) -> dict:
        ms = (ctypes.c_float * 8)()
        n = _I32(0)
        _check(lib.pariskv_debug_stage_ms(self.handle, ms, ctypes.byref(n)),
               "pariskv_debug_stage_ms")
        return {STAGES[i]: float(ms[i]) for i in range(n.value)}

    def export_index(self):
        units = self.cfg.batch * self.cfg.num_kv_heads
        n = self.size
        ids = np.empty((units, n, 16), np.uint8)
        codes = np.empty((units, n, 128), np.uint8)
        fac = np.empty((units, n, 16), np.float32)
        _check(lib.pariskv_debug_export_index(self.handle, ids.ctypes.data, codes.ctypes.data,
                                              fac.ctypes.data), "pariskv_debug_export_index")
        return ids, codes, fac

    def export_search(self):
        H = self.cfg.batch * self.cfg.num_q_heads
        n = self.size
        C = _I64(0)
        _check(lib.pariskv_debug_export_search(self.handle, None, None, ctypes.byref(C), None,
                                               None), "pariskv_debug_export_search")
        C = int(C.value)
        lut = np.empty((H, 16, 256), np.uint8)
        scores = np.empty((H, n), np.int32)
        cand = np.empty((H, C), np.int32)
        S = np.empty((H, C), np.float32)
        _check(lib.pariskv_debug_export_search(self.handle, lut.ctypes.data, scores.ctypes.data,
                                               None, cand.ctypes.data, S.ctypes.data),
               "pariskv_debug_export_search")
        return lut, scores, cand, S


def build_index(cfg: Config, signs, keys, n: Optional[int] = None, stream=None) -> Index:
    """keys: tensor [batch, num_kv_heads, L, d] (device or pinned host); n <= L tokens used."""
    n = keys.shape[-2] if n is None else n
    sa, sp = _signs_ptr(signs)
    h = _P()
    _check(lib.pariskv_build_index(ctypes.byref(cfg), sp, keys.data_ptr(), _slab(keys), n,
                                   _stream(stream), ctypes.byref(h)), "pariskv_build_index")
    return Index(h.value, cfg)


def import_index(image, capacity: int = 0, stream=None) -> Index:
    """pariskv_import: an index from an image (a uint8 numpy array or bytes)."""
    buf = np.ascontiguousarray(np.frombuffer(image, np.uint8) if isinstance(image, bytes)
                               else image, dtype=np.uint8)
    h = _P()
    if stream is None:
        import torch
        # the legacy default stream when no device is visible (the call then fails in the
        # library with ECUDA, after it has checked the image on the host)
        st = torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else 0
    else:
        st = _stream(stream)
    _check(lib.pariskv_import(buf.ctypes.data, buf.nbytes, capacity, st, ctypes.byref(h)),
           "pariskv_import")
    o = 16 + ctypes.sizeof(Config)              # header: magic, version, size, config, n
    cfg = Config.from_buffer_copy(bytes(buf[16:o]))
    cfg.capacity = capacity if capacity else max(1, int(np.frombuffer(bytes(buf[o:o + 8]),
                                                                      np.int64)[0]))
    if cfg.levels == LEVELS_PRIOR:              # imported with the levels it was coded with
        cfg.levels = LEVELS_TABLE
    return Index(h.value, cfg)


def train_centroids(cfg: Config, signs, keys, iters: int, n: Optional[int] = None, stream=None):
    """pariskv_train_centroids: spherical k-means centroids [units, 16, 256, 8] (fp32, on the
    keys' device) from the first n keys of every (sequence, KV head)."""
    import torch
    n = keys.shape[-2] if n is None else n
    units = cfg.batch * cfg.num_kv_heads
    out = torch.empty((units, 16, 256, 8), dtype=torch.float32, device=keys.device)
    sa, sp = _signs_ptr(signs)
    _check(lib.pariskv_train_centroids(ctypes.byref(cfg), sp, keys.data_ptr(), _slab(keys), n,
                                       int(iters), out.data_ptr(), _stream(stream)),
           "pariskv_train_centroids")
    return out


def build_index_rotated(cfg: Config, signs, y, knorm, n: Optional[int] = None,
                        stream=None) -> Index:
    n = y.shape[-2] if n is None else n
    sa, sp = _signs_ptr(signs)
    h = _P()
    _check(lib.pariskv_debug_build_index_rotated(ctypes.byref(cfg), sp, y.data_ptr(),
                                                 knorm.data_ptr(), _slab(y), n, _stream(stream),
                                                 ctypes.byref(h)),
           "pariskv_debug_build_index_rotated")
    return Index(h.value, cfg)


def rotate(cfg: Config, signs, x, stream=None):
    import torch
    n = x.numel() // 128
    y = torch.empty((n, 128), dtype=torch.float32, device=x.device)
    nr = torch.empty((n,), dtype=torch.float32, device=x.device)
    sa, sp = _signs_ptr(signs)
    _check(lib.pariskv_debug_rotate(ctypes.byref(cfg), sp, x.data_ptr(), n, y.data_ptr(),
                                    nr.data_ptr(), _stream(stream)), "pariskv_debug_rotate")
    return y, nr


def check_guards() -> None:
    """pariskv_debug_check_guards: the guard bytes around every live index buffer are intact
    (requires PARISKV_GUARD=1 in the environment before the first index is created)."""
    _check(lib.pariskv_debug_check_guards(), "pariskv_debug_check_guards")


def union_rows() -> int:
    """pariskv_debug_union_rows: K/V rows the GQA-group union attention fetched since the
    last call (current device)."""
    r = _I64(0)
    _check(lib.pariskv_debug_union_rows(ctypes.byref(r)), "pariskv_debug_union_rows")
    return int(r.value)


def sparse_attend(cfg: Config, q, K, V, topk_idx, k: int, scale: float, n: Optional[int] = None,
                  out=None, out_dtype=None, stream=None):
    """q [batch, Hq, d]; K, V [batch, Hkv, L, d] (device or pinned host); topk [batch*Hq, k].
    out_dtype: torch.float32 (fp32 accumulator precision) or torch.bfloat16; defaults to the
    dtype of ``out`` when given, else to q's dtype."""
    import torch
    n = K.shape[-2] if n is None else n
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
    od = BF16 if out.dtype == torch.bfloat16 else F32
    _check(lib.pariskv_sparse_attend(ctypes.byref(cfg), q.data_ptr(), K.data_ptr(), V.data_ptr(),
                                     _slab(K), n, topk_idx.data_ptr(), k, float(scale),
                                     out.data_ptr(), od, _stream(stream)), "pariskv_sparse_attend")
    return out


def sparse_attend_noalloc(cfg: Config, q, K, V, topk_idx, k: int, scale: float,
                          n: Optional[int] = None, out=None, out_dtype=None, stream=None):
    """pariskv_sparse_attend_noalloc: the attention above with its partials in the library's
    fixed device workspace instead of a per-call allocation (``out`` is still the caller's)."""
    import torch
    n = K.shape[-2] if n is None else n
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
    od = BF16 if out.dtype == torch.bfloat16 else F32
    _check(lib.pariskv_sparse_attend_noalloc(ctypes.byref(cfg), q.data_ptr(), K.data_ptr(),
                                             V.data_ptr(), _slab(K), n, topk_idx.data_ptr(), k,
                                             float(scale), out.data_ptr(), od, _stream(stream)),
           "pariskv_sparse_attend_noalloc")
    return out


def dense_attend(cfg: Config, q, K, V, scale: float, n: Optional[int] = None, out=None,
                 out_dtype=None, stream=None):
    """pariskv_dense_attend: softmax attention over all n tokens (bf16 q, K, V; K/V
    [batch, Hkv, L, d]); the full-attention baseline."""
    import torch
    n = K.shape[-2] if n is None else n
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
    od = BF16 if out.dtype == torch.bfloat16 else F32
    _check(lib.pariskv_dense_attend(ctypes.byref(cfg), q.data_ptr(), K.data_ptr(), V.data_ptr(),
                                    _slab(K), n, float(scale), out.data_ptr(), od,
                                    _stream(stream)), "pariskv_dense_attend")
    return out


def last_launch_count() -> int:
    return int(lib.pariskv_last_launch_count())


def read_stream(src, nbytes: int, sink, stream=None) -> None:
    """pariskv_debug_read_stream: one coalesced pass over nbytes of ``src`` (a device tensor
    or a pinned host tensor); ``sink`` is a device tensor of at least 4 bytes."""
    _check(lib.pariskv_debug_read_stream(src.data_ptr(), int(nbytes), sink.data_ptr(),
                                         _stream(stream)), "pariskv_debug_read_stream")


class Cache:
    """Owner of a ``pariskv_cache*`` (include/pariskv_cache.h): Sink, Local and Update Buffer
    on the GPU, the Retrieval zone in pinned host memory behind a ParisKV index."""

    REGIONS = ("sink", "local", "buffer", "retrieval")

    def __init__(self, cfg: Config, signs, n_sink: int, n_local: int, n_buffer: int, k: int,
                 retrieval_capacity: int, stream=None):
        self.cfg = cfg
        self.cc = CacheConfig(n_sink, n_local, n_buffer, k, retrieval_capacity)
        sa, sp = _signs_ptr(signs)
        h = _P()
        self.handle = ctypes.c_void_p(0)
        _check(lib.pariskv_cache_create(ctypes.byref(cfg), ctypes.byref(self.cc), sp,
                                        _stream(stream), ctypes.byref(h)),
               "pariskv_cache_create")
        self.handle = ctypes.c_void_p(h.value)

    def prefill(self, K, V, n: Optional[int] = None, stream=None) -> None:
        """K, V: [batch, num_kv_heads, L, d] (device or pinned host); n <= L tokens used."""
        n = K.shape[-2] if n is None else n
        assert _slab(K) == _slab(V)
        _check(lib.pariskv_cache_prefill(self.handle, K.data_ptr(), V.data_ptr(), _slab(K), n,
                                         _stream(stream)), "pariskv_cache_prefill")

    def step(self, q, k_new, v_new, scale: float, out=None, out_dtype=None,
             topk_idx=None, want_topk: bool = False, stream=None):
        """q [batch, Hq, d]; k_new, v_new [batch, Hkv, d] (device). Returns (out, topk_idx)."""
        import torch
        if out is None:
            out = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
        if topk_idx is None and want_topk:
            topk_idx = torch.empty((self.cfg.batch * self.cfg.num_q_heads, self.cc.k),
                                   dtype=torch.int32, device=q.device)
        od = BF16 if out.dtype == torch.bfloat16 else F32
        _check(lib.pariskv_cache_step(self.handle, q.data_ptr(), k_new.data_ptr(),
                                      v_new.data_ptr(), float(scale), out.data_ptr(), od,
                                      topk_idx.data_ptr() if topk_idx is not None else None,
                                      _stream(stream)), "pariskv_cache_step")
        return out, topk_idx

    def counts(self) -> dict:
        c = (_I64 * 4)()
        _check(lib.pariskv_cache_counts(self.handle, c), "pariskv_cache_counts")
        return dict(zip(self.REGIONS, (int(x) for x in c)))

    def index(self) -> Index:
        """A non-owning view of the Retrieval zone's index."""
        cfg = Config.from_buffer_copy(self.cfg)
        cfg.capacity = self.cc.retrieval_capacity
        return Index(lib.pariskv_cache_index(self.handle), cfg, owned=False)

    def destroy(self) -> None:
        if self.handle:
            lib.pariskv_cache_destroy(self.handle)
            self.handle = ctypes.c_void_p(0)

    def __del__(self):
        try:
            self.destroy()
        except Exception:
            pass
