"""Plain CPU oracle for the ParisKV KV-cache retrieval path.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline leg are the only callers allowed. The product path never imports this package,
and this package imports nothing from the product package.

The arithmetic lives in ``pariskv_oracle.c`` (plain C, built with ``-ffp-contract=off`` and
no fast-math). This module only compiles it, marshals numpy arrays to it, and composes the
per-step pipeline in the order the method states it:

  normalise + rotate -> bucket ids, RSQ codes, calibration factors (keys)
  normalise + rotate -> top-rho centroid lookup table (query)
  collision vote -> candidate pruning -> RSQ-IP rerank -> top-k -> sparse attention.

Sources: "Technical Summary: ParisKV" (gist.science/paper/2602.07721), Methodology and
System-Level Innovations; "ParisKV: Fast and Drift-Robust KV-Cache Retrieval for
Long-Context LLMs" (ICML 2026 poster abstract).

Parity status: every function here is pinned by tests in ``tests/test_oracle_pins.py``.
Two readings the pages leave open are pinned only to their stated definitions and to the
invariants and laws they imply, not to values the pages print (parity unpinned against the
pages for these two): the exact definition of the calibration weight w_{i,b}, and the rule
that turns the pages' "Beta priors" into magnitude levels (uniform levels, the default, and
the prior-derived table levels of ``ratio_levels``; the law behind the latter is pinned
against rotated keys and its Lloyd-Max conditions by independent quadrature).
"""
from __future__ import annotations

import ctypes
import functools
import os
import subprocess
import threading
from dataclasses import dataclass
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pariskv_oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "liboracle.so")
_lock = threading.Lock()
_lib = None

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
          "-fopenmp", "-Wall"]


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/_build/liboracle.so`` (skipped when up to date)."""
    os.makedirs(_LIB_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    subprocess.run(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"], check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            i32, i64 = ctypes.c_int32, ctypes.c_int64
            lib.orc_num_threads.restype = i32
            lib.orc_set_num_threads.argtypes = [i32]
            lib.orc_rotate_f64.argtypes = [i32, P, P, P]
            lib.orc_normalize_rotate.argtypes = [i32, P, P, i64, P, P]
            lib.orc_encode_rotated.argtypes = [i32, i32, i32, P, P, i64, P, P, P, P]
            lib.orc_query_lut.argtypes = [i32, i32, i32, i32, i32, P, P]
            lib.orc_vote.argtypes = [i32, i32, P, i64, P, P]
            lib.orc_candidate_count.argtypes = [i64, i64, i32]
            lib.orc_candidate_count.restype = i64
            lib.orc_select_candidates.argtypes = [P, i64, i64, P]
            lib.orc_rerank.argtypes = [i32, i32, P, P, P, P, i64, P, P]
            lib.orc_encode_rotated_table.argtypes = [i32, i32, P, P, P, i64, P, P, P, P]
            lib.orc_rerank_table.argtypes = [i32, i32, P, P, P, P, P, i64, P, P]
            lib.orc_learned_ids.argtypes = [i32, i32, P, P, i64, P]
            lib.orc_learned_lut.argtypes = [i32, i32, i32, i32, i32, P, P, P]
            lib.orc_topk.argtypes = [P, P, i64, i64, P, P]
            lib.orc_attend.argtypes = [i32, P, P, P, P, i64, ctypes.c_double, P]
            _lib = lib
    return _lib


def _p(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def num_threads() -> int:
    return int(_load().orc_num_threads())


def set_num_threads(t: int) -> None:
    _load().orc_set_num_threads(int(t))


# ---------------------------------------------------------------------------------------
# Single steps (canonical layouts; see pariskv_oracle.c for each definition)
# ---------------------------------------------------------------------------------------
def rotate_f64(x: np.ndarray, signs: np.ndarray) -> np.ndarray:
    """y = (1/sqrt(d)) H diag(s) x in fp64 (explicit product)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    s = np.ascontiguousarray(signs, dtype=np.int8)
    y = np.empty_like(x)
    _load().orc_rotate_f64(x.shape[0], _p(s), _p(x), _p(y))
    return y


def normalize_rotate(x: np.ndarray, signs: np.ndarray):
    """Rows of x [n, d] -> (y f32 [n, d], norm f32 [n]); fp64 inside, rounded to fp32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    n, d = x.shape
    s = np.ascontiguousarray(signs, dtype=np.int8)
    y = np.empty((n, d), np.float32)
    nr = np.empty((n,), np.float32)
    _load().orc_normalize_rotate(d, _p(s), _p(x), n, _p(y), _p(nr))
    return y, nr


@dataclass
class Encoded:
    """Oracle index of one (sequence, KV head): canonical layouts."""
    ids: np.ndarray      # u8  [n, B]
    mag: np.ndarray      # i32 [n, d]
    neg: np.ndarray      # u8  [n, d]
    factor: np.ndarray   # f32 [n, B]
    table: Optional[np.ndarray] = None   # f32 [8] magnitude levels; None: uniform integers

    @property
    def codes(self) -> np.ndarray:
        """4-bit RSQ codes [n, d]: sign bit in bit 3, magnitude in bits 0..2."""
        assert int(self.mag.max(initial=0)) <= 7, "4-bit codes need levels == 7"
        return ((self.neg.astype(np.uint8) << 3) | self.mag.astype(np.uint8)).astype(np.uint8)

    @property
    def vt(self) -> np.ndarray:
        """Dequantised vectors (sign applied) as f64 [n, d]: the integer levels, or the table's
        levels for table-coded keys."""
        if self.table is not None:
            v = self.table.astype(np.float64)[self.mag]
            return np.where(self.neg != 0, -v, v)
        return np.where(self.neg != 0, -self.mag, self.mag).astype(np.float64)


def encode_rotated(y: np.ndarray, norm: np.ndarray, m: int, levels: int = 7,
                   table: Optional[np.ndarray] = None) -> Encoded:
    """Uniform integer levels 0..levels (R5), or, with `table` (8 ascending fp32 magnitudes),
    the table-level codes of R24."""
    y = np.ascontiguousarray(y, dtype=np.float32)
    nr = np.ascontiguousarray(norm, dtype=np.float32)
    n, d = y.shape
    B = d // m
    ids = np.empty((n, B), np.uint8)
    mag = np.empty((n, d), np.int32)
    neg = np.empty((n, d), np.uint8)
    fac = np.empty((n, B), np.float32)
    if table is not None:
        table = np.ascontiguousarray(table, dtype=np.float32)
        assert table.shape == (8,) and np.all(np.diff(table) > 0)
        _load().orc_encode_rotated_table(d, m, _p(table), _p(y), _p(nr), n, _p(ids), _p(mag),
                                         _p(neg), _p(fac))
        return Encoded(ids, mag, neg, fac, table)
    _load().orc_encode_rotated(d, m, levels, _p(y), _p(nr), n, _p(ids), _p(mag), _p(neg),
                               _p(fac))
    return Encoded(ids, mag, neg, fac)


def query_lut(qt: np.ndarray, m: int, rho: int, w_rank1: int = 2, w_rest: int = 1) -> np.ndarray:
    """Rotated query [d] -> vote lookup table u8 [B, 2^m]."""
    qt = np.ascontiguousarray(qt, dtype=np.float32)
    d = qt.shape[0]
    lut = np.empty((d // m, 1 << m), np.uint8)
    _load().orc_query_lut(d, m, rho, w_rank1, w_rest, _p(qt), _p(lut))
    return lut


def vote(ids: np.ndarray, lut: np.ndarray, m: int) -> np.ndarray:
    ids = np.ascontiguousarray(ids, dtype=np.uint8)
    lut = np.ascontiguousarray(lut, dtype=np.uint8)
    n, B = ids.shape
    sc = np.empty((n,), np.int32)
    _load().orc_vote(B, m, _p(ids), n, _p(lut), _p(sc))
    return sc


def candidate_count(n: int, k: int, bp: int) -> int:
    return int(_load().orc_candidate_count(n, k, bp))


def select_candidates(score: np.ndarray, C: int) -> np.ndarray:
    score = np.ascontiguousarray(score, dtype=np.int32)
    cand = np.empty((C,), np.int32)
    _load().orc_select_candidates(_p(score), score.shape[0], C, _p(cand))
    return cand


def rerank(enc: Encoded, cand: np.ndarray, qt: np.ndarray, m: int) -> np.ndarray:
    cand = np.ascontiguousarray(cand, dtype=np.int32)
    qt = np.ascontiguousarray(qt, dtype=np.float32)
    d = qt.shape[0]
    S = np.empty((cand.shape[0],), np.float32)
    if enc.table is not None:
        _load().orc_rerank_table(d, m, _p(enc.table), _p(enc.mag), _p(enc.neg), _p(enc.factor),
                                 _p(cand), cand.shape[0], _p(qt), _p(S))
        return S
    _load().orc_rerank(d, m, _p(enc.mag), _p(enc.neg), _p(enc.factor), _p(cand),
                       cand.shape[0], _p(qt), _p(S))
    return S


def topk(S: np.ndarray, cand: np.ndarray, k: int):
    S = np.ascontiguousarray(S, dtype=np.float32)
    cand = np.ascontiguousarray(cand, dtype=np.int32)
    kk = min(k, S.shape[0])
    idx = np.empty((kk,), np.int32)
    so = np.empty((kk,), np.float32)
    _load().orc_topk(_p(S), _p(cand), S.shape[0], kk, _p(idx), _p(so))
    return idx, so


def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, idx: np.ndarray, scale: float) -> np.ndarray:
    """Sparse softmax attention over rows idx of K/V [n, d] (fp64 result)."""
    q = np.ascontiguousarray(q, dtype=np.float32)
    K = np.ascontiguousarray(K, dtype=np.float32)
    V = np.ascontiguousarray(V, dtype=np.float32)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    out = np.empty((q.shape[0],), np.float64)
    _load().orc_attend(q.shape[0], _p(q), _p(K), _p(V), _p(idx), idx.shape[0], float(scale),
                       _p(out))
    return out


# ---------------------------------------------------------------------------------------
# Composed pipeline for one (sequence, KV head) and its group of query heads
# ---------------------------------------------------------------------------------------
@dataclass
class SearchParams:
    m: int = 8
    rho: int = 4
    w_rank1: int = 2
    w_rest: int = 1
    cand_bp: int = 500
    centroids: Optional[np.ndarray] = None   # learned centroids [B, 256, m] (R25), or analytic


def build_unit(keys: np.ndarray, signs: np.ndarray, m: int,
               table: Optional[np.ndarray] = None) -> Encoded:
    """Index of one (sequence, KV head): keys [n, d] -> Encoded (table: R24 levels)."""
    y, nr = normalize_rotate(keys, signs)
    return encode_rotated(y, nr, m, table=table)


def search_rotated(enc: Encoded, qt: np.ndarray, qnorm: float, k: int, p: SearchParams):
    """One query head from its rotated query: returns (topk idx, S, est, candidates, scores).
    With p.centroids the coarse stage uses the learned centroids (enc.ids must be learned
    ids, from learned_ids)."""
    n = enc.ids.shape[0]
    lut = (query_lut(qt, p.m, p.rho, p.w_rank1, p.w_rest) if p.centroids is None else
           learned_lut(qt, p.centroids, p.m, p.rho, p.w_rank1, p.w_rest))
    sc = vote(enc.ids, lut, p.m)
    C = candidate_count(n, k, p.cand_bp)
    cand = select_candidates(sc, C)
    S = rerank(enc, cand, qt, p.m)
    idx, s_top = topk(S, cand, k)
    est = (np.float32(qnorm) * s_top).astype(np.float32)
    return idx, s_top, est, cand, sc


def search(enc: Encoded, q: np.ndarray, signs: np.ndarray, k: int, p: SearchParams):
    """One query head from its raw query vector [d]."""
    qt, qn = normalize_rotate(q[None, :], signs)
    return search_rotated(enc, qt[0], float(qn[0]), k, p)


# ---------------------------------------------------------------------------------------
# Four-region KV cache ("Technical Summary: ParisKV", System-Level Innovations 2,
# "Sliding-Window Update Mechanism"): Sink and Local stay on the GPU, older tokens go to
# the Retrieval zone, new tokens collect in an Update Buffer; a full buffer evicts the oldest
# Local tokens to Retrieval and joins Local. Token positions are tracked as plain lists.
# Readings where the page is silent: a token enters Sink while Sink is short, else the
# buffer; a promotion evicts the max(0, |Local| + |buffer| - n_local) oldest Local tokens;
# prefill fills Sink first, then the last n_local tokens go to Local and the rest between
# the two to Retrieval.
# ---------------------------------------------------------------------------------------
class CacheRegions:
    def __init__(self, n_sink: int, n_local: int, n_buffer: int):
        assert n_sink >= 0 and 1 <= n_buffer <= n_local
        self.n_sink, self.n_local, self.n_buffer = n_sink, n_local, n_buffer
        self.sink, self.local, self.buffer, self.retrieval = [], [], [], []
        self.total = 0

    def prefill(self, n: int) -> None:
        assert self.total == 0
        toks = list(range(n))
        self.sink = toks[: self.n_sink]
        rest = toks[self.n_sink:]
        n_loc = min(len(rest), self.n_local)
        self.local = rest[len(rest) - n_loc:]
        self.retrieval = rest[: len(rest) - n_loc]
        self.total = n

    def append(self) -> None:
        t = self.total
        self.total += 1
        if len(self.sink) < self.n_sink:
            self.sink.append(t)
            return
        self.buffer.append(t)
        if len(self.buffer) == self.n_buffer:
            drop = max(0, len(self.local) + len(self.buffer) - self.n_local)
            self.retrieval += self.local[:drop]
            self.local = self.local[drop:] + self.buffer
            self.buffer = []

    def dense(self) -> list:
        """Tokens every step attends to exactly: Sink, Local and buffer."""
        return self.sink + self.local + self.buffer


def cache_step_attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, regions: CacheRegions,
                      enc: Encoded, signs: np.ndarray, k: int, scale: float, p: SearchParams):
    """One decode step's attention for one query head: a ParisKV search over the Retrieval
    zone's index (enc holds the Retrieval tokens in order), then one softmax over the dense
    tokens plus the retrieved ones. K, V: [total, d] indexed by token position. Returns
    (out, retrieved Retrieval rows)."""
    rows = np.empty((0,), np.int32)
    if regions.retrieval:
        rows, *_ = search(enc, q, signs, min(k, len(regions.retrieval)), p)
    toks = np.asarray(regions.dense() + [regions.retrieval[r] for r in rows], np.int32)
    return attend(q, K, V, toks, scale), rows


# ---------------------------------------------------------------------------------------
# Magnitude levels from the rotation prior ("Technical Summary: ParisKV", Core Algorithmic
# Innovations 2, "Quantization": the 3-bit magnitude is derived from rotation-induced Beta
# priors).
# After the random rotation the direction of a subspace y_b is uniform on the sphere of
# R^m, so each coordinate has u_j^2 ~ Beta(1/2, (m-1)/2); equivalently u = g / |g| with g
# i.i.d. standard normal. The codes quantise r_j = |y_j| / max_i |y_i|, which does not depend
# on |g|: r has the law of |g_j| / max_i |g_i| for i.i.d. half-normals. With psi the
# half-normal density and Psi its CDF (erf(t / sqrt 2)), r has mass 1/m at 1 (the maximal
# coordinate) and on [0, 1) the density
#     f(x) = (m - 1) * integral_0^inf psi(t) psi(x t) t Psi(t)^(m-2) dt.
# The levels are the 8-level Lloyd-Max quantiser of that law (nearest-level cells,
# conditional-mean levels), reading R24.
# ---------------------------------------------------------------------------------------
def ratio_density(x: np.ndarray, m: int = 8, t_max: float = 9.0, nt: int = 4096) -> np.ndarray:
    """f(x) above on [0, 1) by the midpoint rule in t (the integrand is below 1e-17 past
    t = 9)."""
    from scipy.special import erf
    t = (np.arange(nt) + 0.5) * (t_max / nt)
    psi = np.sqrt(2.0 / np.pi) * np.exp(-0.5 * t * t)
    Psi = erf(t / np.sqrt(2.0))
    w = psi * t * Psi ** (m - 2) * (t_max / nt)
    xt = np.outer(np.asarray(x, dtype=np.float64), t)
    return (m - 1) * (np.sqrt(2.0 / np.pi) * np.exp(-0.5 * xt * xt)) @ w


@functools.lru_cache(maxsize=4)
def ratio_levels(m: int = 8, nx: int = 16384, iters: int = 2000) -> np.ndarray:
    """The 8 Lloyd-Max levels (ascending, fp32) of r = |y_j| / max_i |y_i| (reading R24).
    Cell masses and first moments come from the cumulative integrals of f (trapezoid rule on
    nx + 1 points), interpolated at the thresholds, so that cells are not snapped to a grid."""
    x = np.linspace(0.0, 1.0, nx + 1)
    f = ratio_density(x, m)
    h = 1.0 / nx
    F0 = np.concatenate([[0.0], np.cumsum(0.5 * h * (f[1:] + f[:-1]))])
    xf = x * f
    F1 = np.concatenate([[0.0], np.cumsum(0.5 * h * (xf[1:] + xf[:-1]))])
    pm = 1.0 / m                                # point mass at r = 1
    lv = (np.arange(8) + 0.5) / 8
    for _ in range(iters):
        edges = np.concatenate([[0.0], 0.5 * (lv[:-1] + lv[1:]), [1.0]])
        c0 = np.interp(edges, x, F0)
        c1 = np.interp(edges, x, F1)
        s0 = np.diff(c0)
        s1 = np.diff(c1)
        s0[7] += pm                             # r = 1 always falls in the top cell
        s1[7] += pm
        lv = s1 / s0
    return lv.astype(np.float32)


# ---------------------------------------------------------------------------------------
# Learned centroids: the comparator of the drift claim (reading R25; see pariskv_oracle.c)
# ---------------------------------------------------------------------------------------
def learned_ids(y: np.ndarray, cent: np.ndarray, m: int = 8) -> np.ndarray:
    """ids [n, B]: argmax_c <y_b, mu_c> per subspace (fp32 chains, ties to the lower c)."""
    y = np.ascontiguousarray(y, dtype=np.float32)
    cent = np.ascontiguousarray(cent, dtype=np.float32)
    n, d = y.shape
    ids = np.empty((n, d // m), np.uint8)
    _load().orc_learned_ids(d, m, _p(cent), _p(y), n, _p(ids))
    return ids


def learned_lut(qt: np.ndarray, cent: np.ndarray, m: int = 8, rho: int = 4, w_rank1: int = 2,
                w_rest: int = 1) -> np.ndarray:
    """Vote table [B, 256] from the rho centroids with the largest <q~_b, mu_c>."""
    qt = np.ascontiguousarray(qt, dtype=np.float32)
    cent = np.ascontiguousarray(cent, dtype=np.float32)
    lut = np.empty((qt.shape[0] // m, 1 << m), np.uint8)
    _load().orc_learned_lut(qt.shape[0], m, rho, w_rank1, w_rest, _p(cent), _p(qt), _p(lut))
    return lut


def train_centroids(y: np.ndarray, iters: int, m: int = 8) -> np.ndarray:
    """Spherical k-means (Lloyd) per subspace on the prefill keys' rotated directions
    (reading R25): 256 unit-norm centroids; start from the directions of keys
    floor(c n / 256); each iteration assigns every key by learned_ids and replaces each
    centroid by the normalised sum (fp64) of its keys' unit directions (a centroid with no
    key keeps its value). Returns fp32 [B, 256, m]."""
    y = np.ascontiguousarray(y, dtype=np.float32)
    n, d = y.shape
    B = d // m
    yb = y.reshape(n, B, m).astype(np.float64)
    nrm = np.linalg.norm(yb, axis=2, keepdims=True)
    u = np.divide(yb, nrm, out=np.zeros_like(yb), where=nrm > 0)
    cent = u[(np.arange(256) * n) // 256].transpose(1, 0, 2).astype(np.float32)   # [B, 256, m]
    for _ in range(iters):
        ids = learned_ids(y, cent, m)
        new = cent.astype(np.float64).copy()
        for b in range(B):
            sums = np.zeros((256, m))
            np.add.at(sums, ids[:, b], u[:, b])
            norm = np.linalg.norm(sums, axis=1)
            ok = norm > 0
            new[b, ok] = sums[ok] / norm[ok, None]
        cent = new.astype(np.float32)
    return np.ascontiguousarray(cent)


def sign_centroids(m: int = 8) -> np.ndarray:
    """The analytic centroids as a table [B, 256, m]: c's sign pattern / sqrt(m)."""
    c = np.arange(1 << m)
    pat = np.where((c[:, None] >> np.arange(m)) & 1, -1.0, 1.0) / np.sqrt(m)
    return np.ascontiguousarray(np.broadcast_to(pat, (128 // m, 1 << m, m)).astype(np.float32))
