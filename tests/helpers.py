"""Shared test helpers: oracle-side references for whole (sequence, KV head) units and small
input builders. Nothing here computes the method itself; the oracle package does."""
from __future__ import annotations

import numpy as np

import oracle


def oracle_unit_from_rotated(y, kn, qts, qns, k, p: oracle.SearchParams, table=None):
    """Oracle stages for one unit from rotated inputs: y [n, d], kn [n]; qts [G, d]; table:
    the magnitude levels of table-coded keys (None: uniform levels)."""
    enc = oracle.encode_rotated(y, kn, p.m, table=table)
    out = []
    for qt, qn in zip(qts, qns):
        lut = oracle.query_lut(qt, p.m, p.rho, p.w_rank1, p.w_rest)
        sc = oracle.vote(enc.ids, lut, p.m)
        C = oracle.candidate_count(y.shape[0], k, p.cand_bp)
        cand = oracle.select_candidates(sc, C)
        S = oracle.rerank(enc, cand, qt, p.m)
        idx, s_top = oracle.topk(S, cand, k)
        est = (np.float32(qn) * s_top).astype(np.float32)
        out.append(dict(lut=lut, scores=sc, cand=cand, S=S, idx=idx, est=est))
    return enc, out


def rotate_all(x, signs):
    """Oracle rotation of [..., n, d] -> (y [..., n, d] f32, norm [..., n] f32)."""
    shp = x.shape
    y, nr = oracle.normalize_rotate(x.reshape(-1, shp[-1]), signs)
    return y.reshape(shp), nr.reshape(shp[:-1])


def recall(a, b) -> float:
    a, b = set(np.asarray(a).tolist()), set(np.asarray(b).tolist())
    return len(a & b) / max(1, len(b))


def random_signs(seed=0, d=128):
    return np.where(np.random.default_rng(seed).integers(0, 2, d) == 1, -1, 1).astype(np.int8)
