"""Parity at the full workload sizes, in the launch configuration the benchmark times.

The index covers every (sequence, KV head) unit of the workload. Sampled units are built
from the oracle's rotated fp32 keys and searched with the oracle's rotated queries, and their
candidates, rerank values, top-k indices and estimates are compared bit for bit with the
oracle; the remaining units are filled with the library's own rotation of their keys so that
every kernel runs at full size. End-to-end recall from raw inputs is checked on the sampled
units too. Inputs come from the workload generator's device backend."""
import numpy as np
import pytest
import torch

import oracle
from long_context_kv_srht_b200 import pariskv as pk
from long_context_kv_srht_b200 import workload
from helpers import oracle_unit_from_rotated

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _run(name, sample_units, sample_heads=None, table=None):
    """table: code with the oracle's prior-derived levels (given to the library as a table for
    the bit-exact part; the end-to-end part uses the library's own prior levels)."""
    sp = workload.spec(name)
    d = workload.generate_torch(sp, DEV)
    signs = d["signs"].numpy()
    units, G, n = sp.batch * sp.num_kv_heads, sp.group, sp.n
    lv = {} if table is None else {"levels": "table", "level_table": table}
    cfg = pk.config(batch=sp.batch, num_kv_heads=sp.num_kv_heads, group=G, capacity=n,
                    dtype=sp.dtype, rho=sp.rho, cand_bp=sp.cand_bp, **lv)
    keys = d["keys"].reshape(units, n, 128)
    y, kn = pk.rotate(cfg, signs, keys)
    y = y.reshape(units, n, 128)
    kn = kn.reshape(units, n)
    q_host = d["queries"].float().cpu().numpy().reshape(units * G, 128)
    qt, qn = oracle.normalize_rotate(q_host, signs)
    host = {}
    for u in sample_units:
        yo, no = oracle.normalize_rotate(keys[u].float().cpu().numpy(), signs)
        host[u] = (yo, no)
        y[u].copy_(torch.from_numpy(yo))
        kn[u].copy_(torch.from_numpy(no))
    ix = pk.build_index_rotated(cfg, signs, y, kn)
    k = sp.k
    idx, est = ix.search_rotated(torch.from_numpy(qt).to(DEV), torch.from_numpy(qn).to(DEV), k)
    ix.sync()                                   # device-side consistency flags must be clear
    glut, gsc, gcand, gS = ix.export_search()
    gidx, gest = idx.cpu().numpy(), est.cpu().numpy()
    p = oracle.SearchParams(m=8, rho=sp.rho, cand_bp=sp.cand_bp)
    for u in sample_units:
        yo, no = host[u]
        heads = range(G) if sample_heads is None else sample_heads
        enc, outs = oracle_unit_from_rotated(yo, no, qt[u * G:(u + 1) * G][list(heads)],
                                             qn[u * G:(u + 1) * G][list(heads)], k, p,
                                             table=table)
        for g, o in zip(heads, outs):
            h = u * G + g
            np.testing.assert_array_equal(gsc[h], o["scores"])
            np.testing.assert_array_equal(gcand[h], o["cand"])
            np.testing.assert_array_equal(gS[h].view(np.uint32), o["S"].view(np.uint32))
            np.testing.assert_array_equal(gidx[h], o["idx"])
            np.testing.assert_array_equal(gest[h].view(np.uint32), o["est"].view(np.uint32))
    del ix, y, kn
    # end to end from raw inputs on one sampled unit (the library rotates keys and queries)
    if table is not None:
        cfg.levels = pk.LEVELS_PRIOR
    ixr = pk.build_index(cfg, signs, d["keys"])
    ridx, _ = ixr.search(d["queries"], k)
    ixr.sync()
    ridx = ridx.cpu().numpy()
    u = sample_units[0]
    enc = oracle.encode_rotated(host[u][0], host[u][1], 8, table=table)   # oracle index of u
    hits = 0
    for g in range(G):
        o_idx, *_ = oracle.search(enc, q_host[u * G + g], signs, k, p)
        hits += len(set(o_idx.tolist()) & set(ridx[u * G + g].tolist()))
    assert hits / (G * k) >= 0.999, hits / (G * k)


def test_llama3_8b_128k_full_size():
    _run("llama3_8b_128k", sample_units=[0, 7])


def test_batched_64k_full_size():
    _run("batched_64k", sample_units=[0, 77], sample_heads=[0, 3])


def test_million_offload_full_size():
    _run("million_offload", sample_units=[3], sample_heads=[0, 2])


def test_llama3_8b_128k_full_size_prior_levels():
    _run("llama3_8b_128k", sample_units=[0, 5], table=oracle.ratio_levels())


def test_levels_against_exact_inner_products():
    """Uniform levels against the rotation prior's levels at the llama3_8b_128k size, measured
    against exact inner products (fp32, torch on the device):
      - recall of the top-k against the exact top-k over all keys (bounded by the vote's
        pruning, which the levels do not touch);
      - recall against the exact top-k among each head's candidates (the rerank's own
        accuracy, which the levels decide);
      - the estimator's relative RMS error ||q|| S - <k, q> over the candidates.
    The figures are printed for the record; the prior's levels must estimate more accurately
    and rank candidates at least as well (within sampling noise)."""
    sp = workload.spec("llama3_8b_128k")
    d = workload.generate_torch(sp, DEV)
    signs = d["signs"].numpy()
    units, G, n, k = sp.batch * sp.num_kv_heads, sp.group, sp.n, sp.k
    keys = d["keys"].reshape(units, n, 128).float()
    q = d["queries"].reshape(units, G, 128).float()
    dots = torch.einsum("ugd,und->ugn", q, keys).reshape(units * G, n)
    exact = torch.topk(dots, k, dim=-1).indices.cpu().numpy()
    qnorm = q.reshape(units * G, 128).norm(dim=-1)
    out = {}
    for levels in ("uniform", "prior"):
        cfg = pk.config(batch=sp.batch, num_kv_heads=sp.num_kv_heads, group=G, capacity=n,
                        dtype=sp.dtype, rho=sp.rho, cand_bp=sp.cand_bp, levels=levels)
        ix = pk.build_index(cfg, signs, d["keys"])
        idx, _ = ix.search(d["queries"], k)
        got = idx.cpu().numpy()
        _, _, cand, S = ix.export_search()
        ct = torch.from_numpy(cand.astype(np.int64)).to(DEV)
        cd = torch.gather(dots, 1, ct)                              # exact <k, q> of candidates
        est = qnorm[:, None] * torch.from_numpy(S).to(DEV)
        err = float(torch.sqrt(((est - cd) ** 2).mean() / (cd ** 2).mean()))
        inner = torch.gather(ct, 1, torch.topk(cd, k, dim=-1).indices).cpu().numpy()
        H = units * G
        rec = np.mean([len(set(got[h].tolist()) & set(exact[h].tolist())) / k for h in range(H)])
        rrec = np.mean([len(set(got[h].tolist()) & set(inner[h].tolist())) / k for h in range(H)])
        out[levels] = {"recall": float(rec), "rerank_recall": float(rrec), "est_rel_rms": err}
        ix.destroy()
    print("levels vs exact inner products:", out)
    assert out["prior"]["est_rel_rms"] < out["uniform"]["est_rel_rms"], out
    assert out["prior"]["rerank_recall"] > out["uniform"]["rerank_recall"] - 0.002, out
    assert abs(out["prior"]["recall"] - out["uniform"]["recall"]) < 0.01, out
