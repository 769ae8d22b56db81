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


def _run(name, sample_units, sample_heads=None):
    sp = workload.spec(name)
    d = workload.generate_torch(sp, DEV)
    signs = d["signs"].numpy()
    units, G, n = sp.batch * sp.num_kv_heads, sp.group, sp.n
    cfg = pk.config(batch=sp.batch, num_kv_heads=sp.num_kv_heads, group=G, capacity=n,
                    dtype=sp.dtype, rho=sp.rho, cand_bp=sp.cand_bp)
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
                                             qn[u * G:(u + 1) * G][list(heads)], k, p)
        for g, o in zip(heads, outs):
            h = u * G + g
            np.testing.assert_array_equal(gsc[h], o["scores"])
            np.testing.assert_array_equal(gcand[h], o["cand"])
            np.testing.assert_array_equal(gS[h].view(np.uint32), o["S"].view(np.uint32))
            np.testing.assert_array_equal(gidx[h], o["idx"])
            np.testing.assert_array_equal(gest[h].view(np.uint32), o["est"].view(np.uint32))
    del ix, y, kn
    # end to end from raw inputs on one sampled unit (the library rotates keys and queries)
    ixr = pk.build_index(cfg, signs, d["keys"])
    ridx, _ = ixr.search(d["queries"], k)
    ixr.sync()
    ridx = ridx.cpu().numpy()
    u = sample_units[0]
    enc = oracle.encode_rotated(host[u][0], host[u][1], 8)   # the oracle's index of unit u
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
