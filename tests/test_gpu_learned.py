"""Learned coarse centroids (include/pariskv_learned.h), the comparator of the drift claim
("Technical Summary: ParisKV", Problem Statement 2 "Decoding Drift", Key Contributions 1),
against the oracle: with the oracle's trained centroids every stage is bit-exact; with the
sign patterns as centroids the learned path is the analytic path; training agrees with the
oracle's (the GPU's atomic sums and fp32 rotation allow last-bit differences)."""
import numpy as np
import pytest
import torch

import oracle
from long_context_kv_srht_b200 import pariskv as pk
from long_context_kv_srht_b200 import workload
from helpers import rotate_all

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _t(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


@pytest.mark.parametrize("hkv,G,n,k,bp", [(2, 4, 20000, 128, 500), (1, 2, 9000, 300, 1000),
                                          (1, 5, 4097, 64, 500)])
def test_learned_stages_bit_exact(hkv, G, n, k, bp):
    sp = workload.spec("tiny", num_kv_heads=hkv, group=G, n=n, dtype="f32", seed=n + 7,
                       planted=min(32, n // (4 * G)))
    w = workload.generate(sp)
    y, kn = rotate_all(w.keys.reshape(hkv, n, 128), w.signs)
    qt, qn = rotate_all(w.queries.reshape(hkv * G, 128), w.signs)
    cents = np.stack([oracle.train_centroids(y[u], 3) for u in range(hkv)])
    cfg = pk.config(batch=1, num_kv_heads=hkv, group=G, capacity=n, dtype="f32", cand_bp=bp)
    ix = pk.build_index_rotated(cfg, w.signs, _t(y[:, :0]), _t(kn[:, :0]), n=0)
    ix.set_centroids(_t(cents))
    ix.append_rotated(_t(y), _t(kn))
    idx, est = ix.search_rotated(_t(qt), _t(qn), k)
    gids, gcodes, gfac = ix.export_index()
    glut, gsc, gcand, gS = ix.export_search()
    gidx, gest = idx.cpu().numpy(), est.cpu().numpy()
    for u in range(hkv):
        enc = oracle.encode_rotated(y[u], kn[u], 8)
        enc.ids = oracle.learned_ids(y[u], cents[u])
        np.testing.assert_array_equal(gids[u], enc.ids)
        nz = (enc.codes & 7) != 0            # the sign of a zero magnitude lives in the id bit
        np.testing.assert_array_equal(gcodes[u][nz], enc.codes[nz])
        np.testing.assert_array_equal(gfac[u].view(np.uint32), enc.factor.view(np.uint32))
        p = oracle.SearchParams(m=8, cand_bp=bp, centroids=cents[u])
        for g in range(G):
            h = u * G + g
            o_idx, o_S, o_est, o_cand, o_sc = oracle.search_rotated(enc, qt[h], float(qn[h]), k, p)
            lut = oracle.learned_lut(qt[h], cents[u])
            packed = glut[h]
            np.testing.assert_array_equal(packed, lut)
            np.testing.assert_array_equal(gsc[h], o_sc)
            np.testing.assert_array_equal(gcand[h], o_cand)
            np.testing.assert_array_equal(gidx[h], o_idx)
            np.testing.assert_array_equal(gest[h].view(np.uint32), o_est.view(np.uint32))


def test_sign_centroids_reproduce_the_analytic_index():
    """Raw bf16 inputs, the GPU's own rotation: an index whose 'learned' centroids are the
    sign patterns / sqrt(8) searches exactly like the analytic index (same top-k indices and
    estimates, same codes and factors)."""
    sp = workload.spec("llama3_8b_128k", n=30000)
    d = workload.generate_torch(sp, DEV)
    signs = d["signs"].numpy()
    units = sp.batch * sp.num_kv_heads
    cfg = pk.config(batch=sp.batch, num_kv_heads=sp.num_kv_heads, group=sp.group,
                    capacity=sp.n, dtype="bf16")
    a = pk.build_index(cfg, signs, d["keys"])
    b = pk.build_index(cfg, signs, d["keys"], n=0)
    sc = np.broadcast_to(oracle.sign_centroids(), (units, 16, 256, 8))
    b.set_centroids(_t(sc))
    b.append(d["keys"])
    ia, ea = a.search(d["queries"], sp.k)
    ib, eb = b.search(d["queries"], sp.k)
    np.testing.assert_array_equal(ia.cpu().numpy(), ib.cpu().numpy())
    np.testing.assert_array_equal(ea.cpu().numpy().view(np.uint32), eb.cpu().numpy().view(np.uint32))
    (ida, ca, fa), (idb, cb, fb) = a.export_index(), b.export_index()
    nz = (ca & 7) != 0          # a zero magnitude's sign is the id bit, absent for learned ids
    np.testing.assert_array_equal(ca & 7, cb & 7)
    np.testing.assert_array_equal(ca[nz], cb[nz])
    np.testing.assert_array_equal(fa.view(np.uint32), fb.view(np.uint32))
    # ids: the fp32 inner products with the sign patterns resolve every sign except in
    # subspaces with coordinates too close to zero for the chain's rounding (a handful in
    # millions, none of which changed the searches above)
    assert (ida != idb).mean() < 1e-5


def test_train_centroids_agrees_with_oracle():
    """The start (directions of fixed keys) within 2e-5; after 5 iterations the fit (mean
    cosine of a key's direction to its centroid) within 1e-3 of the oracle's, and 99 % of the
    keys assigned alike."""
    sp = workload.spec("tiny", num_kv_heads=2, n=20000, dtype="f32", seed=5)
    w = workload.generate(sp)
    keys = _t(w.keys)                                     # [1, 2, n, 128]
    cfg = pk.config(batch=1, num_kv_heads=2, capacity=sp.n, dtype="f32")
    y, kn = rotate_all(w.keys.reshape(2, sp.n, 128), w.signs)
    c0 = pk.train_centroids(cfg, w.signs, keys, 0).cpu().numpy()
    for u in range(2):
        np.testing.assert_allclose(c0[u], oracle.train_centroids(y[u], 0), atol=2e-5)
    c5 = pk.train_centroids(cfg, w.signs, keys, 5).cpu().numpy()
    for u in range(2):
        o5 = oracle.train_centroids(y[u], 5)
        ub = y[u].reshape(-1, 16, 8).astype(np.float64)
        ub /= np.linalg.norm(ub, axis=2, keepdims=True)

        def fit(c):
            ids = oracle.learned_ids(y[u], c)
            cos = np.einsum("nbj,nbj->nb", ub, c.astype(np.float64)[np.arange(16), ids])
            return float(cos.mean()), ids
        fg, ig = fit(c5[u])
        fo, io = fit(o5)
        assert abs(fg - fo) < 1e-3, (fg, fo)
        assert (ig == io).mean() > 0.99


def test_learned_errors():
    sp = workload.spec("tiny", n=300, dtype="f32")
    w = workload.generate(sp)
    cfg = pk.config(batch=1, num_kv_heads=1, capacity=300, dtype="f32")
    ix = pk.build_index(cfg, w.signs, _t(w.keys))
    cent = _t(np.broadcast_to(oracle.sign_centroids(), (1, 16, 256, 8)))
    with pytest.raises(pk.PariskvError) as e:          # not empty
        ix.set_centroids(cent)
    assert e.value.status == pk.EINVAL
    e0 = pk.build_index(cfg, w.signs, _t(w.keys), n=0)
    e0.set_centroids(cent)
    e0.append(_t(w.keys))
    with pytest.raises(pk.PariskvError) as e:          # learned indexes have no image
        e0.export_image()
    assert e.value.status == pk.EINVAL
    with pytest.raises(pk.PariskvError) as e:
        pk.train_centroids(cfg, w.signs, _t(w.keys), 1001)
    assert e.value.status == pk.EINVAL
