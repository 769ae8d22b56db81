"""GPU path vs the CPU oracle, through the C ABI.

Bit-exact gates (identical rotated fp32 inputs on both sides): bucket ids, 4-bit codes,
calibration factors, vote lookup tables, coarse scores, candidate sets, rerank values, top-k
indices and estimates. Tolerance gates: rotation <= 1e-5 absolute per coordinate of the
unit vector; end-to-end top-k recall from raw inputs >= 0.999; sparse attention <= 2e-3
absolute with fp32 output (bf16 output adds its own rounding bound)."""
import numpy as np
import pytest
import torch

import oracle
from long_context_kv_srht_b200 import pariskv as pk
from long_context_kv_srht_b200 import workload
from helpers import oracle_unit_from_rotated, random_signs, recall, rotate_all

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _cfg(batch, hkv, G, cap, dtype="f32", rho=4, w1=2, wr=1, bp=500, table=None):
    if table is None:
        return pk.config(batch=batch, num_kv_heads=hkv, group=G, capacity=cap, dtype=dtype,
                         rho=rho, w_rank1=w1, w_rest=wr, cand_bp=bp)
    return pk.config(batch=batch, num_kv_heads=hkv, group=G, capacity=cap, dtype=dtype, rho=rho,
                     w_rank1=w1, w_rest=wr, cand_bp=bp, levels="table", level_table=table)


def _t(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def _compare_rotated(batch, hkv, G, n, k, keys, qs, signs, rho=4, w1=2, wr=1, bp=500, cap=None,
                     table=None, edit_qt=None):
    """Build + search from the oracle's rotated inputs; compare every stage bit for bit
    (table: code both sides with these magnitude levels; edit_qt(qt) may change the rotated
    queries in place before both sides see them)."""
    units = batch * hkv
    y, kn = rotate_all(keys.reshape(units, n, 128), signs)
    qt, qn = rotate_all(qs.reshape(units * G, 128), signs)
    if edit_qt is not None:
        edit_qt(qt)
    cfg = _cfg(batch, hkv, G, cap or n, rho=rho, w1=w1, wr=wr, bp=bp, table=table)
    ix = pk.build_index_rotated(cfg, signs, _t(y), _t(kn))
    idx, est = ix.search_rotated(_t(qt), _t(qn), k)
    torch.cuda.synchronize()
    gids, gcodes, gfac = ix.export_index()
    glut, gsc, gcand, gS = ix.export_search()
    gidx, gest = idx.cpu().numpy(), est.cpu().numpy()
    p = oracle.SearchParams(m=8, rho=rho, w_rank1=w1, w_rest=wr, cand_bp=bp)
    for u in range(units):
        enc, heads = oracle_unit_from_rotated(y[u], kn[u], qt[u * G:(u + 1) * G],
                                              qn[u * G:(u + 1) * G], k, p, table=table)
        np.testing.assert_array_equal(gids[u], enc.ids)
        np.testing.assert_array_equal(gcodes[u], enc.codes)
        np.testing.assert_array_equal(gfac[u].view(np.uint32), enc.factor.view(np.uint32))
        for g, o in enumerate(heads):
            h = u * G + g
            np.testing.assert_array_equal(glut[h], o["lut"])
            np.testing.assert_array_equal(gsc[h], o["scores"])
            np.testing.assert_array_equal(gcand[h], o["cand"])
            np.testing.assert_array_equal(gS[h].view(np.uint32), o["S"].view(np.uint32))
            np.testing.assert_array_equal(gidx[h], o["idx"])
            np.testing.assert_array_equal(gest[h].view(np.uint32), o["est"].view(np.uint32))
    ix.destroy()


# ------------------------------------------------------------------------------- rotation
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_rotation_within_tolerance(dtype):
    rng = np.random.default_rng(0)
    x = (rng.standard_normal((5000, 128)) * rng.uniform(0.1, 20, (5000, 1))).astype(np.float32)
    x[7] = 0.0
    if dtype == "bf16":
        x = workload.bf16_round(x)
        xt = _t(workload.bf16_bits(x)).view(torch.bfloat16)
    else:
        xt = _t(x)
    s = random_signs(3)
    y, nr = pk.rotate(_cfg(1, 1, 1, 1, dtype=dtype), s, xt)
    yo, no = oracle.normalize_rotate(x, s)
    assert np.max(np.abs(y.cpu().numpy() - yo)) <= 1e-5
    np.testing.assert_allclose(nr.cpu().numpy(), no, rtol=2e-6)


# ------------------------------------------------------------------------------- stages
@pytest.mark.parametrize("batch,hkv,G,n,k,bp", [
    (1, 1, 1, 4096, 64, 1000),     # the tiny single-head workload shape
    (1, 2, 4, 20000, 128, 500),    # several chunks and a ragged tail, one full pack
    (2, 1, 5, 9000, 100, 500),     # two vote packs (group > 4)
    (1, 1, 3, 1, 1, 500),          # a single key
    (1, 1, 2, 31, 31, 500),        # k = n
    (1, 1, 1, 33, 5, 10000),       # every key is a candidate
    (1, 1, 4, 8193, 700, 300),     # one key past a chunk boundary
    (1, 1, 2, 70000, 3000, 10000), # > 65536 candidates per head: top-k reads them from memory
])
def test_stages_bit_exact(batch, hkv, G, n, k, bp):
    sp = workload.spec("tiny", batch=batch, num_kv_heads=hkv, group=G, n=n, dtype="f32",
                       planted=min(32, max(1, n // (4 * G))), seed=n)
    w = workload.generate(sp)
    _compare_rotated(batch, hkv, G, n, k, w.keys, w.queries, w.signs, bp=bp)


@pytest.mark.parametrize("batch,hkv,G,n,k,bp", [
    (1, 1, 1, 4096, 64, 1000),
    (1, 2, 4, 20000, 128, 500),
    (2, 1, 5, 9000, 100, 500),
    (1, 1, 2, 70000, 3000, 10000),
])
def test_table_levels_stages_bit_exact(batch, hkv, G, n, k, bp):
    """Codes from the rotation prior's levels (the oracle's table, given to both sides):
    every stage bit for bit, as with uniform levels."""
    sp = workload.spec("tiny", batch=batch, num_kv_heads=hkv, group=G, n=n, dtype="f32",
                       planted=min(32, max(1, n // (4 * G))), seed=n + 1)
    w = workload.generate(sp)
    _compare_rotated(batch, hkv, G, n, k, w.keys, w.queries, w.signs, bp=bp,
                     table=oracle.ratio_levels())


def test_table_levels_adversarial_and_zero_level():
    """Table coding of zero keys and subspaces, -0, duplicates, and a table whose lowest level
    is 0 (the two zero-magnitude nibbles then decode to +0 and -0)."""
    rng = np.random.default_rng(15)
    n, G = 3000, 4
    keys = rng.standard_normal((n, 128)).astype(np.float32)
    qs = rng.standard_normal((G, 128)).astype(np.float32)
    keys[0:10] = 0.0
    keys[10:40, 0:8] = 0.0
    keys[40:60, 1::4] = -0.0
    keys[100:300] = keys[99]
    keys[500:520] = qs[0] * 2.0
    for table in (oracle.ratio_levels(), np.array([0.0, 0.1, 0.2, 0.35, 0.5, 0.65, 0.8, 1.0],
                                                   np.float32)):
        _compare_rotated(1, 1, G, n, 300, keys, qs, random_signs(19), bp=1000, table=table)


@pytest.mark.parametrize("rho,w1,wr", [(1, 2, 1), (16, 2, 1), (256, 2, 1), (4, 3, 0), (4, 1, 1)])
def test_rho_and_weights_bit_exact(rho, w1, wr):
    sp = workload.spec("tiny", num_kv_heads=1, group=4, n=6000, seed=rho + 10 * w1)
    w = workload.generate(sp)
    _compare_rotated(1, 1, 4, 6000, 200, w.keys, w.queries, w.signs, rho=rho, w1=w1, wr=wr)


def test_adversarial_keys_bit_exact():
    """Zero keys, exact zeros and -0 coordinates, duplicate keys (ties in score and in S),
    and keys equal to the query."""
    rng = np.random.default_rng(5)
    n, G = 3000, 4
    keys = rng.standard_normal((n, 128)).astype(np.float32)
    qs = rng.standard_normal((G, 128)).astype(np.float32)
    keys[0:10] = 0.0
    keys[10:40, ::3] = 0.0
    keys[40:60, 1::4] = -0.0
    keys[100:400] = keys[99]                      # 300 identical keys
    keys[500:520] = qs[0] * 3.0                   # exact multiples of a query
    keys[600:620] = qs[1]
    _compare_rotated(1, 1, G, n, 400, keys, qs, random_signs(9), bp=1000)


def test_tiny_query_components_bit_exact():
    """Rotated queries with components near the bottom of the fp32 range (2^-110, normal
    values below 2^-100, subnormals), exact zeros and -0: the rerank stages the query scaled
    by powers of 16 only when that is exact, and every stage stays bit for bit."""
    rng = np.random.default_rng(23)
    n, G = 5000, 4
    keys = rng.standard_normal((n, 128)).astype(np.float32)
    qs = rng.standard_normal((G, 128)).astype(np.float32)

    def edit(qt):
        qt[0, 3] = np.float32(2.0 ** -110)
        qt[0, 77] = np.float32(-3.0e-36)
        qt[1, 5] = np.float32(1.0e-40)               # subnormal
        qt[1, 100] = np.float32(-2.0 ** -101)
        qt[2, 0:16] = 0.0
        qt[2, 16:20] = -0.0
        qt[3, 9] = np.float32(2.0 ** -99)             # just above the exactness bound

    _compare_rotated(1, 1, G, n, 300, keys, qs, random_signs(29), bp=1000, edit_qt=edit)


def test_append_equals_build():
    sp = workload.spec("tiny", num_kv_heads=2, group=4, n=12000, seed=21)
    w = workload.generate(sp)
    s = w.signs
    y, kn = rotate_all(w.keys.reshape(2, 12000, 128), s)
    cfg = _cfg(1, 2, 4, 12000)
    full = pk.build_index_rotated(cfg, s, _t(y), _t(kn))
    part = pk.build_index_rotated(cfg, s, _t(y[:, :9000]), _t(kn[:, :9000]))
    part.append_rotated(_t(y[:, 9000:9001]), _t(kn[:, 9000:9001]))
    for a in range(9001, 12000, 1000):
        b = min(12000, a + 1000)
        part.append_rotated(_t(y[:, a:b]), _t(kn[:, a:b]))
    assert part.size == full.size == 12000
    for x, z in zip(full.export_index(), part.export_index()):
        np.testing.assert_array_equal(x, z)
    # raw-key append matches a raw-key build too
    cfgb = _cfg(1, 2, 4, 12000, dtype="f32")
    kt = _t(w.keys)
    rb = pk.build_index(cfgb, s, kt)
    ra = pk.build_index(cfgb, s, kt[:, :, :5000].contiguous())
    ra.append(kt[:, :, 5000:])
    for x, z in zip(rb.export_index(), ra.export_index()):
        np.testing.assert_array_equal(x, z)


# ------------------------------------------------------------------------------- end to end
@pytest.mark.parametrize("name,n", [("tiny", None), ("llama3_8b_128k", 16384),
                                    ("batched_64k", 8192)])
def test_end_to_end_recall_from_raw_inputs(name, n):
    sp = workload.spec(name, batch=min(2, workload.SPECS[name].batch))
    w = workload.generate(sp, n=n)
    n = w.keys.shape[2]
    k = min(sp.k, n // 8)
    cfg = _cfg(sp.batch, sp.num_kv_heads, sp.group, n, dtype=sp.dtype, bp=sp.cand_bp)
    if sp.dtype == "bf16":
        keys = _t(workload.bf16_bits(w.keys)).view(torch.bfloat16)
        qs = _t(workload.bf16_bits(w.queries)).view(torch.bfloat16)
    else:
        keys, qs = _t(w.keys), _t(w.queries)
    ix = pk.build_index(cfg, w.signs, keys)
    idx, est = ix.search(qs, k)
    idx = idx.cpu().numpy()
    p = oracle.SearchParams(m=8, rho=sp.rho, cand_bp=sp.cand_bp)
    hits, tot, planted_hits, planted_tot = 0, 0, 0, 0
    for b in range(sp.batch):
        for h in range(sp.num_kv_heads):
            enc = oracle.build_unit(w.keys[b, h], w.signs, 8)
            for g in range(sp.group):
                hq = h * sp.group + g
                o_idx, *_ = oracle.search(enc, w.queries[b, hq], w.signs, k, p)
                g_idx = idx[b * sp.num_q_heads + hq]
                assert np.all(np.diff(g_idx) > 0)
                hits += len(set(g_idx.tolist()) & set(o_idx.tolist()))
                tot += k
                pl = set(w.planted[b, hq].tolist())
                planted_hits += len(pl & set(g_idx.tolist()))
                planted_tot += len(pl)
    assert hits / tot >= 0.999, hits / tot
    if planted_tot:
        assert planted_hits / planted_tot >= 0.9


# ------------------------------------------------------------------------------- attention
@pytest.mark.parametrize("dtype,G,n,k", [("bf16", 4, 5000, 512), ("f32", 1, 3000, 3000),
                                         ("bf16", 2, 70, 1), ("bf16", 4, 20000, 2048)])
@pytest.mark.parametrize("host_kv", [False, True])
@pytest.mark.parametrize("out_f32", [True, False])
def test_sparse_attend_matches_oracle(dtype, G, n, k, host_kv, out_f32):
    """fp32 output: |gpu - oracle| <= 2e-3. bf16 output additionally carries its own
    round-to-nearest error, at most 2^-9 |x| (8 significand bits), so the bound there is
    2e-3 + 2^-8 |oracle| (one rounding of the result plus fp32 accumulation slack)."""
    rng = np.random.default_rng(n + k)
    batch, hkv = 2, 2
    K = rng.standard_normal((batch, hkv, n, 128)).astype(np.float32) * 0.5
    V = rng.standard_normal((batch, hkv, n, 128)).astype(np.float32)
    q = rng.standard_normal((batch, hkv * G, 128)).astype(np.float32)
    if dtype == "bf16":
        K, V, q = workload.bf16_round(K), workload.bf16_round(V), workload.bf16_round(q)
        conv = lambda a: torch.from_numpy(workload.bf16_bits(a)).view(torch.bfloat16)
    else:
        conv = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    topk = np.stack([np.sort(rng.choice(n, k, replace=False)) for _ in range(batch * hkv * G)])
    cfg = _cfg(batch, hkv, G, n, dtype=dtype)
    Kt, Vt = conv(K), conv(V)
    if host_kv:
        Kt, Vt = Kt.pin_memory(), Vt.pin_memory()
    else:
        Kt, Vt = Kt.to(DEV), Vt.to(DEV)
    od = torch.float32 if out_f32 else torch.bfloat16
    out = pk.sparse_attend(cfg, conv(q).to(DEV), Kt, Vt, _t(topk.astype(np.int32)), k,
                           1 / np.sqrt(128), out_dtype=od)
    got = out.float().cpu().numpy()
    for b in range(batch):
        for h in range(hkv * G):
            ref = oracle.attend(q[b, h], K[b, h // G], V[b, h // G],
                                topk[b * hkv * G + h].astype(np.int32), 1 / np.sqrt(128))
            tol = 2e-3 if out_f32 else 2e-3 + np.abs(ref) * 2.0 ** -8
            assert np.all(np.abs(got[b, h] - ref) <= tol)


@pytest.mark.parametrize("dtype,G,host_kv,n,k", [("bf16", 4, True, 20000, 1024),
                                                 ("f32", 4, False, 20000, 1024),
                                                 ("bf16", 8, True, 20000, 1024),
                                                 ("bf16", 3, True, 20000, 1024),
                                                 ("bf16", 2, True, 20000, 1024),
                                                 ("bf16", 4, True, 20001, 999),
                                                 ("f32", 2, False, 70, 33)])
def test_group_union_attention_shares_rows(dtype, G, host_kv, n, k, monkeypatch):
    """The query heads of a group select overlapping rows (a common core, a shared pool and
    rows of their own); the row-gather attention fetches each row of the group's union once
    and still matches the oracle per head at 2e-3. The fetched-row count equals the union
    size, and turning the union off gives the same outputs within the same bound."""
    rng = np.random.default_rng(31 + G + n)
    batch, hkv = 2, 2
    K = rng.standard_normal((batch, hkv, n, 128)).astype(np.float32) * 0.5
    V = rng.standard_normal((batch, hkv, n, 128)).astype(np.float32)
    q = rng.standard_normal((batch, hkv * G, 128)).astype(np.float32)
    if dtype == "bf16":
        K, V, q = workload.bf16_round(K), workload.bf16_round(V), workload.bf16_round(q)
        conv = lambda a: torch.from_numpy(workload.bf16_bits(a)).view(torch.bfloat16)
    else:
        conv = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    topk, union = [], 0
    for u in range(batch * hkv):
        core = rng.choice(n, k // 2, replace=False)            # every head of the group
        pool = np.setdiff1d(rng.choice(n, 2 * k, replace=False), core)
        rows = set()
        for g in range(G):
            own = rng.choice(pool, k - k // 2, replace=False)   # partly shared, partly not
            sel = np.sort(np.concatenate([core, own]))
            assert len(np.unique(sel)) == k
            topk.append(sel)
            rows |= set(sel.tolist())
        union += len(rows)
    topk = np.stack(topk).astype(np.int32)
    cfg = _cfg(batch, hkv, G, n, dtype=dtype)
    Kt, Vt = conv(K), conv(V)
    Kt, Vt = (Kt.pin_memory(), Vt.pin_memory()) if host_kv else (Kt.to(DEV), Vt.to(DEV))
    pk.union_rows()                                            # reset the counter
    out = pk.sparse_attend(cfg, conv(q).to(DEV), Kt, Vt, _t(topk), k, 1 / np.sqrt(128),
                           out_dtype=torch.float32)
    assert pk.union_rows() == union < batch * hkv * G * k
    got = out.cpu().numpy()
    for b in range(batch):
        for h in range(hkv * G):
            ref = oracle.attend(q[b, h], K[b, h // G], V[b, h // G],
                                topk[b * hkv * G + h], 1 / np.sqrt(128))
            assert np.all(np.abs(got[b, h] - ref) <= 2e-3)
    monkeypatch.setenv("PARISKV_ATTEND_UNION", "0")
    per_head = pk.sparse_attend(cfg, conv(q).to(DEV), Kt, Vt, _t(topk), k, 1 / np.sqrt(128),
                                out_dtype=torch.float32)
    assert pk.union_rows() == 0
    assert (per_head - out).abs().max().item() <= 2e-3


# ------------------------------------------------------------------------------- errors
def test_error_paths():
    sp = workload.spec("tiny", n=100)
    w = workload.generate(sp)
    cfg = _cfg(1, 1, 1, 100)
    ix = pk.build_index(cfg, w.signs, _t(w.keys))
    with pytest.raises(pk.PariskvError) as e:
        ix.append(_t(w.keys[:, :, :1]))
    assert e.value.status == pk.ECAPACITY and ix.size == 100
    with pytest.raises(pk.PariskvError) as e:
        ix.search(_t(w.queries), 101)
    assert e.value.status == pk.EINVAL
    with pytest.raises(pk.PariskvError) as e:   # pageable host memory is rejected
        pk.build_index(cfg, w.signs, torch.from_numpy(w.keys))
    assert e.value.status == pk.EINVAL
    bad = w.signs.copy()
    bad[3] = 0
    with pytest.raises(pk.PariskvError) as e:
        pk.build_index(cfg, bad, _t(w.keys))
    assert e.value.status == pk.EINVAL
    ix.sync()
    assert ix.size == 100


def test_allocation_failure_is_reported(monkeypatch):
    sp = workload.spec("tiny", n=100)
    w = workload.generate(sp)
    keys = _t(w.keys)
    monkeypatch.setenv("PARISKV_FAULT", "alloc")
    with pytest.raises(pk.PariskvError) as e:
        pk.build_index(_cfg(1, 1, 1, 100), w.signs, keys)
    assert e.value.status == pk.ENOMEM
    monkeypatch.delenv("PARISKV_FAULT")
    ix = pk.build_index(_cfg(1, 1, 1, 100), w.signs, keys)
    idx, _ = ix.search(_t(w.queries), 10)
    assert idx.shape == (1, 10)


def test_injected_launch_failure(monkeypatch):
    """PARISKV_FAULT=launch: search, append and both attention calls fail with ECUDA before
    launching, the index keeps its size and state, and once the hook is off the index
    searches exactly as before."""
    sp = workload.spec("tiny", n=2000, seed=41)
    w = workload.generate(sp)
    cfg = _cfg(1, 1, 1, 2100)
    keys = _t(w.keys)
    ix = pk.build_index(cfg, w.signs, keys)
    q = _t(w.queries)
    ref_idx, ref_est = ix.search(q, 50)
    torch.cuda.synchronize()
    monkeypatch.setenv("PARISKV_FAULT", "launch")
    for call in (lambda: ix.search(q, 50), lambda: ix.append(keys[:, :, :10]),
                 lambda: pk.sparse_attend(cfg, q, keys, keys, ref_idx, 50, 0.1),
                 lambda: pk.sparse_attend_noalloc(cfg, q, keys, keys, ref_idx, 50, 0.1)):
        with pytest.raises(pk.PariskvError) as e:
            call()
        assert e.value.status == pk.ECUDA and "injected" in pk.last_error()
    assert ix.size == 2000
    monkeypatch.delenv("PARISKV_FAULT")
    idx, est = ix.search(q, 50)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx.cpu().numpy())
    np.testing.assert_array_equal(est.cpu().numpy().view(np.uint32),
                                  ref_est.cpu().numpy().view(np.uint32))
    ix.sync()
