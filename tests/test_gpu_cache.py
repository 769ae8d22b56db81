"""Four-region KV cache through the C ABI (include/pariskv_cache.h) against the oracle's
region model and attention ("Technical Summary: ParisKV", System-Level Innovations 2,
"Sliding-Window Update Mechanism"; System-Level Innovations 1, UVA offloading).

Each decode step is checked for: the region sizes (oracle.CacheRegions), the Retrieval
index (bit-identical to an index built in one call from the tokens the oracle says were
evicted, in order), the retrieved rows (identical to a standalone search of that index, and
recall against the oracle's search from raw inputs), and the attention output (oracle.attend
over Sink + Local + buffer + the retrieved tokens, within 2e-3)."""
import numpy as np
import pytest
import torch

import oracle
from long_context_kv_srht_b200 import pariskv as pk
from long_context_kv_srht_b200 import workload
from helpers import random_signs

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
SCALE = 1 / np.sqrt(128)


def _conv(a, dtype):
    if dtype == "bf16":
        return torch.from_numpy(workload.bf16_bits(a)).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))


def _data(seed, hkv, G, total, dtype):
    rng = np.random.default_rng(seed)
    K = rng.standard_normal((1, hkv, total, 128)).astype(np.float32) * 0.5
    K += rng.standard_normal((1, hkv, 1, 128)).astype(np.float32) * 0.3   # shared key mean
    V = rng.standard_normal((1, hkv, total, 128)).astype(np.float32)
    q = rng.standard_normal((total, hkv * G, 128)).astype(np.float32)
    if dtype == "bf16":
        K, V, q = workload.bf16_round(K), workload.bf16_round(V), workload.bf16_round(q)
    return K, V, q


def _run(dtype, hkv, G, n_sink, n_local, n_buffer, k, n0, steps, host_prefill, out_f32,
         check_every, seed, batch=1):
    total = n0 + steps
    if batch > 1:                      # sequences of a batch are further KV heads here
        return _run_batched(dtype, batch, hkv, G, n_sink, n_local, n_buffer, k, n0, steps,
                            seed)
    K, V, q = _data(seed, hkv, G, total, dtype)
    signs = random_signs(seed)
    cfg = pk.config(batch=1, num_kv_heads=hkv, group=G, capacity=1, dtype=dtype, rho=4,
                    cand_bp=1000)
    cache = pk.Cache(cfg, signs, n_sink, n_local, n_buffer, k, retrieval_capacity=total)
    Kt, Vt = _conv(K, dtype), _conv(V, dtype)
    if host_prefill:
        Kp, Vp = Kt.pin_memory(), Vt.pin_memory()
    else:
        Kp, Vp = Kt.to(DEV), Vt.to(DEV)
    Kd, Vd, qd = Kt.to(DEV), Vt.to(DEV), _conv(q, dtype).to(DEV)
    cache.prefill(Kp, Vp, n=n0)
    model = oracle.CacheRegions(n_sink, n_local, n_buffer)
    model.prefill(n0)
    assert cache.counts() == dict(zip(pk.Cache.REGIONS, (len(model.sink), len(model.local),
                                                         len(model.buffer),
                                                         len(model.retrieval))))
    p = oracle.SearchParams(m=8, rho=4, cand_bp=1000)
    od = torch.float32 if out_f32 else torch.bfloat16
    hits = want = 0
    promotions = 0
    for t in range(steps):
        tok = n0 + t
        before = len(model.retrieval)
        out, topk = cache.step(qd[tok].view(1, hkv * G, 128),
                               Kd[:, :, tok].contiguous(), Vd[:, :, tok].contiguous(), SCALE,
                               out_dtype=od, want_topk=True)
        model.append()
        promotions += len(model.retrieval) != before
        counts = cache.counts()
        assert counts == dict(zip(pk.Cache.REGIONS, (len(model.sink), len(model.local),
                                                     len(model.buffer),
                                                     len(model.retrieval)))), t
        if t % check_every and t != steps - 1 and len(model.retrieval) == before:
            continue
        R = len(model.retrieval)
        k_eff = min(k, R)
        got = out.float().cpu().numpy()[0]
        gtop = topk.cpu().numpy()
        assert np.all(gtop[:, k_eff:] == -1)
        if R:
            # the cache's index holds exactly the evicted tokens, in order
            ix = cache.index()
            ref_ix = pk.build_index(pk.config(batch=1, num_kv_heads=hkv, group=G, capacity=R,
                                              dtype=dtype, rho=4, cand_bp=1000),
                                    signs, Kd[:, :, model.retrieval[0]:model.retrieval[-1] + 1])
            assert model.retrieval == list(range(n_sink, n_sink + R))
            for a, b in zip(ix.export_index(), ref_ix.export_index()):
                np.testing.assert_array_equal(a, b)
            sidx, _ = ref_ix.search(qd[tok].view(1, hkv * G, 128), k_eff)
            np.testing.assert_array_equal(gtop[:, :k_eff], sidx.cpu().numpy())
        for h in range(hkv * G):
            rows = gtop[h, :k_eff]
            if R:
                assert np.all(np.diff(rows) > 0) and rows.max() < R
                enc = oracle.build_unit(K[0, h // G, model.retrieval], signs, 8)
                o_idx, *_ = oracle.search(enc, q[tok, h], signs, k_eff, p)
                hits += len(set(rows.tolist()) & set(o_idx.tolist()))
                want += k_eff
            toks = np.asarray(model.dense() + [model.retrieval[r] for r in rows], np.int32)
            ref = oracle.attend(q[tok, h], K[0, h // G], V[0, h // G], toks, SCALE)
            tol = 2e-3 if out_f32 else 2e-3 + np.abs(ref) * 2.0 ** -8
            assert np.all(np.abs(got[h] - ref) <= tol), (t, h, np.abs(got[h] - ref).max())
    # raw inputs: the GPU rotates in fp32, the oracle in fp64, so a near-tied key may differ
    if want:
        assert hits / want >= 0.999, hits / want
    cache.destroy()
    return promotions


def _run_batched(dtype, batch, hkv, G, n_sink, n_local, n_buffer, k, n0, steps, seed):
    """batch > 1: the attention output against the oracle at every promotion and at the last
    step, every sequence and head (region sizes are shared by all sequences)."""
    total = n0 + steps
    units = batch * hkv
    K, V, q = _data(seed, units, G, total, dtype)            # [1, units, total, 128]
    signs = random_signs(seed)
    cfg = pk.config(batch=batch, num_kv_heads=hkv, group=G, capacity=1, dtype=dtype, rho=4,
                    cand_bp=1000)
    cache = pk.Cache(cfg, signs, n_sink, n_local, n_buffer, k, retrieval_capacity=total)
    Kd, Vd = _conv(K, dtype).to(DEV), _conv(V, dtype).to(DEV)
    qd = _conv(q, dtype).to(DEV)                              # [total, units * G, 128]
    cache.prefill(Kd.view(batch, hkv, total, 128), Vd.view(batch, hkv, total, 128), n=n0)
    model = oracle.CacheRegions(n_sink, n_local, n_buffer)
    model.prefill(n0)
    checked = 0
    for t in range(steps):
        tok = n0 + t
        before = len(model.retrieval)
        out, topk = cache.step(qd[tok].view(batch, hkv * G, 128),
                               Kd[0, :, tok].contiguous().view(batch, hkv, 128),
                               Vd[0, :, tok].contiguous().view(batch, hkv, 128), SCALE,
                               out_dtype=torch.float32, want_topk=True)
        model.append()
        if len(model.retrieval) == before and t != steps - 1:
            continue
        checked += 1
        got = out.cpu().numpy().reshape(units * G, 128)
        gtop = topk.cpu().numpy()
        k_eff = min(k, len(model.retrieval))
        for h in range(units * G):
            rows = gtop[h, :k_eff]
            toks = np.asarray(model.dense() + [model.retrieval[r] for r in rows], np.int32)
            ref = oracle.attend(q[tok, h], K[0, h // G], V[0, h // G], toks, SCALE)
            assert np.all(np.abs(got[h] - ref) <= 2e-3), (t, h)
    cache.destroy()
    return checked


@pytest.mark.parametrize("dtype,hkv,G,n_sink,n_local,n_buffer,k,n0,steps,host,out_f32", [
    ("bf16", 2, 4, 4, 128, 32, 64, 2000, 200, False, True),
    ("f32", 1, 2, 0, 64, 64, 256, 100, 150, True, False),
    ("bf16", 1, 1, 3, 32, 8, 16, 1, 120, False, True),
])
def test_cache_decode_matches_oracle(dtype, hkv, G, n_sink, n_local, n_buffer, k, n0, steps,
                                     host, out_f32):
    promotions = _run(dtype, hkv, G, n_sink, n_local, n_buffer, k, n0, steps, host, out_f32,
                      check_every=17, seed=n0 + steps)
    assert promotions >= 2


def test_cache_batched_group_8():
    """Two sequences of two KV heads with 8 query heads each (the widest group of the
    tensor-core dense pass)."""
    assert _run("bf16", 2, 8, 4, 64, 16, 32, 500, 70, False, True, 0, seed=9, batch=2) >= 3


def test_cache_capacity_and_errors():
    K, V, q = _data(1, 1, 1, 64, "bf16")
    signs = random_signs(1)
    cfg = pk.config(batch=1, num_kv_heads=1, group=1, capacity=1, dtype="bf16")
    Kd, Vd, qd = _conv(K, "bf16").to(DEV), _conv(V, "bf16").to(DEV), _conv(q, "bf16").to(DEV)
    with pytest.raises(pk.PariskvError) as e:          # n_local < n_buffer
        pk.Cache(cfg, signs, 2, 4, 8, 4, 16)
    assert e.value.status == pk.EINVAL
    cache = pk.Cache(cfg, signs, 2, 8, 4, 4, retrieval_capacity=6)
    with pytest.raises(pk.PariskvError) as e:          # 2 + 8 + 7 tokens: 7 > 6 in Retrieval
        cache.prefill(Kd, Vd, n=17)
    assert e.value.status == pk.ECAPACITY
    assert cache.counts() == dict(sink=0, local=0, buffer=0, retrieval=0)
    cache.prefill(Kd, Vd, n=14)                        # Retrieval holds 4
    for t in range(14, 18):                            # fourth step promotes 4 more: 8 > 6
        if t < 17:
            cache.step(qd[t].view(1, 1, 128), Kd[:, :, t].contiguous(),
                       Vd[:, :, t].contiguous(), SCALE)
            continue
        before = cache.counts()
        with pytest.raises(pk.PariskvError) as e:
            cache.step(qd[t].view(1, 1, 128), Kd[:, :, t].contiguous(),
                       Vd[:, :, t].contiguous(), SCALE)
        assert e.value.status == pk.ECAPACITY
        assert cache.counts() == before
    with pytest.raises(pk.PariskvError) as e:          # prefill needs an empty cache
        cache.prefill(Kd, Vd, n=1)
    assert e.value.status == pk.EINVAL
    cache.destroy()


def test_cache_step_launch_count():
    """A step is one token-copy kernel, the search's launches, two attention partials and one
    merge, plus (group > 1) the three kernels that build the GQA group's union of retrieved rows;
    a step that evicts to the Retrieval zone adds the spill, encode and slide kernels."""
    K, V, q = _data(2, 2, 2, 600, "bf16")
    signs = random_signs(2)
    cfg = pk.config(batch=1, num_kv_heads=2, group=2, capacity=1, dtype="bf16")
    Kd, Vd, qd = _conv(K, "bf16").to(DEV), _conv(V, "bf16").to(DEV), _conv(q, "bf16").to(DEV)
    cache = pk.Cache(cfg, signs, 4, 32, 8, 32, retrieval_capacity=600)
    cache.prefill(Kd, Vd, n=500)
    ix = pk.build_index(pk.config(batch=1, num_kv_heads=2, group=2, capacity=600,
                                  dtype="bf16"), signs, Kd[:, :, 4:468])
    ix.search(qd[0].view(1, 4, 128), 32)
    search_launches = pk.last_launch_count()
    seen = []
    for t in range(500, 516):
        cache.step(qd[t].view(1, 4, 128), Kd[:, :, t].contiguous(), Vd[:, :, t].contiguous(),
                   SCALE)
        seen.append(pk.last_launch_count())
    assert seen.count(search_launches + 7) == 14 and seen.count(search_launches + 10) == 2
    cache.destroy()
