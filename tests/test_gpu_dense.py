"""Dense decode attention (include/pariskv_dense.h), the full-attention baseline, against the
oracle's attention over every token (fp64), through the C ABI: several 64-token tiles with
ragged tails, every GQA group size the kernel takes, K/V in HBM and in pinned host memory,
and one million-token unit checked on sampled heads."""
import numpy as np
import pytest
import torch

import oracle
from long_context_kv_srht_b200 import pariskv as pk
from long_context_kv_srht_b200 import workload

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
SCALE = 1 / np.sqrt(128)


def _bf(a):
    return torch.from_numpy(workload.bf16_bits(a)).view(torch.bfloat16)


def _case(batch, hkv, G, n, ld, seed):
    rng = np.random.default_rng(seed)
    K = workload.bf16_round(rng.standard_normal((batch, hkv, ld, 128)).astype(np.float32) * 0.5)
    V = workload.bf16_round(rng.standard_normal((batch, hkv, ld, 128)).astype(np.float32))
    q = workload.bf16_round(rng.standard_normal((batch, hkv * G, 128)).astype(np.float32))
    return K, V, q


def _check(got, K, V, q, G, n, out_f32, heads=None):
    batch, hq = q.shape[:2]
    for b in range(batch):
        for h in (range(hq) if heads is None else heads):
            ref = oracle.attend(q[b, h], K[b, h // G], V[b, h // G], np.arange(n, dtype=np.int32),
                                SCALE)
            tol = 2e-3 if out_f32 else 2e-3 + np.abs(ref) * 2.0 ** -8
            err = np.abs(got[b, h] - ref)
            assert np.all(err <= tol), (b, h, err.max())


@pytest.mark.parametrize("G", [1, 2, 3, 4, 5, 8])
@pytest.mark.parametrize("n,ld", [(1, 1), (63, 70), (64, 64), (65, 65), (1000, 1031),
                                  (4097, 4100), (70001, 70001)])
def test_dense_attend_matches_oracle(G, n, ld):
    batch, hkv = 2, 2
    K, V, q = _case(batch, hkv, G, n, ld, seed=n * 10 + G)
    cfg = pk.config(batch=batch, num_kv_heads=hkv, group=G, capacity=ld, dtype="bf16")
    out = pk.dense_attend(cfg, _bf(q).to(DEV), _bf(K).to(DEV), _bf(V).to(DEV), SCALE, n=n,
                          out_dtype=torch.float32)
    _check(out.cpu().numpy(), K, V, q, G, n, True)


@pytest.mark.parametrize("host_kv,out_f32", [(True, True), (False, False)])
def test_dense_attend_host_kv_and_bf16_out(host_kv, out_f32):
    batch, hkv, G, n = 1, 3, 4, 5000
    K, V, q = _case(batch, hkv, G, n, n, seed=11)
    cfg = pk.config(batch=batch, num_kv_heads=hkv, group=G, capacity=n, dtype="bf16")
    Kt, Vt = _bf(K), _bf(V)
    Kt, Vt = (Kt.pin_memory(), Vt.pin_memory()) if host_kv else (Kt.to(DEV), Vt.to(DEV))
    od = torch.float32 if out_f32 else torch.bfloat16
    out = pk.dense_attend(cfg, _bf(q).to(DEV), Kt, Vt, SCALE, out_dtype=od)
    _check(out.float().cpu().numpy(), K, V, q, G, n, out_f32)


def test_dense_attend_million_tokens_sampled():
    """One KV head of the million-token workload's length (plus a ragged tail), 4 query
    heads; every head checked against the oracle."""
    n = (1 << 20) + 7
    K, V, q = _case(1, 1, 4, n, n, seed=5)
    cfg = pk.config(batch=1, num_kv_heads=1, group=4, capacity=n, dtype="bf16")
    out = pk.dense_attend(cfg, _bf(q).to(DEV), _bf(K).to(DEV), _bf(V).to(DEV), SCALE,
                          out_dtype=torch.float32)
    _check(out.cpu().numpy(), K, V, q, 4, n, True)


def test_dense_attend_errors():
    K, V, q = _case(1, 1, 1, 64, 64, seed=1)
    Kd, Vd, qd = _bf(K).to(DEV), _bf(V).to(DEV), _bf(q).to(DEV)
    for kw, st in [(dict(dtype="f32"), pk.EINVAL), (dict(group=9), pk.EINVAL)]:
        cfg = pk.config(batch=1, num_kv_heads=1, capacity=64, **{"dtype": "bf16", **kw})
        with pytest.raises(pk.PariskvError) as e:
            pk.dense_attend(cfg, qd, Kd, Vd, SCALE)
        assert e.value.status == st
    cfg = pk.config(batch=1, num_kv_heads=1, group=1, capacity=64, dtype="bf16")
    with pytest.raises(pk.PariskvError) as e:
        pk.dense_attend(cfg, qd, Kd, Vd, SCALE, n=0)
    assert e.value.status == pk.EINVAL
    with pytest.raises(pk.PariskvError) as e:          # ld_tok < n
        pk.dense_attend(cfg, qd, Kd, Vd, SCALE, n=65)
    assert e.value.status == pk.EINVAL
