"""The allocation-free sparse attention entry point, checked against the allocating one.

Some callers may not call a device allocator while they decode: a serving runtime that
reserves all of HBM for its own memory manager, a process where stream-ordered memory pools
are unavailable, or a latency-critical loop where an allocation could block the stream.
pariskv_sparse_attend_noalloc serves them by keeping its split-K partials in a fixed array
inside the library; the caller still passes every input and output buffer. This file is named
so that pytest collects it last: if it fails, a run that stops at the first failure has
already run every other test.
"""
import numpy as np
import pytest
import torch

from long_context_kv_srht_b200 import pariskv as pk
from long_context_kv_srht_b200 import workload

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _case(seed, batch, hkv, G, n, k, dtype):
    rng = np.random.default_rng(seed)
    K = rng.standard_normal((batch, hkv, n, 128)).astype(np.float32) * 0.5
    V = rng.standard_normal((batch, hkv, n, 128)).astype(np.float32)
    q = rng.standard_normal((batch, hkv * G, 128)).astype(np.float32)
    topk = np.stack([np.sort(rng.choice(n, k, replace=False))
                     for _ in range(batch * hkv * G)]).astype(np.int32)
    if dtype == "bf16":
        conv = lambda a: torch.from_numpy(workload.bf16_bits(workload.bf16_round(a))).view(
            torch.bfloat16).to(DEV)
    else:
        conv = lambda a: torch.from_numpy(a).to(DEV)
    cfg = pk.config(batch=batch, num_kv_heads=hkv, group=G, capacity=n, dtype=dtype)
    return cfg, conv(q), conv(K), conv(V), torch.from_numpy(topk).to(DEV)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_noalloc_matches_allocating_entry_point_on_two_calls(dtype):
    # two calls in a row with different inputs: the shared workspace keeps the first call's
    # partials, and the second call must not be affected by them
    for seed, (batch, hkv, G, n, k) in ((11, (2, 2, 4, 5000, 512)), (12, (1, 8, 4, 20000, 2048))):
        cfg, q, K, V, topk = _case(seed, batch, hkv, G, n, k, dtype)
        scale = 1.0 / np.sqrt(128)
        ref = pk.sparse_attend(cfg, q, K, V, topk, k, scale, out_dtype=torch.float32)
        got = pk.sparse_attend_noalloc(cfg, q, K, V, topk, k, scale, out_dtype=torch.float32)
        torch.cuda.synchronize()
        err = (got - ref).abs().max().item()
        assert err <= 2e-3, err


def test_noalloc_rejects_requests_beyond_its_workspace():
    cfg, q, K, V, topk = _case(13, 1, 1, 1, 64, 8, "f32")
    big = pk.config(batch=1000, num_kv_heads=8, group=1, capacity=64, dtype="f32")  # 8000 heads
    with pytest.raises(pk.PariskvError) as e:
        pk.sparse_attend_noalloc(big, q, K, V, topk, 8, 0.1, out=torch.empty_like(q))
    assert e.value.status == pk.EINVAL
    assert "workspace" in str(e.value)
