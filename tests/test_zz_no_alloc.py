"""The allocation-free sparse attention entry point, checked against the oracle.

Some callers may not call a device allocator while they decode: a serving runtime that
reserves all of HBM for its own memory manager, a process where stream-ordered memory pools
are unavailable, or a latency-critical loop where an allocation could block the stream.
pariskv_sparse_attend_noalloc serves them by keeping its split-K partials in a fixed array
inside the library; the caller still passes every input and output buffer. Every case below
compares the output with ``oracle.attend`` (fp64 softmax attention over the same rows) at
2e-3, the sparse attention bound, for K/V in HBM and in pinned host memory. This file is named
so that pytest collects it last: if it fails, a run that stops at the first failure has
already run every other test.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_kv_srht_b200 import pariskv as pk
from long_context_kv_srht_b200 import workload

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
SCALE = 1.0 / np.sqrt(128)


def _case(seed, batch, hkv, G, n, k, dtype, host_kv=False):
    rng = np.random.default_rng(seed)
    K = rng.standard_normal((batch, hkv, n, 128)).astype(np.float32) * 0.5
    V = rng.standard_normal((batch, hkv, n, 128)).astype(np.float32)
    q = rng.standard_normal((batch, hkv * G, 128)).astype(np.float32)
    topk = np.stack([np.sort(rng.choice(n, k, replace=False))
                     for _ in range(batch * hkv * G)]).astype(np.int32)
    if dtype == "bf16":
        K, V, q = workload.bf16_round(K), workload.bf16_round(V), workload.bf16_round(q)
        conv = lambda a: torch.from_numpy(workload.bf16_bits(a)).view(torch.bfloat16)
    else:
        conv = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    Kt, Vt = conv(K), conv(V)
    if host_kv:
        Kt, Vt = Kt.pin_memory(), Vt.pin_memory()
    else:
        Kt, Vt = Kt.to(DEV), Vt.to(DEV)
    cfg = pk.config(batch=batch, num_kv_heads=hkv, group=G, capacity=n, dtype=dtype)
    host = dict(q=q, K=K, V=V, topk=topk)
    return cfg, conv(q).to(DEV), Kt, Vt, torch.from_numpy(topk).to(DEV), host


def _check_against_oracle(got, host, G, heads=None):
    q, K, V, topk = host["q"], host["K"], host["V"], host["topk"]
    batch, Hq = q.shape[0], q.shape[1]
    got = got.float().cpu().numpy()
    worst = 0.0
    for i in (range(batch * Hq) if heads is None else heads):
        b, h = divmod(i, Hq)
        ref = oracle.attend(q[b, h], K[b, h // G], V[b, h // G], topk[i], SCALE)
        worst = max(worst, float(np.abs(got[b, h] - ref).max()))
    assert worst <= 2e-3, worst


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("host_kv", [False, True], ids=["hbm", "pinned_host"])
def test_noalloc_matches_oracle_on_two_calls(dtype, host_kv):
    # two calls in a row with different inputs: the shared workspace keeps the first call's
    # partials, and the second call must not be affected by them
    for seed, (batch, hkv, G, n, k) in ((11, (2, 2, 4, 5000, 512)), (12, (1, 8, 4, 20000, 2048))):
        cfg, q, K, V, topk, host = _case(seed, batch, hkv, G, n, k, dtype, host_kv)
        got = pk.sparse_attend_noalloc(cfg, q, K, V, topk, k, SCALE, out_dtype=torch.float32)
        torch.cuda.synchronize()
        _check_against_oracle(got, host, G)
        # and the allocating entry point gives the same numbers
        ref = pk.sparse_attend(cfg, q, K, V, topk, k, SCALE, out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert (got - ref).abs().max().item() <= 2e-3


def test_noalloc_many_heads_near_the_workspace_limit():
    # 4096 query heads (batch 512 x 8 KV heads) with k = 4096 on bf16 K/V in HBM: the fixed
    # workspace then holds one split per head, fewer than the tensor-core gather needs, so
    # the call falls back to the row-gather kernel with a single split. K/V (4.3 GB) are
    # drawn on the device; 64 heads spread over the batch are checked against the oracle.
    batch, hkv, G, n, k = 512, 8, 1, 4096, 4096
    gen = torch.Generator(device=DEV)
    gen.manual_seed(14)
    K = (torch.randn((batch, hkv, n, 128), generator=gen, device=DEV) * 0.5).to(torch.bfloat16)
    V = torch.randn((batch, hkv, n, 128), generator=gen, device=DEV).to(torch.bfloat16)
    q = torch.randn((batch, hkv * G, 128), generator=gen, device=DEV).to(torch.bfloat16)
    topk = torch.arange(n, dtype=torch.int32, device=DEV).repeat(batch * hkv * G, 1)
    cfg = pk.config(batch=batch, num_kv_heads=hkv, group=G, capacity=n, dtype="bf16")
    got = pk.sparse_attend_noalloc(cfg, q, K, V, topk, k, SCALE, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert pk.last_launch_count() == 2
    rows = np.arange(n, dtype=np.int32)
    worst = 0.0
    for i in np.linspace(0, batch * hkv * G - 1, 64).astype(int):
        b, h = divmod(int(i), hkv * G)
        ref = oracle.attend(q[b, h].float().cpu().numpy(), K[b, h // G].float().cpu().numpy(),
                            V[b, h // G].float().cpu().numpy(), rows, SCALE)
        worst = max(worst, float(np.abs(got[b, h].cpu().numpy() - ref).max()))
    assert worst <= 2e-3, worst
    del K, V
    torch.cuda.empty_cache()


def test_noalloc_rejects_requests_beyond_its_workspace():
    cfg, q, K, V, topk, _ = _case(13, 1, 1, 1, 64, 8, "f32")
    big = pk.config(batch=1000, num_kv_heads=8, group=1, capacity=64, dtype="f32")  # 8000 heads
    with pytest.raises(pk.PariskvError) as e:
        pk.sparse_attend_noalloc(big, q, K, V, topk, 8, 0.1, out=torch.empty_like(q))
    assert e.value.status == pk.EINVAL
    assert "workspace" in str(e.value)
