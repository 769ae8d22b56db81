"""Long-generation drift through the C ABI ("ParisKV: Fast and Drift-Robust KV-Cache
Retrieval for Long-Context LLMs", abstract: retrieval under distribution drift; "Technical
Summary: ParisKV", Key Contributions 1 and Core Algorithmic Innovations 1: the index is kept
current as keys are generated).

Workload: 8 KV heads, a 32768-key prefill, then one appended key per KV head per decode step
while the keys' mean vector moves linearly to a fresh random direction; one query head per
KV head searches after every append with k = 1024. The index only ever grows by append.

Gates: at sampled steps the top-k from raw bf16 inputs matches the oracle's search over the
same keys with recall >= 0.999 (the GPU rotates in fp32, the oracle in fp64); after the last
step the appended index is bit-identical to one built from all keys in a single call. Fed
the oracle's own rotations, the index and the search at every 256th step are bit-exact."""
import numpy as np
import pytest
import torch

import oracle
from long_context_kv_srht_b200 import pariskv as pk
from long_context_kv_srht_b200 import workload
from helpers import rotate_all

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
STEPS = 4096          # decode steps run here (the benchmark's drift mode runs all 32768)


def _bf16(a):
    return torch.from_numpy(workload.bf16_bits(a)).view(torch.bfloat16)


def test_drift_append_and_search():
    sp = workload.spec("drift_32k")
    w = workload.generate_drift(sp, steps=STEPS)
    H, n0, k = sp.num_kv_heads, sp.n, sp.k
    cfg = pk.config(batch=1, num_kv_heads=H, group=1, capacity=n0 + STEPS, dtype=sp.dtype,
                    rho=sp.rho, cand_bp=sp.cand_bp)
    pre = _bf16(w.prefill[None]).to(DEV)               # [1, H, n0, d]
    app = _bf16(w.appended).to(DEV)                    # [steps, H, d]
    qs = _bf16(w.queries).to(DEV)                      # [steps, H, d]
    ix = pk.build_index(cfg, w.signs, pre)
    check = sorted(set(range(0, STEPS, 1365)) | {STEPS - 1})
    got = {}
    for t in range(STEPS):
        ix.append(app[t].view(1, H, 1, 128))
        idx, _ = ix.search(qs[t].view(1, H, 128), k)
        if t in check:
            got[t] = idx.cpu().numpy()
    ix.sync()
    assert ix.size == n0 + STEPS

    p = oracle.SearchParams(m=8, rho=sp.rho, cand_bp=sp.cand_bp)
    for t in check:
        hits = 0
        for h in range(H):
            keys = np.concatenate([w.prefill[h], w.appended[: t + 1, h]], axis=0)
            enc = oracle.build_unit(keys, w.signs, 8)
            o_idx, *_ = oracle.search(enc, w.queries[t, h], w.signs, k, p)
            g_idx = got[t][h]
            assert np.all(np.diff(g_idx) > 0)
            assert g_idx.max() <= n0 + t      # only keys present at step t
            hits += len(set(g_idx.tolist()) & set(o_idx.tolist()))
        assert hits / (H * k) >= 0.999, (t, hits / (H * k))

    # append-only growth leaves the same index as one build over all keys
    allk = torch.cat([pre, app.permute(1, 0, 2).unsqueeze(0)], dim=2).contiguous()
    ref = pk.build_index(cfg, w.signs, allk)
    for a, b in zip(ix.export_index(), ref.export_index()):
        np.testing.assert_array_equal(a, b)


def test_drift_rotated_bit_exact_every_256_steps():
    """The same drift, fed the oracle's own rotations (identical fp32 inputs on both sides):
    the appended index and the search at every 256th step equal the oracle's bit for bit."""
    sp = workload.spec("drift_32k")
    w = workload.generate_drift(sp, steps=STEPS)
    H, n0, k = sp.num_kv_heads, sp.n, sp.k
    y_pre, kn_pre = rotate_all(w.prefill, w.signs)                  # [H, n0, d], [H, n0]
    y_app, kn_app = rotate_all(w.appended, w.signs)                 # [T, H, d], [T, H]
    qt, qn = rotate_all(w.queries, w.signs)                         # [T, H, d], [T, H]
    cfg = pk.config(batch=1, num_kv_heads=H, group=1, capacity=n0 + STEPS, dtype="f32",
                    rho=sp.rho, cand_bp=sp.cand_bp)
    t_ = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(DEV)
    ix = pk.build_index_rotated(cfg, w.signs, t_(y_pre[None]), t_(kn_pre[None]))
    ya, ka, qa, qna = t_(y_app), t_(kn_app), t_(qt), t_(qn)
    check = list(range(0, STEPS, 256)) + [STEPS - 1]
    got = {}
    for t in range(STEPS):
        ix.append_rotated(ya[t].view(1, H, 1, 128), ka[t].view(1, H, 1))
        idx, est = ix.search_rotated(qa[t].view(1, H, 128), qna[t].view(1, H), k)
        if t in check:
            got[t] = (idx.cpu().numpy(), est.cpu().numpy())
    ix.sync()

    p = oracle.SearchParams(m=8, rho=sp.rho, cand_bp=sp.cand_bp)
    encs = [oracle.encode_rotated(np.concatenate([y_pre[h], y_app[:, h]]),
                                  np.concatenate([kn_pre[h], kn_app[:, h]]), 8) for h in range(H)]
    gids, gcodes, gfac = ix.export_index()
    for h in range(H):
        np.testing.assert_array_equal(gids[h], encs[h].ids)
        np.testing.assert_array_equal(gcodes[h], encs[h].codes)
        np.testing.assert_array_equal(gfac[h].view(np.uint32), encs[h].factor.view(np.uint32))
    for t in check:
        m = n0 + t + 1
        for h in range(H):
            e = encs[h]
            enc_t = oracle.Encoded(e.ids[:m], e.mag[:m], e.neg[:m], e.factor[:m])
            o_idx, _, o_est, _, _ = oracle.search_rotated(enc_t, qt[t, h], float(qn[t, h]), k, p)
            np.testing.assert_array_equal(got[t][0][h], o_idx, err_msg=f"step {t} head {h}")
            np.testing.assert_array_equal(got[t][1][h].view(np.uint32), o_est.view(np.uint32),
                                          err_msg=f"step {t} head {h}")
