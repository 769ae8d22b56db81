"""Checks that stand in for a memory checker and a race detector (no sanitizer is run):

* an out-of-range candidate index written by a test hook (as a selection bug would) is
  skipped by the rerank and reported by pariskv_sync, and no other query head changes;
* every launch shape of the vote scan, the rerank and the top-k gives the same bits (work
  split over any number of CTAs, top-k on one CTA, on a cluster, from shared or global
  memory): no result depends on scheduling;
* the guard bytes around the index's device buffers catch a write past a buffer's end (the
  autouse fixture in conftest.py checks them after every GPU test);
* the top-k's bounded wait for its bulk copies runs out when a test hook arms its barrier for
  bytes that never arrive, and the timeout reaches the caller as PARISKV_ETIMEOUT.
"""
import numpy as np
import pytest
import torch

from long_context_kv_srht_b200 import pariskv as pk
from long_context_kv_srht_b200 import workload

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _index(n, hkv=2, G=4, cand_bp=1000, seed=5):
    sp = workload.spec("llama3_8b_128k", num_kv_heads=hkv, group=G, n=n, k=256, seed=seed)
    data = workload.generate_torch(sp, DEV, n=n)
    cfg = pk.config(batch=1, num_kv_heads=hkv, group=G, capacity=n, dtype=sp.dtype, rho=4,
                    cand_bp=cand_bp)
    return pk.build_index(cfg, data["signs"], data["keys"]), data["queries"], cfg


def _candidates(n, k, cand_bp):
    return min(n, max(k, (n * cand_bp + 9999) // 10000))


def test_bad_candidate_is_reported_and_other_heads_are_unchanged():
    n, k = 20000, 256
    ix, q, cfg = _index(n)
    ref_idx, ref_est = ix.search(q, k)
    ix.sync()
    H = cfg.batch * cfg.num_q_heads
    for head, value in ((5, n + 1000), (0, -2)):
        ix.inject_bad_candidate(head, 17, value)
        idx, est = ix.search(q, k)
        with pytest.raises(pk.PariskvError) as e:
            ix.sync()
        assert e.value.status == pk.ECUDA and "out of range" in str(e.value)
        others = [h for h in range(H) if h != head]
        assert torch.equal(idx[others], ref_idx[others])
        assert torch.equal(est[others], ref_est[others])
        # the hook is consumed: the next search is clean and identical everywhere
        idx, est = ix.search(q, k)
        ix.sync()
        assert torch.equal(idx, ref_idx) and torch.equal(est, ref_est)
    # a valid key index is refused, and so is a slot past the candidate count
    with pytest.raises(pk.PariskvError):
        ix.inject_bad_candidate(1, 3, 7)
    ix.inject_bad_candidate(1, _candidates(n, k, 1000) + 5, -1)
    with pytest.raises(pk.PariskvError) as e:
        ix.search(q, k)
    assert e.value.status == pk.EINVAL
    ix.destroy()


@pytest.mark.parametrize("n,k,modes", [(60000, 256, (1, 2, 3, 4)), (60030, 256, (1, 2, 3, 4)),
                                       (200000, 512, (3, 4))])
def test_every_launch_shape_gives_the_same_bits(n, k, modes):
    # (n = 60030 gives C = 6003, so the four-CTA top-k parts start 0, 1 and 2 words past a
    # 16-byte boundary: the bulk copies' offset path)
    ix, q, cfg = _index(n)
    ref_idx, ref_est = ix.search(q, k)
    ix.sync()
    _, ref_scores, ref_cand, ref_S = ix.export_search()
    shapes = [(v, r, t) for v, r in ((1, 1), (3, 7), (1000, 500), (0, 0)) for t in modes]
    for vote_ctas, rerank_ctas, topk_mode in shapes:
        ix.set_launch(vote_ctas, rerank_ctas, topk_mode)
        idx, est = ix.search(q, k)
        ix.sync()
        shape = (vote_ctas, rerank_ctas, topk_mode)
        assert torch.equal(idx, ref_idx), shape
        assert torch.equal(est, ref_est), shape
        _, scores, cand, S = ix.export_search()
        np.testing.assert_array_equal(scores, ref_scores)
        np.testing.assert_array_equal(cand, ref_cand)
        np.testing.assert_array_equal(S.view(np.uint32), ref_S.view(np.uint32))
    # a forced top-k shape that cannot hold C is refused
    if 1 not in modes:
        ix.set_launch(0, 0, 1)
        with pytest.raises(pk.PariskvError) as e:
            ix.search(q, k)
        assert e.value.status == pk.EINVAL
    ix.destroy()


def test_guard_bytes_catch_a_write_past_a_buffer():
    import os
    if os.environ.get("PARISKV_GUARD") != "1":
        pytest.skip("guard bytes are off in this process")
    n, k = 20000, 256
    ix, q, cfg = _index(n)
    ix.search(q, k)
    ix.sync()
    pk.check_guards()                                   # intact so far
    H = cfg.batch * cfg.num_q_heads
    cmax = -(-_candidates(n, k, 1000) // 32) * 32       # the candidate rows' stride
    ix.inject_bad_candidate(H - 1, cmax, -1)            # one int past the buffer's end
    ix.search(q, k)
    ix.sync()                                           # nothing read the slot
    with pytest.raises(pk.PariskvError) as e:
        pk.check_guards()
    assert e.value.status == pk.ECUDA and "after" in str(e.value)
    # the buffer is checked again when it is freed; that report is consumed here
    ix.destroy()
    with pytest.raises(pk.PariskvError):
        pk.check_guards()
    pk.check_guards()


def test_candidate_gather_needs_a_search_and_leaves_results_alone():
    n, k = 20000, 256
    ix, q, cfg = _index(n)
    sink = torch.zeros(1, dtype=torch.int32, device=DEV)
    with pytest.raises(pk.PariskvError) as e:
        ix.gather_candidates(sink)
    assert e.value.status == pk.EINVAL
    ref_idx, ref_est = ix.search(q, k)
    ix.sync()
    ref_idx, ref_est = ref_idx.clone(), ref_est.clone()
    ix.gather_candidates(sink)
    idx, est = ix.search(q, k)
    ix.sync()
    assert torch.equal(idx, ref_idx) and torch.equal(est, ref_est)
    ix.destroy()


def test_bounded_copy_wait_runs_out_and_is_reported():
    # the hook arms the top-k's copy barrier for 16 bytes that never arrive: every CTA's wait
    # runs out after about a second, the kernel finishes, and the status word reports it
    import time
    n, k = 20000, 256
    ix, q, cfg = _index(n)
    ref_idx, ref_est = ix.search(q, k)
    ix.sync()
    ref_idx, ref_est = ref_idx.clone(), ref_est.clone()
    for mode in (0, 3):          # one CTA per head; a four-CTA cluster per head
        ix.set_launch(0, 0, mode)
        ix.inject_wait_timeout()
        t0 = time.perf_counter()
        ix.search(q, k)
        with pytest.raises(pk.PariskvError) as e:
            ix.sync()
        waited = time.perf_counter() - t0
        assert e.value.status == pk.ETIMEOUT, e.value
        assert 0.9 <= waited < 30.0, waited
        # consumed: the next search is clean and gives the reference bits
        idx, est = ix.search(q, k)
        ix.sync()
        assert torch.equal(idx, ref_idx) and torch.equal(est, ref_est)
    # a top-k that reads its part from global memory has no copy to wait for
    ix.set_launch(0, 0, 4)
    ix.inject_wait_timeout()
    with pytest.raises(pk.PariskvError) as e:
        ix.search(q, k)
    assert e.value.status == pk.EINVAL
    ix.set_launch(0, 0, 0)
    ix.search(q, k)
    ix.sync()
    ix.destroy()
