"""The benchmark's accounting on the host: the candidate count it reports agrees with the
oracle's, the algorithmic bytes behind the roofline are the per-unit figures times the units
one launch processes (16 B of bucket ids per key per KV head and vote pack; one 128-byte
record per candidate per query head), the DRAM traffic figure is withheld for a kernel with
no capture, and the L2 eviction between timed steps touches two buffers larger than L2."""
import os
import sys

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from long_context_kv_srht_b200 import workload  # noqa: E402


@pytest.mark.parametrize("n,k,bp", [(1 << 20, 4096, 500), (131072, 2048, 500), (65536, 2048, 500),
                                    (33, 5, 10000), (31, 31, 500), (4096, 64, 1000), (1, 1, 500)])
def test_candidate_count_matches_the_oracle(n, k, bp):
    assert bench.candidate_count(n, k, bp) == oracle.candidate_count(n, k, bp)


def test_algorithmic_bytes_of_the_million_token_search():
    sp = workload.spec("million_offload")
    C = bench.candidate_count(sp.n, sp.k, sp.cand_bp)
    assert C == 52429
    units = sp.batch * sp.num_kv_heads
    packs = -(-sp.group // 4)
    assert bench.algorithmic_bytes("vote", sp, C) == units * packs * sp.n * 16 == 134217728
    assert bench.algorithmic_bytes("rerank", sp, C) == 32 * 52429 * 128 == 214749184
    assert bench.algorithmic_bytes("topk", sp, C) == 0


def test_algorithmic_bytes_count_vote_packs_for_wide_groups():
    sp = workload.spec("tiny", batch=2, num_kv_heads=3, group=5, n=1000)
    # a group of five query heads takes two vote packs: the ids are read once per pack
    assert bench.algorithmic_bytes("vote", sp, 100) == 2 * 3 * 2 * 1000 * 16
    assert bench.algorithmic_bytes("rerank", sp, 100) == 2 * 15 * 100 * 128


def test_traffic_is_withheld_without_a_capture():
    assert bench.kernel_traffic("no_such_kernel", "million_offload") is None
    assert bench.kernel_traffic("rerank", "no_such_workload") is None


def test_l2_eviction_buffers_exceed_l2():
    f = bench.L2Flush("cpu")
    f(7)
    assert f.w.numel() * f.w.element_size() > 126 * 10**6
    assert f.r.numel() * f.r.element_size() == f.w.numel() * f.w.element_size()
    assert int(f.w[0]) == 7 and int(f.w[-1]) == 7
    assert f.w.data_ptr() != f.r.data_ptr()
