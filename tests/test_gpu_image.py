"""Index images (pariskv_export / pariskv_import, include/pariskv.h): an imported index is the
exported one -- identical stored ids, codes and factors, bit-identical searches, and appends
after the import give the same index as appends to the original."""
import numpy as np
import pytest
import torch

from long_context_kv_srht_b200 import pariskv as pk
from long_context_kv_srht_b200 import workload

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _keys(sp, n):
    w = workload.generate(workload.spec(sp.name, n=n, batch=sp.batch))
    conv = (lambda a: torch.from_numpy(workload.bf16_bits(a)).view(torch.bfloat16)) \
        if sp.dtype == "bf16" else (lambda a: torch.from_numpy(np.ascontiguousarray(a)))
    return w, conv(w.keys).to(DEV), conv(w.queries).to(DEV)


@pytest.mark.parametrize("name,n,extra", [("tiny", 9000, 700), ("llama3_8b_128k", 20000, 333),
                                          ("tiny", 0, 50)])
def test_export_import_round_trip(name, n, extra):
    sp = workload.spec(name, n=max(n, 1))
    w, keys, qs = _keys(sp, n + extra)
    cfg = pk.config(batch=sp.batch, num_kv_heads=sp.num_kv_heads, group=sp.group,
                    capacity=n + extra, dtype=sp.dtype, rho=sp.rho, cand_bp=sp.cand_bp)
    a = pk.build_index(cfg, w.signs, keys, n=n)
    img = a.export_image()
    assert img.nbytes == 256 + sp.batch * sp.num_kv_heads * n * 144
    b = pk.import_index(img, capacity=n + extra)
    assert b.size == n
    if n:
        for x, y in zip(a.export_index(), b.export_index()):
            np.testing.assert_array_equal(x, y)
        k = min(sp.k, n)
        ia, ea = a.search(qs, k)
        ib, eb = b.search(qs, k)
        np.testing.assert_array_equal(ia.cpu().numpy(), ib.cpu().numpy())
        np.testing.assert_array_equal(ea.cpu().numpy().view(np.uint32),
                                      eb.cpu().numpy().view(np.uint32))
    a.append(keys[:, :, n:n + extra])
    b.append(keys[:, :, n:n + extra])
    for x, y in zip(a.export_index(), b.export_index()):
        np.testing.assert_array_equal(x, y)
    ia, _ = a.search(qs, min(sp.k, n + extra))
    ib, _ = b.search(qs, min(sp.k, n + extra))
    np.testing.assert_array_equal(ia.cpu().numpy(), ib.cpu().numpy())
    # a second image of the grown index equals the first one's header fields and grows by
    # exactly the appended keys
    img2 = b.export_image()
    assert img2.nbytes == img.nbytes + sp.batch * sp.num_kv_heads * extra * 144
    assert bytes(img2[:104]) == bytes(img[:104])


def test_import_capacity_rules():
    sp = workload.spec("tiny", n=300)
    w, keys, qs = _keys(sp, 300)
    cfg = pk.config(batch=sp.batch, num_kv_heads=sp.num_kv_heads, group=sp.group,
                    capacity=300, dtype=sp.dtype)
    img = pk.build_index(cfg, w.signs, keys).export_image()
    b = pk.import_index(img)                      # capacity 0: exactly the image's size
    assert b.size == 300
    with pytest.raises(pk.PariskvError) as e:
        b.append(keys[:, :, :1])
    assert e.value.status == pk.ECAPACITY
    with pytest.raises(pk.PariskvError) as e:
        pk.import_index(img, capacity=299)
    assert e.value.status == pk.EINVAL


def test_cache_index_image():
    """The Retrieval index of a four-region cache exports like any other index."""
    rng = np.random.default_rng(3)
    K = workload.bf16_round(rng.standard_normal((1, 2, 3000, 128)).astype(np.float32))
    conv = lambda a: torch.from_numpy(workload.bf16_bits(a)).view(torch.bfloat16).to(DEV)
    signs = np.where(rng.integers(0, 2, 128) == 1, -1, 1).astype(np.int8)
    cfg = pk.config(batch=1, num_kv_heads=2, group=2, capacity=1, dtype="bf16")
    cache = pk.Cache(cfg, signs, 4, 256, 64, 32, retrieval_capacity=3000)
    cache.prefill(conv(K), conv(K), n=3000)
    ix = cache.index()
    b = pk.import_index(ix.export_image())
    assert b.size == 3000 - 4 - 256
    ref = pk.build_index(pk.config(batch=1, num_kv_heads=2, group=2, capacity=3000,
                                   dtype="bf16"), signs, conv(K)[:, :, 4:2744])
    for x, y in zip(b.export_index(), ref.export_index()):
        np.testing.assert_array_equal(x, y)
    cache.destroy()
