"""Host-side checks of the C ABI that need no GPU: the library loads, exports every symbol
the headers declare, and rejects invalid configurations before touching the device."""
import ctypes
import subprocess

import pytest

from long_context_kv_srht_b200 import build as kbuild
from long_context_kv_srht_b200 import pariskv as pk


def test_library_exports_every_declared_symbol():
    declared = pk.declared_symbols()
    assert len(declared) >= 17
    out = subprocess.run(["nm", "-D", "--defined-only", kbuild.LIB], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [s for s in declared if s not in exported]
    assert not missing, missing
    # nothing but the C ABI is exported
    assert all(s.startswith("pariskv_") for s in exported), sorted(exported)
    for s in declared:
        assert hasattr(pk.lib, s)


def test_config_default():
    c = pk.config()
    assert (c.d, c.B, c.m, c.rho, c.w_rank1, c.w_rest, c.cand_bp) == (128, 16, 8, 4, 2, 1, 500)
    assert ctypes.sizeof(pk.Config) == 88


@pytest.mark.parametrize("field,value", [("d", 64), ("m", 4), ("B", 8), ("rho", 0), ("rho", 257),
                                         ("w_rank1", 4), ("w_rest", 3), ("cand_bp", 0),
                                         ("cand_bp", 10001), ("batch", 0), ("group", 0),
                                         ("capacity", -1), ("dtype", 7), ("levels", 3)])
def test_invalid_config_rejected(field, value):
    c = pk.config(capacity=10)
    setattr(c, field, value)
    h = ctypes.c_void_p()
    st = pk.lib.pariskv_build_index(ctypes.byref(c), None, None, 0, 0, None, ctypes.byref(h))
    assert st == pk.EINVAL
    assert h.value is None
    assert pk.last_error()


def test_too_many_heads_rejected():
    c = pk.config(batch=1024, num_kv_heads=8, group=8, capacity=10)
    h = ctypes.c_void_p()
    assert pk.lib.pariskv_build_index(ctypes.byref(c), None, None, 0, 0, None,
                                      ctypes.byref(h)) == pk.EINVAL


def test_status_strings_and_null_handles():
    for s in range(6):
        assert pk.lib.pariskv_status_string(s)
    assert pk.lib.pariskv_size(None) == -1
    assert pk.lib.pariskv_destroy(None) == pk.OK
    assert pk.lib.pariskv_search(None, None, 1, None, None, None) == pk.EINVAL
    # the debug hooks refuse a NULL index before touching the device
    assert pk.lib.pariskv_debug_inject_wait_timeout(None) == pk.EINVAL
    assert pk.lib.pariskv_debug_inject_bad_candidate(None, 0, 0, -2) == pk.EINVAL
    assert pk.lib.pariskv_debug_set_launch(None, 0, 0, 0) == pk.EINVAL
    assert pk.lib.pariskv_debug_gather_candidates(None, None, None) == pk.EINVAL


# ------------------------------------------------------------------ index images (host checks)
def _header(n=5, units=2, version=2, magic=b"PARISKV\0", **cfg_kw):
    """A 256-byte image header laid out as include/pariskv.h describes it."""
    import numpy as np
    cfg = pk.config(batch=1, num_kv_heads=units, capacity=max(n, 1), **cfg_kw)
    h = bytearray(256)
    h[0:8] = magic
    h[8:12] = int(version).to_bytes(4, "little")
    h[12:16] = (256).to_bytes(4, "little")
    h[16:104] = bytes(cfg)
    h[104:112] = int(n).to_bytes(8, "little", signed=True)
    h[112:116] = int(units).to_bytes(4, "little", signed=True)
    h[120:248] = np.ones(128, np.int8).tobytes()
    return bytes(h)


@pytest.mark.parametrize("case", ["short", "magic", "version", "units", "truncated",
                                  "capacity", "config"])
def test_import_rejects_bad_images_on_the_host(case):
    """pariskv_import validates the image before any device work, so these run without a GPU."""
    n, units = 5, 2
    body = bytes(units * n * 144)
    img, cap = _header(n, units) + body, 0
    if case == "short":
        img = img[:100]
    elif case == "magic":
        img = _header(n, units, magic=b"PARISKW\0") + body
    elif case == "version":
        img = _header(n, units, version=3) + body
    elif case == "units":
        img = _header(n, 3) + body          # header says 3 units, config says 3 KV heads
        img = img[:16] + bytes(pk.config(batch=1, num_kv_heads=2, capacity=5)) + img[104:]
    elif case == "truncated":
        img = img[:-1]
    elif case == "capacity":
        cap = n - 1
    elif case == "config":
        img = _header(n, units, rho=0) + body
    h = ctypes.c_void_p()
    st = pk.lib.pariskv_import(img, len(img), cap, None, ctypes.byref(h))
    assert st == pk.EINVAL and not h.value, pk.last_error()


def test_import_accepts_a_well_formed_image_up_to_the_device():
    """A well-formed image passes every host check; without a GPU the call then fails in the
    device allocation (ECUDA or ENOMEM), not in validation."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is visible: the import would succeed (covered by the GPU tests)")
    img = _header(5, 2) + bytes(2 * 5 * 144)
    h = ctypes.c_void_p()
    st = pk.lib.pariskv_import(img, len(img), 0, None, ctypes.byref(h))
    assert st in (pk.ECUDA, pk.ENOMEM) and not h.value, (st, pk.last_error())


def test_prior_levels_match_the_oracle():
    """The library's prior-derived levels (its own quadrature and Lloyd-Max iteration, host
    code) agree with the oracle's derivation of the same law."""
    import numpy as np
    import oracle
    np.testing.assert_allclose(pk.prior_levels(), oracle.ratio_levels(), atol=1e-6)


@pytest.mark.parametrize("table", [[0.1, 0.2, 0.3, 0.3, 0.5, 0.6, 0.7, 0.8],
                                   [-0.1, 0.2, 0.3, 0.4, 0.5, 0.6, 0.7, 0.8],
                                   [0.1, 0.2, 0.3, float("nan"), 0.5, 0.6, 0.7, 0.8]])
def test_invalid_level_table_rejected(table):
    import numpy as np
    c = pk.config(capacity=10, levels="table", level_table=table)
    signs = np.ones(128, np.int8)
    h = ctypes.c_void_p()
    st = pk.lib.pariskv_build_index(ctypes.byref(c), signs.ctypes.data, None, 0, 0, None,
                                    ctypes.byref(h))
    assert st == pk.EINVAL and not h.value and "level_table" in pk.last_error()


@pytest.mark.parametrize("cc", [(-1, 8, 4, 4, 16), (2, 4, 8, 4, 16), (2, 8, 0, 4, 16),
                                (2, 8, 4, 0, 16), (2, 8, 4, 4, 0)])
def test_cache_config_rejected_on_the_host(cc):
    """pariskv_cache_create validates the region sizes before it touches the device."""
    import numpy as np
    cfg = pk.config(capacity=1)
    ccfg = pk.CacheConfig(*cc)
    signs = np.ones(128, np.int8)
    h = ctypes.c_void_p()
    st = pk.lib.pariskv_cache_create(ctypes.byref(cfg), ctypes.byref(ccfg), signs.ctypes.data,
                                     None, ctypes.byref(h))
    assert st == pk.EINVAL and not h.value


@pytest.mark.parametrize("field,value", [("dtype", 0), ("group", 9)])
def test_dense_attend_config_rejected_on_the_host(field, value):
    c = pk.config(capacity=64, **{field: value})
    st = pk.lib.pariskv_dense_attend(ctypes.byref(c), None, None, None, 64, 64, 0.1, None, 0,
                                     None)
    assert st == pk.EINVAL


def test_train_centroids_arguments_rejected_on_the_host():
    import numpy as np
    c = pk.config(capacity=64)
    signs = np.ones(128, np.int8)
    bad = signs.copy()
    bad[5] = 0
    for sg, n, iters in ((bad, 10, 1), (signs, 0, 1), (signs, 10, -1), (signs, 10, 1001)):
        st = pk.lib.pariskv_train_centroids(ctypes.byref(c), sg.ctypes.data, None, 10, n, iters,
                                            None, None)
        assert st == pk.EINVAL
