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
    assert ctypes.sizeof(pk.Config) == 56


@pytest.mark.parametrize("field,value", [("d", 64), ("m", 4), ("B", 8), ("rho", 0), ("rho", 257),
                                         ("w_rank1", 4), ("w_rest", 3), ("cand_bp", 0),
                                         ("cand_bp", 10001), ("batch", 0), ("group", 0),
                                         ("capacity", -1), ("dtype", 7), ("reserved", 1)])
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
