"""The C-ABI library builds, loads and exports every symbol its header
declares; host-side argument checks (no GPU needed)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    inc = os.path.join(ROOT, "include")
    for f in os.listdir(inc):
        if f.endswith(".h"):
            src = open(os.path.join(inc, f)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(indexer_[a-z_0-9]+)\s*\(", src))
    return names


@pytest.fixture(scope="module")
def lib():
    from head_weighted_relu_b200 import build
    build.build()
    return ctypes.CDLL(build.LIB)


def test_exports_every_declared_symbol(lib):
    declared = _declared()
    assert "indexer_topk" in declared and len(declared) >= 8
    for name in sorted(declared):
        assert hasattr(lib, name), name


def test_binding_covers_header():
    from head_weighted_relu_b200 import indexer as I
    assert set(I.EXPORTS) == _declared()
    assert I.indexer_abi_version() == 1


def test_out_width_and_argument_checks():
    from head_weighted_relu_b200 import indexer as I
    assert I.indexer_out_width(I.make_problem(65536, 65536, 64, 128, 2048)) == 2048
    # pooled: 2,048 budget with pools of 4 needs 2,051 slots (KPool §2)
    assert I.indexer_out_width(I.make_problem(131072, 131072, 32, 128, 2048, I.POOLED, 4)) == 2051
    assert I.indexer_out_width(I.make_problem(10, 10, 64, 128, 16, I.COMPRESSED, 4)) == 16
    bad = [
        I.make_problem(10, 10, 64, 128, 0),                  # K < 1
        I.make_problem(10, 0, 64, 128, 4),                   # no keys
        I.make_problem(10, 9, 64, 128, 4),                   # a query without its own token
        I.make_problem(8, 8, 32, 128, 6, I.POOLED, 4),       # K not a whole number of pools
        I.make_problem(10, 10, 64, 128, 4, 7),               # unknown visibility
    ]
    for p in bad:
        with pytest.raises(I.IndexerError) as e:
            I.indexer_out_width(p)
        assert e.value.status == 1
    with pytest.raises(I.IndexerError) as e:
        I.indexer_out_width(I.make_problem(10, 10, 48, 128, 4))   # no compiled variant
    assert e.value.status == 3


def test_status_strings(lib):
    lib.indexer_status_string.restype = ctypes.c_char_p
    for s in range(6):
        assert lib.indexer_status_string(s)
