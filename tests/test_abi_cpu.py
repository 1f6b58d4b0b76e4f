"""The C-ABI library: it loads, exports every symbol the header declares, and rejects bad
arguments on the host before anything reaches a GPU (these tests run without one)."""
import ctypes
import os
import re

import pytest

import oracle
from free_weight_quantization_b200 import build as fbuild
from free_weight_quantization_b200 import hqq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hqq_b200.h")


@pytest.fixture(scope="module")
def L():
    fbuild.build()
    return hqq.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(hqq_[a-z_0-9]+)\s*\(", text)))


def test_header_symbols_exported(L):
    names = declared_functions()
    assert {"hqq_quantize", "hqq_dequantize", "hqq_packed_bytes",
            "hqq_quantize_workspace_bytes", "hqq_default_opt", "hqq_strerror"} <= set(names)
    raw = ctypes.CDLL(hqq.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), n
    assert set(names) == set(hqq.SIGNATURES), "binding and header disagree"


def test_default_opt_is_the_pages_defaults(L):
    o = hqq.default_opt()
    assert (o.iters, o.lp_norm, o.beta, o.kappa) == (20, 0.7, 10.0, 1.01)
    assert abs(o.eps_tiny - 1e-4) < 1e-9 and o.scale_max == 2e4


@pytest.mark.parametrize("nbits", [1, 2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("n", [0, 1, 7, 10, 64, 4096 * 4096, 4096 * 11008 + 3])
def test_packed_bytes_match_oracle(L, nbits, n):
    assert hqq.hqq_packed_bytes(n, nbits) == oracle.packed_bytes(n, nbits)


def test_packed_bytes_rejects(L):
    assert hqq.hqq_packed_bytes(10, 9) == -1
    assert hqq.hqq_packed_bytes(10, 0) == -1
    assert hqq.hqq_packed_bytes(-1, 4) == -1


def test_workspace_bytes(L):
    ws = hqq.hqq_quantize_workspace_bytes
    assert ws(4096, 4096, 4, 64, 1, 20) > 0
    # small: round sums + 1 byte per group (its last round)
    G = 4096 * 4096 // 64
    assert G <= ws(4096, 4096, 4, 64, 1, 20) < G + 65536
    assert ws(10, 10, 4, 3, 1, 20) == 0        # 100 % 3 != 0
    assert ws(16, 16, 9, 16, 1, 20) == 0       # 9 bits
    assert ws(16, 16, 0, 16, 1, 20) == 0       # 0 bits
    assert ws(16, 16, 5, 16, 1, 20) > 0        # 5 bits: the tile engine
    assert ws(16, 16, 4, 16, 2, 20) == 0       # axis 2
    assert ws(16, 1024, 4, 512, 1, 20) == 0    # group beyond the library limit
    assert ws(16, 16, 4, 16, 1, 65) == 0       # iters beyond the library limit
    # axis=0 whose packed words do not line up with tiles needs byte staging of all codes
    assert ws(8, 6, 4, 2, 0, 20) >= 48
    # a small stream-engine tensor (at most 16384 groups) also keeps each group's zero after
    # every update, G x iters binary32; a large one, the tile engine and iters = 0 do not
    small = ws(256, 512, 4, 64, 1, 20)
    assert small >= 2048 * 20 * 4
    assert ws(256, 512, 4, 64, 1, 10) <= small - 2048 * 10 * 4
    assert ws(256, 512, 3, 64, 1, 20) < 2048 * 20 * 4      # 3 bit: the tile engine
    assert ws(256, 512, 4, 64, 1, 0) < 2048 * 4
    assert ws(4096, 4096, 4, 64, 1, 20) < G + 65536          # 262144 groups: none


FAKE = 0x10000  # never dereferenced: every call below fails its host-side checks first


def q(L, W=FAKE, rows=64, cols=64, nbits=4, g=64, axis=1, opt=None, packed=FAKE, scale=FAKE,
      zero=FAKE, ws=FAKE, wsb=1 << 20, iters_run=None):
    P = ctypes.c_void_p
    return L.hqq_quantize(P(W), rows, cols, nbits, g, axis, opt, P(packed), P(scale), P(zero),
                          P(iters_run) if iters_run else None, None, None, None, None, P(ws), wsb,
                          None)


def test_quantize_rejects_on_host(L):
    assert q(L, nbits=9) == 1
    assert q(L, nbits=0) == 1
    assert q(L, axis=3) == 1
    assert q(L, g=0) == 1
    assert q(L, rows=0) == 1
    assert q(L, cols=-4) == 1
    assert q(L, g=48) == 1                     # 4096 % 48 != 0
    assert q(L, rows=2, cols=512, g=512) == 5  # group_size > 256
    assert q(L, W=0) == 1
    assert q(L, packed=0) == 1
    assert q(L, W=FAKE + 2) == 2               # W not 16-byte aligned
    assert q(L, packed=FAKE + 4) == 2
    assert q(L, scale=FAKE + 1) == 2
    assert q(L, iters_run=FAKE + 2) == 2
    assert q(L, ws=0) == 3
    assert q(L, wsb=16) == 3
    assert q(L, ws=FAKE + 8) == 2
    for field, bad in [("lp_norm", 0.0), ("lp_norm", 2.0), ("beta", 0.0), ("kappa", -1.0),
                       ("scale_max", 0.0), ("eps_tiny", -1.0), ("iters", -1), ("iters", 65)]:
        o = hqq.default_opt()
        setattr(o, field, bad)
        rc = q(L, opt=ctypes.byref(o))
        assert rc == (5 if (field, bad) == ("iters", 65) else 1), (field, bad, rc)


def test_dequantize_rejects_on_host(L):
    P = ctypes.c_void_p
    d = L.hqq_dequantize
    assert d(P(FAKE), P(FAKE), P(FAKE), 64, 64, 9, 64, 1, P(FAKE), None) == 1
    assert d(P(FAKE), P(FAKE), P(FAKE), 64, 64, 4, 63, 1, P(FAKE), None) == 1
    assert d(None, P(FAKE), P(FAKE), 64, 64, 4, 64, 1, P(FAKE), None) == 1
    assert d(P(FAKE + 4), P(FAKE), P(FAKE), 64, 64, 4, 64, 1, P(FAKE), None) == 2
    assert d(P(FAKE), P(FAKE), P(FAKE), 64, 64, 4, 64, 1, P(FAKE + 2), None) == 2


def test_strerror(L):
    for code in range(6):
        assert L.hqq_strerror(code)
    assert L.hqq_strerror(99) == b"unknown error"


def test_gemv_rejects_on_host(L):
    P = ctypes.c_void_p
    gv = L.hqq_gemv
    args = lambda **k: dict(dict(pk=FAKE, sc=FAKE, ze=FAKE, rows=64, cols=64, nb=4, g=64, ax=1,
                                 x=FAKE, y=FAKE), **k)

    def call(**k):
        a = args(**k)
        return gv(P(a["pk"]), P(a["sc"]), P(a["ze"]), a["rows"], a["cols"], a["nb"], a["g"],
                  a["ax"], P(a["x"]) if a["x"] else None, P(a["y"]) if a["y"] else None, None)
    assert call(nb=9) == 1
    assert call(nb=0) == 1
    assert call(g=48) == 1                 # 4096 % 48 != 0
    assert call(ax=2) == 1
    assert call(x=0) == 1
    assert call(y=0) == 1
    assert call(pk=FAKE + 4) == 2          # packed not 16-byte aligned
    assert call(x=FAKE + 1) == 2
    assert call(y=FAKE + 2) == 2


def test_binding_arity_matches_the_header():
    # every prototype's parameter count equals the binding's ctypes argtypes
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    protos = dict(re.findall(r"\b(hqq_[a-z_0-9]+)\s*\(([^)]*)\)\s*;", text))
    assert set(protos) == set(hqq.SIGNATURES)
    for name, params in protos.items():
        n = 0 if params.strip() in ("", "void") else params.count(",") + 1
        assert n == len(hqq.SIGNATURES[name][1]), (name, n, len(hqq.SIGNATURES[name][1]))


def test_shrink_rejects_bad_arguments(L):
    # host-side checks only: nothing reaches a device
    assert L.hqq_shrink_lp(None, 0, 10.0, 0.7, None, None) == 0
    assert L.hqq_shrink_lp(None, -1, 10.0, 0.7, None, None) == 1
    assert L.hqq_shrink_lp(ctypes.c_void_p(16), 4, 0.0, 0.7, ctypes.c_void_p(16), None) == 1
    assert L.hqq_shrink_lp(ctypes.c_void_p(16), 4, 10.0, 0.0, ctypes.c_void_p(16), None) == 1
    assert L.hqq_shrink_lp(None, 4, 10.0, 0.7, None, None) == 1
    assert L.hqq_shrink_lp(ctypes.c_void_p(18), 4, 10.0, 0.7, ctypes.c_void_p(16), None) == 2


def test_noalloc_scratch_size_binding_matches_the_header():
    import os
    import re
    text = open(os.path.join(ROOT, "include", "hqq_b200.h")).read()
    m = re.search(r"#define\s+HQQ_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", text)
    assert m, "HQQ_NOALLOC_SCRATCH_BYTES not found in the header"
    assert hqq.HQQ_NOALLOC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))
