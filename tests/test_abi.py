"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/pc.h declares, and its host-only calls and argument
validation behave as documented."""
import ctypes
import os
import re

import numpy as np
import pytest

from tests.conftest import ROOT


def _declared():
    src = open(os.path.join(ROOT, "include", "pc.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pc_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def pc():
    from key_switching_b200 import build, pc as pcmod
    build.build()
    return pcmod


def test_exports_every_declared_symbol(pc):
    lib = pc.lib()
    names = _declared()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(pc.EXPORTS)


def test_gen_primes_matches_oracle(pc, oracle):
    for logN, bits, count in [(10, 30, 8), (12, 30, 6), (16, 31, 28), (17, 31, 45)]:
        assert pc.gen_primes(logN, bits, count) == [int(v) for v in oracle.gen_primes(logN, bits, count)]


def _params(pc, logN, q, p, dnum=None):
    qa = (ctypes.c_uint32 * len(q))(*q)
    pa = (ctypes.c_uint32 * len(p))(*p)
    d = dnum if dnum is not None else -(-len(q) // len(p))
    return pc._Params(logN, len(q), len(p), d, qa, pa), (qa, pa)


def test_ctx_create_rejects_bad_params_before_touching_cuda(pc):
    q, p = pc.chain(12, 30, 4, 2)
    h = ctypes.c_void_p()
    lib = pc.lib()
    prm, keep = _params(pc, 12, q, p, dnum=3)          # dnum != ceil(L/alpha)
    assert lib.pc_ctx_create(ctypes.byref(prm), 0, ctypes.byref(h)) == -1
    prm, keep = _params(pc, 9, q, p)                   # logN out of range
    assert lib.pc_ctx_create(ctypes.byref(prm), 0, ctypes.byref(h)) == -1
    prm, keep = _params(pc, 12, q[:3] + [q[3] + 2], p)  # not prime
    assert lib.pc_ctx_create(ctypes.byref(prm), 0, ctypes.byref(h)) == -6
    prm, keep = _params(pc, 12, q[:3] + [q[0]], p)       # repeated
    assert lib.pc_ctx_create(ctypes.byref(prm), 0, ctypes.byref(h)) == -6
    # 1 mod 2^13 (N=2^12) but not 1 mod 2^14: not NTT-friendly for N=2^13
    bad = next(int(v) for v in q if (int(v) - 1) % (1 << 14))
    prm, keep = _params(pc, 13, [bad], [p[0]])
    assert lib.pc_ctx_create(ctypes.byref(prm), 0, ctypes.byref(h)) == -6


def test_strerror_and_null_args(pc):
    lib = pc.lib()
    for code in (0, -1, -2, -3, -4, -6, -7, -8, -9):
        assert len(pc.strerror(code)) >= 2
    assert pc.strerror(-9) != pc.strerror(-100)  # -9 is a known code
    assert lib.pc_ntt_fwd(None, None, 0, 1, 1, None) == -1
    assert lib.pc_timeline_read(None, None, 0) == -1
    assert lib.pc_keyswitch(None, None, None, 1, None, None, None, None) == -1
    assert lib.pc_workspace_bytes(None, 1, 1) == 0
    assert lib.pc_gen_primes(16, 40, 1, (ctypes.c_uint32 * 1)()) == -1
