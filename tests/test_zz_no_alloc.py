"""pc_modup_noalloc: ModUp for callers that cannot allocate device memory.

A plugin inside a host framework that owns every device allocation, or a
latency-critical path that cannot afford cudaMalloc, cannot hand the library a
workspace.  pc_modup_noalloc computes what pc_modup computes with its scratch
in a static device array of the library instead.  This test calls it through
the C ABI and checks that its output equals pc_modup's bit for bit (the
library's tolerance for integer results) on two calls in a row, that a size
beyond its static scratch is refused, and that it needs no workspace.

The file is named so that pytest collects it last: the calls share one
static array for the whole process, so these checks must hold after every
other test has run in the same process (and they must also hold when the file
runs alone in a fresh process); a run that stops at the first failure has
then already run every other test.
"""
import ctypes

import numpy as np
import pytest

from key_switching_b200 import synth
from tests import gpu_util as G

pytestmark = pytest.mark.gpu


def _noalloc(pc, ctx, c1, l, ext):
    lib = pc.lib()
    stream = ctypes.c_void_p(None)
    return lib.pc_modup_noalloc(ctx._h, ctypes.c_void_p(c1.data_ptr()), l,
                                ctypes.c_void_p(ext.data_ptr()), stream)


@pytest.mark.parametrize("logN,L,alpha,bits,l", [(12, 4, 2, 30, 4), (16, 24, 4, 31, 24), (16, 24, 4, 31, 9),
                                                   (16, 32, 4, 31, 32), (17, 16, 4, 31, 16)])
def test_noalloc_matches_modup_twice(oracle, logN, L, alpha, bits, l):
    import torch
    from key_switching_b200 import build, pc
    build.build()
    P, C = G.contexts(oracle, logN, L, alpha, bits)
    beta = -(-l // alpha)
    C.set_workspace(None)
    for call in range(2):
        c1 = synth.uniform_residues(P.q[:l], P.N, 123, call, l)
        d1 = G.dev(c1)
        got = G.filled(beta, l + alpha, P.N)
        assert _noalloc(pc, C, d1, l, got) == 0  # no workspace is set
        torch.cuda.synchronize()
        C.ensure_workspace(l)
        want = G.filled(beta, l + alpha, P.N)
        C.modup(d1, l, want)
        C.set_workspace(None)
        assert np.array_equal(G.host(got), G.host(want)), call
    C.check()


def test_noalloc_rejects_sizes_beyond_its_scratch(oracle):
    from key_switching_b200 import pc
    P, C = G.contexts(oracle, 16, 34, 4, 31)
    l = 33  # 33 * 2^16 words > 2^21 (32 * 2^16 = 2^21 is the largest accepted)
    c1 = G.empty(l, P.N)
    ext = G.empty(-(-l // 4), l + 4, P.N)
    assert _noalloc(pc, C, c1, l, ext) == -8
    assert "static scratch" in pc.strerror(-8)
