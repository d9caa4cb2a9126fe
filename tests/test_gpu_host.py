"""GPU parity of pc_keyswitch_host (ciphertexts and results in host memory,
copies pipelined with the key switches through two device staging slots):
every ciphertext bit-exact with the oracle at N=2^12, with pageable numpy and
page-locked torch buffers, n = 1 and n > 2 (slot reuse); at N=2^16 against
the device-buffer call."""
import numpy as np
import pytest

from key_switching_b200 import synth
from tests import gpu_util as G

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def built():
    from key_switching_b200 import build
    build.build()


def _cts(P, n, l, tag):
    return np.stack([np.stack([synth.uniform_residues(P.q[:l], P.N, tag, k, h) for h in range(2)])
                     for k in range(n)])


@pytest.mark.parametrize("n,l,pinned", [(5, 4, False), (1, 3, False), (4, 4, True)])
def test_keyswitch_host_n12(built, oracle, n, l, pinned):
    import torch
    from key_switching_b200 import pc
    P, C = G.contexts(oracle, 12, 4, 2, 30)
    keys = [G.random_key(P, 400 + k) for k in range(n)]
    kk = [pc.KSK(s, G.dev(b)) for s, b in keys]
    C.ensure_host_workspace(l)
    ct = _cts(P, n, l, 70 + l)
    if pinned:
        h_ct = torch.from_numpy(ct.view(np.int32)).pin_memory()
        h_out = torch.full(ct.shape, 0x7FFFFFFF, dtype=torch.int32).pin_memory()
    else:
        h_ct = ct.copy()
        h_out = np.full(ct.shape, 0x7FFFFFFF, dtype=np.uint32)
    C.keyswitch_host(h_ct, n, l, kk, h_out)
    torch.cuda.synchronize()
    got = h_out.numpy().view(np.uint32) if pinned else h_out
    for k in range(n):
        w0, w1 = oracle.keyswitch(P, ct[k, 0], ct[k, 1], l, keys[k][0], keys[k][1])
        assert np.array_equal(got[k, 0], w0), k
        assert np.array_equal(got[k, 1], w1), k
    C.check()


def test_keyswitch_host_n16_matches_device_call(built, oracle):
    import torch
    from key_switching_b200 import pc
    P, C = G.contexts(oracle, 16, 24, 4, 31)
    l, n = 24, 3
    keys = [G.random_key(P, 500 + k) for k in range(n)]
    kk = [pc.KSK(s, G.dev(b)) for s, b in keys]
    C.ensure_host_workspace(l)
    ct = _cts(P, n, l, 9)
    h_ct = torch.from_numpy(ct.view(np.int32)).pin_memory()
    h_out = torch.empty(ct.shape, dtype=torch.int32).pin_memory()
    C.keyswitch_host(h_ct, n, l, kk, h_out)
    torch.cuda.synchronize()
    got = h_out.numpy().view(np.uint32)
    w0, w1 = oracle.keyswitch(P, ct[0, 0], ct[0, 1], l, keys[0][0], keys[0][1])
    assert np.array_equal(got[0, 0], w0) and np.array_equal(got[0, 1], w1)
    for k in range(1, n):
        o0, o1 = G.empty(l, P.N), G.empty(l, P.N)
        C.keyswitch(G.dev(ct[k, 0]), G.dev(ct[k, 1]), l, kk[k], o0, o1)
        assert np.array_equal(got[k, 0], G.host(o0)) and np.array_equal(got[k, 1], G.host(o1)), k


def test_keyswitch_host_errors(built, oracle):
    from key_switching_b200 import pc
    P, C = G.contexts(oracle, 12, 4, 2, 30)
    seed, b = G.random_key(P, 5)
    key = pc.KSK(seed, G.dev(b))
    ct = np.zeros((2, 2, 4, P.N), dtype=np.uint32)
    out = np.zeros_like(ct)
    C.ensure_workspace(4)  # the key switch's workspace only: no staging slots
    if C.workspace_bytes(4, 1) < C.host_workspace_bytes(4):
        with pytest.raises(pc.PCError) as ei:
            C.keyswitch_host(ct, 2, 4, [key, key], out)
        assert ei.value.code == -7
    C.ensure_host_workspace(4)
    with pytest.raises(pc.PCError) as ei:
        C.keyswitch_host(ct, 2, 4, [key, key], ct)  # out over the input
    assert ei.value.code == -1
    with pytest.raises(pc.PCError) as ei:
        C.keyswitch_host(ct, 2, 5, [key, key], out)  # level above L
    assert ei.value.code == -1
    C.check()
