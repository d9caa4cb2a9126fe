"""GPU parity of the CUDA-graph replay of a key switch (pc_keyswitch_capture /
pc_graph_launch): the graph, replayed on new data written into the captured
buffers, gives exactly the oracle's result each time (N=2^12), and the direct
call's result at the N=2^16 workload's size."""
import numpy as np
import pytest

from key_switching_b200 import synth
from tests import gpu_util as G

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def built():
    from key_switching_b200 import build
    build.build()


def test_graph_replays_match_oracle_n12(built, oracle):
    import torch
    from key_switching_b200 import pc
    P, C = G.contexts(oracle, 12, 4, 2, 30)
    l = 4
    C.ensure_workspace(l)
    seed, b = G.random_key(P, 21)
    key = pc.KSK(seed, G.dev(b))
    d0, d1 = G.empty(l, P.N), G.empty(l, P.N)
    o0, o1 = G.filled(l, P.N), G.filled(l, P.N)
    graph = C.keyswitch_capture(d0, d1, l, key, o0, o1)
    for rep in range(3):
        c0 = synth.uniform_residues(P.q, P.N, 90 + rep, 0)
        c1 = synth.uniform_residues(P.q, P.N, 90 + rep, 1)
        d0.copy_(G.dev(c0))
        d1.copy_(G.dev(c1))
        graph.launch()
        torch.cuda.synchronize()
        w0, w1 = oracle.keyswitch(P, c0, c1, l, seed, b)
        assert np.array_equal(G.host(o0), w0) and np.array_equal(G.host(o1), w1), rep
    graph.close()
    C.check()


def test_graph_matches_direct_call_n16(built, oracle):
    import torch
    from key_switching_b200 import pc
    P, C = G.contexts(oracle, 16, 24, 4, 31)
    l = 24
    C.ensure_workspace(l)
    seed, b = G.random_key(P, 22)
    key = pc.KSK(seed, G.dev(b))
    d0 = G.dev(synth.uniform_residues(P.q, P.N, 95, 0))
    d1 = G.dev(synth.uniform_residues(P.q, P.N, 95, 1))
    g0, g1 = G.empty(l, P.N), G.empty(l, P.N)
    graph = C.keyswitch_capture(d0, d1, l, key, g0, g1)
    graph.launch()
    graph.launch()
    o0, o1 = G.empty(l, P.N), G.empty(l, P.N)
    C.keyswitch(d0, d1, l, key, o0, o1)
    torch.cuda.synchronize()
    assert np.array_equal(G.host(g0), G.host(o0)) and np.array_equal(G.host(g1), G.host(o1))
    graph.close()


def test_capture_errors(built, oracle):
    from key_switching_b200 import pc
    P, C = G.contexts(oracle, 12, 4, 2, 30)
    seed, b = G.random_key(P, 5)
    key = pc.KSK(seed, G.dev(b))
    c = G.empty(4, P.N)
    with pytest.raises(pc.PCError) as ei:  # no workspace yet
        C.keyswitch_capture(c, c, 4, key, c, c)
    assert ei.value.code == -7
    C.ensure_workspace(4)
    with pytest.raises(pc.PCError) as ei:
        C.keyswitch_capture(c, c, 5, key, c, c)
    assert ei.value.code == -1
    C.check()


def test_general_capture_of_several_calls(built, oracle):
    """One graph holding a rotation, two hoisted rotations and a
    relinearisation (pc_capture_begin / pc_capture_end), replayed twice:
    bit-exact with the oracle."""
    import torch
    from key_switching_b200 import pc
    P, C = G.contexts(oracle, 12, 4, 2, 30)
    l = 4
    C.ensure_workspace(l, 2)
    seed, b = G.random_key(P, 23)
    key = pc.KSK(seed, G.dev(b))
    c0 = synth.uniform_residues(P.q, P.N, 96, 0)
    c1 = synth.uniform_residues(P.q, P.N, 96, 1)
    y = np.stack([synth.uniform_residues(P.q, P.N, 97, h) for h in range(2)])
    d0, d1, dy, dx = G.dev(c0), G.dev(c1), G.dev(y), G.dev(np.stack([c0, c1]))
    g = oracle.galois_elt(1, 12)
    gs = [g, oracle.galois_elt(4, 12)]
    r0, r1 = G.filled(l, P.N), G.filled(l, P.N)
    hout = G.filled(2, 2, l, P.N)
    rel = G.filled(2, l, P.N)

    def calls(st):
        C.rotate(d0, d1, l, g, key, r0, r1, st)
        C.rotate_hoisted(d0, d1, l, gs, [key, key], hout, st)
        C.relinearize(dx, dy, l, key, rel, st)
    graph = C.capture(calls, keep=(d0, d1, dx, dy, key))
    for _ in range(2):
        graph.launch()
        torch.cuda.synchronize()
        w0, w1 = oracle.rotate(P, c0, c1, l, g, seed, b)
        assert np.array_equal(G.host(r0), w0) and np.array_equal(G.host(r1), w1)
        for i, (h0, h1) in enumerate(oracle.rotate_hoisted(P, c0, c1, l, gs, [seed, seed], [b, b])):
            assert np.array_equal(G.host(hout[i, 0]), h0) and np.array_equal(G.host(hout[i, 1]), h1), i
        w0, w1 = oracle.relinearize(P, c0, c1, y[0], y[1], l, seed, b)
        assert np.array_equal(G.host(rel[0]), w0) and np.array_equal(G.host(rel[1]), w1)
    graph.close()
    C.check()
