"""Helpers for the GPU parity tests: numpy uint32 <-> torch CUDA tensors,
contexts, and oracle-generated keys (test code only)."""
from __future__ import annotations

import numpy as np

from key_switching_b200 import synth


def dev(a: np.ndarray):
    import torch
    a = np.ascontiguousarray(a, dtype=np.uint32)
    return torch.from_numpy(a.view(np.int32)).cuda()


def host(t) -> np.ndarray:
    return t.cpu().numpy().view(np.uint32)


def empty(*shape):
    import torch
    return torch.empty(shape, dtype=torch.int32, device="cuda")


def filled(*shape, value=0x7FFFFFFF):
    """Device buffer pre-filled with a value no canonical residue takes in a
    stored result unless the kernel wrote it (catches unwritten outputs)."""
    import torch
    return torch.full(shape, value, dtype=torch.int32, device="cuda")


def contexts(oracle, logN, L, alpha, bits):
    from key_switching_b200 import pc
    pr = oracle.gen_primes(logN, bits, L + alpha)
    P = oracle.Params(logN, pr[alpha:], pr[:alpha])
    C = pc.Context(logN, [int(v) for v in P.q], [int(v) for v in P.p])
    return P, C


def real_key(oracle, P, kind="rot", seed=0, r=1, hw=None):
    """Secret s, s' and the oracle's key 'b' half for s' -> s."""
    s = synth.ternary_secret(P.N, seed, hw)
    if kind == "square":
        sp = oracle.negacyclic_mul(s, s, P.logN)
    else:
        sp = oracle.automorph(s, P.logN, oracle.galois_elt(r, P.logN))
    e = synth.gaussian_errors(P.dnum, P.N, seed)
    kseed = synth.chacha_seed(seed, r)
    b = oracle.ksk_gen(P, s, sp, e, kseed)
    return s, sp, e, kseed, b


def random_key(P, seed=0):
    """A 'b' half of uniform residues (any b defines the same function)."""
    prim = [P.prime(g) for g in range(P.L + P.alpha)]
    b = np.stack([synth.uniform_residues(prim, P.N, seed, 0xB, j) for j in range(P.dnum)])
    return synth.chacha_seed(seed, 77), b


def oracle_map(oracle, P, calls):
    """Run independent oracle calls [(fn, args), ...] on the host's cores and
    return their results in order.  The oracle's C entry points run without
    the GIL (ctypes), so threads run them in parallel; the psi memo is filled
    first so the threads only read it."""
    from concurrent.futures import ThreadPoolExecutor
    import os
    for g in range(P.L + P.alpha):
        oracle.min_psi(P.prime(g), P.logN)
    with ThreadPoolExecutor(max_workers=max(1, min(len(calls), os.cpu_count() or 1))) as ex:
        futs = [ex.submit(fn, *args) for fn, args in calls]
        return [f.result() for f in futs]
