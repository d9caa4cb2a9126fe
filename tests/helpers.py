"""Big-integer and brute-force helpers for the oracle pins (test code only).

Nothing here imports the CUDA library; everything is plain Python integers or
numpy, so that the pins do not lean on the code they check.
"""
from __future__ import annotations

from functools import reduce

import numpy as np


def prod(xs) -> int:
    return reduce(lambda a, b: a * b, (int(x) for x in xs), 1)


def crt_lift(res: np.ndarray, primes) -> np.ndarray:
    """Residues [k][N] modulo pairwise-coprime primes -> object array of the
    unique integers in [0, prod(primes))."""
    primes = [int(p) for p in primes]
    M = prod(primes)
    acc = np.zeros(res.shape[1], dtype=object)
    for r, p in zip(res, primes):
        Mi = M // p
        c = (Mi * pow(Mi, -1, p)) % M
        acc = acc + r.astype(object) * c
    return acc % M


def centered(x: np.ndarray, M: int) -> np.ndarray:
    h = M // 2
    return np.array([int(v) - M if int(v) > h else int(v) for v in x], dtype=object)


def trial_division_is_prime(n: int) -> bool:
    if n < 2:
        return False
    if n % 2 == 0:
        return n == 2
    d = 3
    while d * d <= n:
        if n % d == 0:
            return False
        d += 2
    return True


def bitrev(x: int, bits: int) -> int:
    return int(format(x, f"0{bits}b")[::-1], 2) if bits else 0


def ntt_by_definition(a, logN: int, q: int, psi: int):
    """O(N^2) evaluation a_hat[k] = sum_n a[n] psi^((2 brv(k)+1) n) mod q."""
    N = 1 << logN
    out = []
    for k in range(N):
        r = pow(psi, 2 * bitrev(k, logN) + 1, q)
        acc, x = 0, 1
        for n in range(N):
            acc += int(a[n]) * x
            x = x * r % q
        out.append(acc % q)
    return np.array(out, dtype=np.uint32)


def negacyclic_schoolbook(a, b, q: int):
    """(a*b) mod (X^N+1, q) by the O(N^2) definition, Python integers."""
    N = len(a)
    out = [0] * N
    for i in range(N):
        ai = int(a[i])
        if ai == 0:
            continue
        for j in range(N):
            k = i + j
            if k < N:
                out[k] += ai * int(b[j])
            else:
                out[k - N] -= ai * int(b[j])
    return np.array([v % q for v in out], dtype=np.uint32)


def mulmod(a: np.ndarray, b: np.ndarray, q: int) -> np.ndarray:
    return ((a.astype(np.uint64) * b.astype(np.uint64)) % np.uint64(q)).astype(np.uint32)


def addmod(a, b, q):
    return ((a.astype(np.uint64) + b.astype(np.uint64)) % np.uint64(q)).astype(np.uint32)


def submod(a, b, q):
    return ((a.astype(np.uint64) + np.uint64(q) - b.astype(np.uint64)) % np.uint64(q)).astype(np.uint32)


def reduce_signed(s: np.ndarray, q: int) -> np.ndarray:
    return np.mod(s.astype(np.int64), q).astype(np.uint32)
