"""Seeded synthetic inputs shared by the tests, the bench and the oracle.

This module holds random draws only: uniform residues modulo given primes,
ternary secrets, rounded-Gaussian errors and ChaCha seeds.  It performs none of
the key-switching arithmetic (no NTT, basis conversion, inner product or key
generation) and depends on neither the oracle nor the CUDA library.

Workloads (ring degree, basis shape, secret and key kind) are the five
key-switching workloads of this project, named by what they are.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

SIGMA = 3.2          # error standard deviation (CKKS standard)
ERR_BOUND = 19       # 6-sigma tail cut: |e| <= 19
HAMMING_WEIGHT = 192  # sparse ternary secret of the N=2^16 / 2^17 workloads


@dataclass(frozen=True)
class Workload:
    name: str
    logN: int
    L: int
    alpha: int
    bits: int            # primes are below 2^bits
    secret: str          # "ternary" (uniform) or "hw" (Hamming weight 192)
    key: str             # "square" (s^2 -> s) or "rot" (rotation keys)
    n_ct: int = 1        # ciphertexts per step
    levels: tuple = ()   # () = top level only
    op: str = "keyswitch"  # "keyswitch", "rotate", "hoisted" (n_rot rotations, one ModUp), "relin", "bsgs"
    n_rot: int = 1
    bsgs: tuple = ()     # (n1, n2): baby and giant steps of a linear transform

    @property
    def N(self) -> int:
        return 1 << self.logN

    @property
    def dnum(self) -> int:
        return -(-self.L // self.alpha)


WORKLOADS = {
    # relinearisation-style key switch s^2 -> s on a small ring
    "relin_n12": Workload("relin_n12", 12, 4, 2, 30, "ternary", "square"),
    # one rotation key switch at N=2^16, L=24, alpha=4, dnum=6
    "rot1_n16": Workload("rot1_n16", 16, 24, 4, 31, "hw", "rot"),
    # 16 ciphertexts under 16 rotation keys (2^k, k<16), same basis
    "batch16_n16": Workload("batch16_n16", 16, 24, 4, 31, "hw", "rot", n_ct=16),
    # standalone NTT throughput: 64 polynomials x 28 limbs of the N=2^16 chain
    "ntt_n16": Workload("ntt_n16", 16, 24, 4, 31, "hw", "rot", n_ct=64),
    # level sweep at N=2^17, L=40, alpha=5, dnum=8, levels 40..1
    "sweep_n17": Workload("sweep_n17", 17, 40, 5, 31, "hw", "rot",
                          levels=tuple(range(40, 0, -1))),
    # rotation by one slot (automorphism X -> X^5 fused into the key switch)
    "rotate_n16": Workload("rotate_n16", 16, 24, 4, 31, "hw", "rot", op="rotate"),
    # rotations by 1, 2, 4, ..., 128 slots of one ciphertext sharing one ModUp
    "hoisted8_n16": Workload("hoisted8_n16", 16, 24, 4, 31, "hw", "rot", op="hoisted", n_rot=8),
    # ciphertext product: tensor, then relinearisation with the s^2 -> s key
    "relin_mul_n12": Workload("relin_mul_n12", 12, 4, 2, 30, "ternary", "square", op="relin"),
    "relin_mul_n16": Workload("relin_mul_n16", 16, 24, 4, 31, "hw", "square", op="relin"),
    # baby-step giant-step linear transform (4 x 4 diagonals: 3 hoisted baby
    # rotations, 3 giant rotations) at every level of the N=2^17 sweep
    "bsgs_n17": Workload("bsgs_n17", 17, 40, 5, 31, "hw", "rot", levels=tuple(range(40, 0, -1)), op="bsgs",
                         bsgs=(4, 4)),
}


def rng(seed: int, *stream: int) -> np.random.Generator:
    """Independent PCG64 stream per (seed, stream ids)."""
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), *map(int, stream)])))


def uniform_residues(primes, N: int, seed: int, *stream: int) -> np.ndarray:
    """[len(primes)][N] uint32, row i uniform in [0, primes[i])."""
    g = rng(seed, *stream)
    out = np.empty((len(primes), N), dtype=np.uint32)
    for i, q in enumerate(primes):
        out[i] = g.integers(0, int(q), size=N, dtype=np.uint64).astype(np.uint32)
    return out


def uniform_residues_batch(primes, N: int, batch: int, seed: int, *stream: int) -> np.ndarray:
    """[batch][len(primes)][N] uint32."""
    return np.stack([uniform_residues(primes, N, seed, *stream, b) for b in range(batch)])


def ternary_secret(N: int, seed: int, hamming_weight: int | None = None) -> np.ndarray:
    """int64 coefficients in {-1,0,1}: uniform ternary, or exactly h nonzero
    positions (uniform subset) with uniform signs."""
    g = rng(seed, 0x5EC)
    if hamming_weight is None:
        return g.integers(-1, 2, size=N).astype(np.int64)
    s = np.zeros(N, dtype=np.int64)
    pos = g.choice(N, size=hamming_weight, replace=False)
    s[pos] = np.where(g.integers(0, 2, size=hamming_weight) == 1, 1, -1)
    return s


def gaussian_errors(count: int, N: int, seed: int, sigma: float = SIGMA,
                    bound: int = ERR_BOUND) -> np.ndarray:
    """[count][N] int64 rounded Gaussians, redrawn while |e| > bound."""
    g = rng(seed, 0xE77)
    out = np.rint(g.normal(0.0, sigma, size=(count, N))).astype(np.int64)
    bad = np.abs(out) > bound
    while bad.any():
        out[bad] = np.rint(g.normal(0.0, sigma, size=int(bad.sum()))).astype(np.int64)
        bad = np.abs(out) > bound
    return out


def chacha_seed(seed: int, key_id: int = 0) -> bytes:
    """32 random bytes: the ChaCha key of one key-switching key."""
    return rng(seed, 0x5EED, key_id).integers(0, 256, size=32, dtype=np.uint8).tobytes()
