"""ctypes wrapper around oracle/oracle.c, the plain CPU reference.

TEST INFRASTRUCTURE ONLY: tests/, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this module; the library under
``key_switching_b200/`` never does.  It shares no code with the CUDA path.

Functions mirror the C entry points one to one; arrays are numpy uint32 in the
layouts documented in oracle.c ([limb][N], [digit][limb][N], [half][limb][N]).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

ROUNDS = 12  # ChaCha12 (the method); 20 is used only by the ChaCha20 pin


def build(force: bool = False) -> str:
    """Compile liboracle.so with gcc (plain -O2, single thread)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-shared", "-fPIC", "-o", _LIB, _SRC])
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        u32, i32, vp = ctypes.c_uint32, ctypes.c_int, ctypes.c_void_p
        L.or_is_prime.argtypes = [u32]
        L.or_is_prime.restype = i32
        L.or_gen_primes.argtypes = [u32, u32, u32, vp]
        L.or_gen_primes.restype = i32
        L.or_min_psi.argtypes = [u32, u32]
        L.or_min_psi.restype = u32
        L.or_ntt_fwd.argtypes = [vp, u32, u32, u32]
        L.or_ntt_inv.argtypes = [vp, u32, u32, u32]
        L.or_chacha_permute.argtypes = [vp, i32]
        L.or_chacha_block.argtypes = [vp, i32, vp]
        L.or_expand_a.argtypes = [vp, u32, u32, u32, u32, i32, vp]
        L.or_modup.argtypes = [vp, vp, u32, vp]
        L.or_modup.restype = i32
        L.or_inner.argtypes = [vp, vp, u32, vp, vp, vp, i32, vp]
        L.or_inner.restype = i32
        L.or_moddown.argtypes = [vp, vp, u32, vp]
        L.or_moddown.restype = i32
        L.or_keyswitch.argtypes = [vp, vp, vp, u32, vp, vp, vp, i32, vp, vp]
        L.or_keyswitch.restype = i32
        L.or_automorph_ntt.argtypes = [vp, u32, u32, vp]
        L.or_rotate.argtypes = [vp, vp, vp, u32, u32, vp, vp, vp, i32, vp, vp]
        L.or_rotate.restype = i32
        L.or_rotate_hoisted_one.argtypes = [vp, vp, vp, u32, u32, vp, vp, vp, i32, vp, vp]
        L.or_rotate_hoisted_one.restype = i32
        L.or_tensor.argtypes = [vp, vp, vp, vp, vp, u32, vp, vp, vp]
        L.or_tensor.restype = i32
        L.or_relinearize.argtypes = [vp, vp, vp, vp, vp, u32, vp, vp, vp, i32, vp, vp]
        L.or_relinearize.restype = i32
        L.or_linear_transform.argtypes = [vp, vp, vp, u32, u32, vp, vp, vp, u32, vp, vp, vp, vp, i32, vp, vp]
        L.or_linear_transform.restype = i32
        L.or_negacyclic_mul.argtypes = [vp, vp, u32, vp]
        L.or_automorph.argtypes = [vp, u32, u32, vp]
        L.or_ksk_gen.argtypes = [vp, vp, vp, vp, vp, i32, vp]
        L.or_ksk_gen.restype = i32
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


class _Params(ctypes.Structure):
    _fields_ = [("logN", ctypes.c_uint32), ("L", ctypes.c_uint32), ("alpha", ctypes.c_uint32),
                ("dnum", ctypes.c_uint32), ("q", ctypes.c_void_p), ("p", ctypes.c_void_p)]


class Params:
    """Ring degree 2^logN, L ciphertext primes q, alpha special primes p."""

    def __init__(self, logN: int, q, p):
        self.logN = int(logN)
        self.N = 1 << self.logN
        self.q = np.ascontiguousarray(np.asarray(q, dtype=np.uint32))
        self.p = np.ascontiguousarray(np.asarray(p, dtype=np.uint32))
        self.L = len(self.q)
        self.alpha = len(self.p)
        self.dnum = -(-self.L // self.alpha)
        self._c = _Params(self.logN, self.L, self.alpha, self.dnum,
                          self.q.ctypes.data, self.p.ctypes.data)

    @property
    def ptr(self):
        return ctypes.byref(self._c)

    def prime(self, g: int) -> int:
        return int(self.q[g]) if g < self.L else int(self.p[g - self.L])

    def glob(self, l: int, t: int) -> int:
        return t if t < l else self.L + (t - l)

    def level_primes(self, l: int):
        """Primes of the local limbs 0..l+alpha-1 at level l."""
        return [self.prime(self.glob(l, t)) for t in range(l + self.alpha)]


def is_prime(n: int) -> bool:
    return bool(lib().or_is_prime(n))


def gen_primes(logN: int, bits: int, count: int) -> np.ndarray:
    out = np.zeros(count, dtype=np.uint32)
    if lib().or_gen_primes(logN, bits, count, _p(out)) != 0:
        raise ValueError("not enough primes")
    return out


def chain(logN: int, bits: int, L: int, alpha: int) -> Params:
    """The first alpha primes found (largest) are the special primes, the next
    L the ciphertext primes."""
    pr = gen_primes(logN, bits, L + alpha)
    return Params(logN, pr[alpha:], pr[:alpha])


def min_psi(q: int, logN: int) -> int:
    return int(lib().or_min_psi(q, logN))


def ntt_fwd(a: np.ndarray, logN: int, q: int) -> np.ndarray:
    x = np.ascontiguousarray(a, dtype=np.uint32).copy()
    lib().or_ntt_fwd(_p(x), logN, q, min_psi(q, logN))
    return x


def ntt_inv(a: np.ndarray, logN: int, q: int) -> np.ndarray:
    x = np.ascontiguousarray(a, dtype=np.uint32).copy()
    lib().or_ntt_inv(_p(x), logN, q, min_psi(q, logN))
    return x


def chacha_permute(state, double_rounds: int) -> np.ndarray:
    x = np.ascontiguousarray(np.asarray(state, dtype=np.uint32)).copy()
    lib().or_chacha_permute(_p(x), double_rounds)
    return x


def chacha_block(state, rounds: int = ROUNDS) -> np.ndarray:
    x = np.ascontiguousarray(np.asarray(state, dtype=np.uint32))
    out = np.zeros(16, dtype=np.uint32)
    lib().or_chacha_block(_p(x), rounds, _p(out))
    return out


def _seed(seed: bytes):
    assert len(seed) == 32
    return np.frombuffer(bytes(seed), dtype=np.uint8).copy()


def expand_a(seed: bytes, j: int, g: int, q: int, logN: int, rounds: int = ROUNDS) -> np.ndarray:
    out = np.zeros(1 << logN, dtype=np.uint32)
    s = _seed(seed)
    lib().or_expand_a(_p(s), j, g, q, logN, rounds, _p(out))
    return out


def expand_a_level(P: Params, seed: bytes, l: int, rounds: int = ROUNDS) -> np.ndarray:
    """a_{j,t} for j < beta and local limbs t < l+alpha: [beta][l+alpha][N]."""
    beta = -(-l // P.alpha)
    ll = l + P.alpha
    out = np.zeros((beta, ll, P.N), dtype=np.uint32)
    for j in range(beta):
        for t in range(ll):
            g = P.glob(l, t)
            out[j, t] = expand_a(seed, j, g, P.prime(g), P.logN, rounds)
    return out


def modup(P: Params, c1: np.ndarray, l: int) -> np.ndarray:
    beta = -(-l // P.alpha)
    c1 = np.ascontiguousarray(c1, dtype=np.uint32)
    assert c1.shape == (l, P.N)
    ext = np.zeros((beta, l + P.alpha, P.N), dtype=np.uint32)
    if lib().or_modup(P.ptr, _p(c1), l, _p(ext)) != 0:
        raise ValueError("or_modup: bad arguments")
    return ext


def inner(P: Params, ext: np.ndarray, l: int, seed: bytes, b: np.ndarray, a=None,
          rounds: int = ROUNDS) -> np.ndarray:
    ext = np.ascontiguousarray(ext, dtype=np.uint32)
    b = np.ascontiguousarray(b, dtype=np.uint32)
    assert b.shape == (P.dnum, P.L + P.alpha, P.N)
    acc = np.zeros((2, l + P.alpha, P.N), dtype=np.uint32)
    s = _seed(seed)
    ap = None
    if a is not None:
        a = np.ascontiguousarray(a, dtype=np.uint32)
        assert a.shape == b.shape
        ap = _p(a)
    if lib().or_inner(P.ptr, _p(ext), l, _p(s), _p(b), ap, rounds, _p(acc)) != 0:
        raise ValueError("or_inner: bad arguments")
    return acc


def moddown(P: Params, acc: np.ndarray, l: int) -> np.ndarray:
    acc = np.ascontiguousarray(acc, dtype=np.uint32)
    assert acc.shape == (2, l + P.alpha, P.N)
    out = np.zeros((2, l, P.N), dtype=np.uint32)
    if lib().or_moddown(P.ptr, _p(acc), l, _p(out)) != 0:
        raise ValueError("or_moddown: bad arguments")
    return out


def keyswitch(P: Params, c0: np.ndarray, c1: np.ndarray, l: int, seed: bytes, b: np.ndarray,
              a=None, rounds: int = ROUNDS):
    c0 = np.ascontiguousarray(c0, dtype=np.uint32)
    c1 = np.ascontiguousarray(c1, dtype=np.uint32)
    b = np.ascontiguousarray(b, dtype=np.uint32)
    assert c0.shape == (l, P.N) and c1.shape == (l, P.N)
    c0o = np.zeros_like(c0)
    c1o = np.zeros_like(c1)
    s = _seed(seed)
    ap = None
    if a is not None:
        a = np.ascontiguousarray(a, dtype=np.uint32)
        ap = _p(a)
    if lib().or_keyswitch(P.ptr, _p(c0), _p(c1), l, _p(s), _p(b), ap, rounds, _p(c0o), _p(c1o)) != 0:
        raise ValueError("or_keyswitch: bad arguments")
    return c0o, c1o


def automorph_ntt(x: np.ndarray, logN: int, g: int) -> np.ndarray:
    """X -> X^g on one NTT-domain limb (a slot permutation)."""
    x = np.ascontiguousarray(x, dtype=np.uint32)
    assert x.shape == (1 << logN,)
    out = np.zeros_like(x)
    lib().or_automorph_ntt(_p(x), logN, g, _p(out))
    return out


def rotate(P: Params, c0: np.ndarray, c1: np.ndarray, l: int, g: int, seed: bytes, b: np.ndarray,
           a=None, rounds: int = ROUNDS):
    """Key switch of (c0(X^g), c1(X^g)) with a key for s(X^g) -> s."""
    c0 = np.ascontiguousarray(c0, dtype=np.uint32)
    c1 = np.ascontiguousarray(c1, dtype=np.uint32)
    b = np.ascontiguousarray(b, dtype=np.uint32)
    assert c0.shape == (l, P.N) and c1.shape == (l, P.N)
    c0o = np.zeros_like(c0)
    c1o = np.zeros_like(c1)
    ap = None
    if a is not None:
        a = np.ascontiguousarray(a, dtype=np.uint32)
        ap = _p(a)
    s = _seed(seed)
    if lib().or_rotate(P.ptr, _p(c0), _p(c1), l, g, _p(s), _p(b), ap, rounds, _p(c0o), _p(c1o)) != 0:
        raise ValueError("or_rotate: bad arguments")
    return c0o, c1o


def rotate_hoisted(P: Params, c0: np.ndarray, c1: np.ndarray, l: int, gs, seeds, bs,
                   rounds: int = ROUNDS):
    """Rotations of one ciphertext by each Galois element in gs, sharing one
    ModUp of c1; returns [(c0', c1')] in the order of gs."""
    c0 = np.ascontiguousarray(c0, dtype=np.uint32)
    ext = modup(P, c1, l)
    outs = []
    for g, seed, b in zip(gs, seeds, bs):
        b = np.ascontiguousarray(b, dtype=np.uint32)
        c0o = np.zeros((l, P.N), dtype=np.uint32)
        c1o = np.zeros((l, P.N), dtype=np.uint32)
        s = _seed(seed)
        if lib().or_rotate_hoisted_one(P.ptr, _p(c0), _p(ext), l, g, _p(s), _p(b), None, rounds,
                                       _p(c0o), _p(c1o)) != 0:
            raise ValueError("or_rotate_hoisted_one: bad arguments")
        outs.append((c0o, c1o))
    return outs


def tensor(P: Params, x0, x1, y0, y1, l: int):
    """(d0, d1, d2) of the product of ciphertexts (x0, x1) and (y0, y1)."""
    xs = [np.ascontiguousarray(v, dtype=np.uint32) for v in (x0, x1, y0, y1)]
    for v in xs:
        assert v.shape == (l, P.N)
    d = [np.zeros((l, P.N), dtype=np.uint32) for _ in range(3)]
    if lib().or_tensor(P.ptr, *[_p(v) for v in xs], l, *[_p(v) for v in d]) != 0:
        raise ValueError("or_tensor: bad arguments")
    return tuple(d)


def relinearize(P: Params, x0, x1, y0, y1, l: int, seed: bytes, b: np.ndarray, a=None,
                rounds: int = ROUNDS):
    """Tensor of two ciphertexts, then key switch of d2 with a key for s^2 -> s."""
    xs = [np.ascontiguousarray(v, dtype=np.uint32) for v in (x0, x1, y0, y1)]
    b = np.ascontiguousarray(b, dtype=np.uint32)
    c0o = np.zeros((l, P.N), dtype=np.uint32)
    c1o = np.zeros((l, P.N), dtype=np.uint32)
    ap = None
    if a is not None:
        a = np.ascontiguousarray(a, dtype=np.uint32)
        ap = _p(a)
    s = _seed(seed)
    if lib().or_relinearize(P.ptr, *[_p(v) for v in xs], l, _p(s), _p(b), ap, rounds,
                            _p(c0o), _p(c1o)) != 0:
        raise ValueError("or_relinearize: bad arguments")
    return c0o, c1o


def linear_transform(P: Params, c0: np.ndarray, c1: np.ndarray, l: int, diag: np.ndarray,
                     gb, seeds_b, bs_b, gg, seeds_g, bs_g, rounds: int = ROUNDS):
    """Baby-step giant-step linear transform with hoisted baby steps:
    out = sum_i rot_{gg_i}( sum_j diag[i][j] (.) rot_{gb_j}(ct) ), with the
    identity as baby step 0 and giant step 0.  diag: [n2][n1][l][N]; gb, seeds_b,
    bs_b: the n1-1 baby rotations (Galois elements, ChaCha seeds, key 'b'
    halves); gg, seeds_g, bs_g: the n2-1 giant rotations.  Returns (c0', c1')."""
    diag = np.ascontiguousarray(diag, dtype=np.uint32)
    n2, n1 = int(diag.shape[0]), int(diag.shape[1])
    assert diag.shape == (n2, n1, l, P.N)
    assert len(gb) == len(seeds_b) == len(bs_b) == n1 - 1 and len(gg) == len(seeds_g) == len(bs_g) == n2 - 1
    c0 = np.ascontiguousarray(c0, dtype=np.uint32)
    c1 = np.ascontiguousarray(c1, dtype=np.uint32)
    keep = []

    def keys(gs, seeds, bs):
        ga = np.ascontiguousarray(np.asarray(gs, dtype=np.uint32).reshape(-1))
        sa = np.frombuffer(b"".join(bytes(x) for x in seeds) or b"\0", dtype=np.uint8).copy()
        arrs = [np.ascontiguousarray(b, dtype=np.uint32) for b in bs]
        ptrs = (ctypes.c_void_p * max(1, len(arrs)))(*[a.ctypes.data for a in arrs])
        keep.extend([ga, sa, arrs, ptrs])
        return _p(ga), _p(sa), ptrs
    gbp, sbp, bbp = keys(gb, seeds_b, bs_b)
    ggp, sgp, bgp = keys(gg, seeds_g, bs_g)
    o0 = np.zeros((l, P.N), dtype=np.uint32)
    o1 = np.zeros((l, P.N), dtype=np.uint32)
    if lib().or_linear_transform(P.ptr, _p(c0), _p(c1), l, n1, gbp, sbp, bbp, n2, ggp, sgp, bgp, _p(diag),
                                 rounds, _p(o0), _p(o1)) != 0:
        raise ValueError("or_linear_transform: bad arguments")
    return o0, o1


def negacyclic_mul(a: np.ndarray, b: np.ndarray, logN: int) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.int64)
    b = np.ascontiguousarray(b, dtype=np.int64)
    out = np.zeros(1 << logN, dtype=np.int64)
    lib().or_negacyclic_mul(_p(a), _p(b), logN, _p(out))
    return out


def automorph(s: np.ndarray, logN: int, g: int) -> np.ndarray:
    s = np.ascontiguousarray(s, dtype=np.int64)
    out = np.zeros(1 << logN, dtype=np.int64)
    lib().or_automorph(_p(s), logN, g, _p(out))
    return out


def galois_elt(r: int, logN: int) -> int:
    """5^r mod 2N, the Galois element of a rotation by r slots."""
    return pow(5, r, 2 << logN)


def ksk_gen(P: Params, s: np.ndarray, sp: np.ndarray, e: np.ndarray, seed: bytes,
            rounds: int = ROUNDS) -> np.ndarray:
    s = np.ascontiguousarray(s, dtype=np.int64)
    sp = np.ascontiguousarray(sp, dtype=np.int64)
    e = np.ascontiguousarray(e, dtype=np.int64)
    assert e.shape == (P.dnum, P.N)
    b = np.zeros((P.dnum, P.L + P.alpha, P.N), dtype=np.uint32)
    sd = _seed(seed)
    if lib().or_ksk_gen(P.ptr, _p(s), _p(sp), _p(e), _p(sd), rounds, _p(b)) != 0:
        raise ValueError("or_ksk_gen: bad arguments")
    return b
