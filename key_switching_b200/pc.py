"""Thin ctypes binding of libpc (include/pc.h): argument marshalling only.

Every operation runs in the CUDA library; there is no CPU path.  Device
buffers are torch CUDA tensors of a 4-byte dtype (int32 or uint32 storage,
contiguous); they are passed as raw pointers.  If libpc.so is missing the
import fails with instructions to build it -- it never falls back.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
# PC_TIMELINE=1 loads the build whose kernels record the per-CTA timeline
TIMELINE = os.environ.get("PC_TIMELINE") == "1"
LIB_PATH = os.path.join(_HERE, "libpc_timeline.so" if TIMELINE else "libpc.so")

PC_OK = 0
ERRORS = {-1: "PC_E_ARG", -2: "PC_E_ALIGN", -3: "PC_E_CUDA", -4: "PC_E_DEVICE",
          -6: "PC_E_PRIME", -7: "PC_E_WORKSPACE", -8: "PC_E_TOO_BIG", -9: "PC_E_UNSUPPORTED"}
CHECK_INPUTS = 1           # pc_set_checks flag
ERR_INPUT, ERR_KEY = 1, 2  # bits of the device error word

# names of every exported entry point of include/pc.h
EXPORTS = ("pc_gen_primes", "pc_ctx_create", "pc_ctx_destroy", "pc_psi", "pc_workspace_bytes",
           "pc_set_workspace", "pc_ntt_fwd", "pc_ntt_inv", "pc_modup", "pc_keyswitch_inner",
           "pc_moddown", "pc_keyswitch", "pc_keyswitch_batch", "pc_expand_a", "pc_check",
           "pc_strerror", "pc_microbench", "pc_profile_begin", "pc_profile_end", "pc_modup_noalloc",
           "pc_rotate", "pc_rotate_hoisted", "pc_relinearize", "pc_keyswitch_host", "pc_host_workspace_bytes",
           "pc_keyswitch_capture", "pc_graph_launch", "pc_graph_destroy", "pc_capture_begin", "pc_capture_end",
           "pc_set_checks", "pc_last_error_word", "pc_linear_transform", "pc_linear_transform_workspace_bytes",
           "pc_timeline_read")
PROFILE_STAGES = ("intt_row_c1", "modup_col", "inner_chacha", "moddown_col", "moddown_finish")
# roles of the per-CTA timeline (PC_TL_* of pc.h, in order)
TL_ROLES = ("row_c1", "conv_up", "inner_special", "conv_down", "inner_ct", "moddown_finish", "row_other",
            "inner_other")
TL_CTAS = 4096


class PCError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {ERRORS.get(code, code)} ({strerror(code)})")


class _Params(ctypes.Structure):
    _fields_ = [("logN", ctypes.c_uint32), ("L", ctypes.c_uint32), ("alpha", ctypes.c_uint32),
                ("dnum", ctypes.c_uint32), ("q", ctypes.POINTER(ctypes.c_uint32)),
                ("p", ctypes.POINTER(ctypes.c_uint32))]


class _Ksk(ctypes.Structure):
    _fields_ = [("seed", ctypes.c_uint8 * 32), ("b", ctypes.c_void_p), ("a", ctypes.c_void_p)]


_lib = None


def lib():
    """Load libpc.so (built by key_switching_b200.build / __graft_entry__.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m key_switching_b200.build"
                              f"{' --timeline' if TIMELINE else ''}` (the library has no CPU fallback)")
        L = ctypes.CDLL(LIB_PATH)
        u32, i32, vp, sz = ctypes.c_uint32, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t
        L.pc_gen_primes.argtypes = [u32, u32, u32, ctypes.POINTER(u32)]
        L.pc_gen_primes.restype = i32
        L.pc_ctx_create.argtypes = [ctypes.POINTER(_Params), i32, ctypes.POINTER(vp)]
        L.pc_ctx_create.restype = i32
        L.pc_ctx_destroy.argtypes = [vp]
        L.pc_ctx_destroy.restype = None
        L.pc_psi.argtypes = [vp, u32]
        L.pc_psi.restype = u32
        L.pc_workspace_bytes.argtypes = [vp, u32, u32]
        L.pc_workspace_bytes.restype = sz
        L.pc_set_workspace.argtypes = [vp, vp, sz]
        L.pc_set_workspace.restype = i32
        for name in ("pc_ntt_fwd", "pc_ntt_inv"):
            getattr(L, name).argtypes = [vp, vp, u32, u32, u32, vp]
            getattr(L, name).restype = i32
        L.pc_modup.argtypes = [vp, vp, u32, vp, vp]
        L.pc_modup.restype = i32
        L.pc_keyswitch_inner.argtypes = [vp, vp, u32, ctypes.POINTER(_Ksk), vp, vp]
        L.pc_keyswitch_inner.restype = i32
        L.pc_moddown.argtypes = [vp, vp, u32, vp, vp]
        L.pc_moddown.restype = i32
        L.pc_keyswitch.argtypes = [vp, vp, vp, u32, ctypes.POINTER(_Ksk), vp, vp, vp]
        L.pc_keyswitch.restype = i32
        L.pc_keyswitch_batch.argtypes = [vp, vp, u32, u32, ctypes.POINTER(_Ksk), vp, vp]
        L.pc_keyswitch_batch.restype = i32
        L.pc_rotate.argtypes = [vp, vp, vp, u32, u32, ctypes.POINTER(_Ksk), vp, vp, vp]
        L.pc_rotate.restype = i32
        L.pc_rotate_hoisted.argtypes = [vp, vp, vp, u32, u32, ctypes.POINTER(u32), ctypes.POINTER(_Ksk), vp, vp]
        L.pc_rotate_hoisted.restype = i32
        L.pc_relinearize.argtypes = [vp, vp, vp, u32, ctypes.POINTER(_Ksk), vp, vp]
        L.pc_relinearize.restype = i32
        L.pc_keyswitch_host.argtypes = [vp, vp, u32, u32, ctypes.POINTER(_Ksk), vp, vp]
        L.pc_keyswitch_host.restype = i32
        L.pc_host_workspace_bytes.argtypes = [vp, u32]
        L.pc_host_workspace_bytes.restype = sz
        L.pc_keyswitch_capture.argtypes = [vp, vp, vp, u32, ctypes.POINTER(_Ksk), vp, vp, ctypes.POINTER(vp)]
        L.pc_keyswitch_capture.restype = i32
        L.pc_graph_launch.argtypes = [vp, vp]
        L.pc_graph_launch.restype = i32
        L.pc_graph_destroy.argtypes = [vp]
        L.pc_graph_destroy.restype = None
        L.pc_capture_begin.argtypes = [vp, ctypes.POINTER(vp)]
        L.pc_capture_begin.restype = i32
        L.pc_capture_end.argtypes = [vp, ctypes.POINTER(vp)]
        L.pc_capture_end.restype = i32
        L.pc_linear_transform.argtypes = [vp, vp, vp, u32, u32, ctypes.POINTER(u32), ctypes.POINTER(_Ksk), u32,
                                          ctypes.POINTER(u32), ctypes.POINTER(_Ksk), vp, vp, vp]
        L.pc_linear_transform.restype = i32
        L.pc_linear_transform_workspace_bytes.argtypes = [vp, u32, u32]
        L.pc_linear_transform_workspace_bytes.restype = sz
        L.pc_expand_a.argtypes = [vp, ctypes.c_char_p, u32, vp, vp]
        L.pc_expand_a.restype = i32
        L.pc_check.argtypes = [vp]
        L.pc_check.restype = i32
        L.pc_set_checks.argtypes = [vp, u32]
        L.pc_set_checks.restype = i32
        L.pc_last_error_word.argtypes = [vp]
        L.pc_last_error_word.restype = u32
        L.pc_strerror.argtypes = [i32]
        L.pc_strerror.restype = ctypes.c_char_p
        L.pc_microbench.argtypes = [i32, i32, u32, ctypes.POINTER(ctypes.c_double)]
        L.pc_microbench.restype = i32
        L.pc_profile_begin.argtypes = [vp, u32, u32]
        L.pc_profile_begin.restype = i32
        L.pc_profile_end.argtypes = [vp, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(u32)]
        L.pc_profile_end.restype = i32
        L.pc_timeline_read.argtypes = [vp, vp, sz]
        L.pc_timeline_read.restype = i32
        L.pc_modup_noalloc.argtypes = [vp, vp, u32, vp, vp]
        L.pc_modup_noalloc.restype = i32
        _lib = L
    return _lib


def strerror(code: int) -> str:
    return lib().pc_strerror(code).decode()


def _ok(rc: int, what: str):
    if rc != PC_OK:
        raise PCError(rc, what)


def _ptr(t) -> int:
    """Raw device pointer of a contiguous 4-byte-element torch tensor (or None)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    assert t.is_cuda and t.is_contiguous() and t.element_size() == 4, "need a contiguous 32-bit CUDA tensor"
    return t.data_ptr()


def _hptr(a) -> int:
    """Host address of a contiguous 4-byte-element CPU torch tensor or numpy array."""
    if hasattr(a, "is_cuda"):
        assert not a.is_cuda and a.is_contiguous() and a.element_size() == 4, "need a contiguous 32-bit CPU tensor"
        return a.data_ptr()
    assert a.flags["C_CONTIGUOUS"] and a.itemsize == 4, "need a contiguous 32-bit array"
    return a.ctypes.data


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def gen_primes(logN: int, bits: int, count: int):
    out = (ctypes.c_uint32 * count)()
    _ok(lib().pc_gen_primes(logN, bits, count, out), "pc_gen_primes")
    return [int(v) for v in out]


def chain(logN: int, bits: int, L: int, alpha: int):
    """(q, p): the first alpha primes are the special primes, the next L the q's."""
    pr = gen_primes(logN, bits, L + alpha)
    return pr[alpha:], pr[:alpha]


def microbench(kind: int, iters: int = 4096, device: int = 0) -> float:
    out = ctypes.c_double()
    _ok(lib().pc_microbench(device, kind, iters, ctypes.byref(out)), "pc_microbench")
    return out.value


class Graph:
    """An executable CUDA graph of one key switch (pc_keyswitch_capture); keeps
    the captured buffers alive."""

    def __init__(self, handle, keep):
        self._h = handle
        self._keep = keep

    def launch(self, stream=None):
        _ok(lib().pc_graph_launch(self._h, _stream(stream)), "pc_graph_launch")

    def close(self):
        if self._h:
            lib().pc_graph_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class KSK:
    """A key-switching key: 32-byte ChaCha12 seed, device 'b' half, optional
    stored 'a' half (None = regenerate in-kernel)."""

    def __init__(self, seed: bytes, b, a=None):
        assert len(seed) == 32
        self.seed, self.b, self.a = bytes(seed), b, a

    def _c(self) -> _Ksk:
        k = _Ksk()
        k.seed[:] = list(self.seed)
        k.b = _ptr(self.b)
        k.a = _ptr(self.a) if self.a is not None else None
        return k


class Context:
    """A libpc context on one device: the RNS basis and its device tables."""

    def __init__(self, logN: int, q: Sequence[int], p: Sequence[int], device: int = 0):
        self.logN, self.N = int(logN), 1 << int(logN)
        self.q, self.p = [int(v) for v in q], [int(v) for v in p]
        self.L, self.alpha = len(self.q), len(self.p)
        self.dnum = -(-self.L // self.alpha)
        self.device = device
        qa = (ctypes.c_uint32 * self.L)(*self.q)
        pa = (ctypes.c_uint32 * self.alpha)(*self.p)
        prm = _Params(self.logN, self.L, self.alpha, self.dnum, qa, pa)
        h = ctypes.c_void_p()
        _ok(lib().pc_ctx_create(ctypes.byref(prm), device, ctypes.byref(h)), "pc_ctx_create")
        self._h = h
        self._ws = None

    def close(self):
        if getattr(self, "_h", None):
            lib().pc_ctx_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def prime(self, g: int) -> int:
        return self.q[g] if g < self.L else self.p[g - self.L]

    def psi(self, g: int) -> int:
        return int(lib().pc_psi(self._h, g))

    def workspace_bytes(self, l: int, B: int = 1) -> int:
        return int(lib().pc_workspace_bytes(self._h, l, B))

    def set_workspace(self, buf) -> None:
        """Hand a device buffer (e.g. a torch uint8/int32 CUDA tensor) to the
        context; keeps a reference so it outlives the calls that use it."""
        if buf is None:
            _ok(lib().pc_set_workspace(self._h, None, 0), "pc_set_workspace")
        else:
            _ok(lib().pc_set_workspace(self._h, buf.data_ptr(), buf.numel() * buf.element_size()),
                "pc_set_workspace")
        self._ws = buf

    def ensure_workspace(self, l: int, B: int = 1):
        """Allocate (with torch) and set a workspace big enough for level l, B cts."""
        import torch
        need = self.workspace_bytes(l, B)
        if self._ws is None or self._ws.numel() * self._ws.element_size() < need:
            self.set_workspace(torch.empty(need, dtype=torch.uint8, device=f"cuda:{self.device}"))
        return self._ws

    def ntt_fwd(self, x, first_prime: int, nlimbs: int, batch: int = 1, stream=None):
        _ok(lib().pc_ntt_fwd(self._h, _ptr(x), first_prime, nlimbs, batch, _stream(stream)), "pc_ntt_fwd")

    def ntt_inv(self, x, first_prime: int, nlimbs: int, batch: int = 1, stream=None):
        _ok(lib().pc_ntt_inv(self._h, _ptr(x), first_prime, nlimbs, batch, _stream(stream)), "pc_ntt_inv")

    def modup(self, c1, l: int, ext, stream=None):
        _ok(lib().pc_modup(self._h, _ptr(c1), l, _ptr(ext), _stream(stream)), "pc_modup")

    def modup_noalloc(self, c1, l: int, ext, stream=None):
        """pc_modup with its scratch in the library's static device array
        (no workspace; for callers that cannot allocate device memory)."""
        _ok(lib().pc_modup_noalloc(self._h, _ptr(c1), l, _ptr(ext), _stream(stream)), "pc_modup_noalloc")

    def keyswitch_inner(self, ext, l: int, key: KSK, acc, stream=None):
        k = key._c()
        _ok(lib().pc_keyswitch_inner(self._h, _ptr(ext), l, ctypes.byref(k), _ptr(acc), _stream(stream)),
            "pc_keyswitch_inner")

    def moddown(self, acc, l: int, out, stream=None):
        _ok(lib().pc_moddown(self._h, _ptr(acc), l, _ptr(out), _stream(stream)), "pc_moddown")

    def keyswitch(self, c0, c1, l: int, key: KSK, c0o, c1o, stream=None):
        k = key._c()
        _ok(lib().pc_keyswitch(self._h, _ptr(c0), _ptr(c1), l, ctypes.byref(k), _ptr(c0o), _ptr(c1o),
                               _stream(stream)), "pc_keyswitch")

    def keyswitch_batch(self, ct, B: int, l: int, keys: Sequence[KSK], out, stream=None):
        arr = (_Ksk * B)(*[k._c() for k in keys])
        _ok(lib().pc_keyswitch_batch(self._h, _ptr(ct), B, l, arr, _ptr(out), _stream(stream)),
            "pc_keyswitch_batch")

    def rotate(self, c0, c1, l: int, galois: int, key: KSK, c0o, c1o, stream=None):
        k = key._c()
        _ok(lib().pc_rotate(self._h, _ptr(c0), _ptr(c1), l, galois, ctypes.byref(k), _ptr(c0o), _ptr(c1o),
                            _stream(stream)), "pc_rotate")

    def rotate_hoisted(self, c0, c1, l: int, galois: Sequence[int], keys: Sequence[KSK], out, stream=None):
        n = len(galois)
        assert len(keys) == n
        gs = (ctypes.c_uint32 * n)(*galois)
        arr = (_Ksk * n)(*[k._c() for k in keys])
        _ok(lib().pc_rotate_hoisted(self._h, _ptr(c0), _ptr(c1), l, n, gs, arr, _ptr(out), _stream(stream)),
            "pc_rotate_hoisted")

    def host_workspace_bytes(self, l: int) -> int:
        return lib().pc_host_workspace_bytes(self._h, l)

    def ensure_host_workspace(self, l: int):
        """Allocate (with torch) and set a workspace big enough for keyswitch_host at level l."""
        import torch
        need = self.host_workspace_bytes(l)
        if self._ws is None or self._ws.numel() * self._ws.element_size() < need:
            self.set_workspace(torch.empty(need, dtype=torch.uint8, device=f"cuda:{self.device}"))
        return self._ws

    def keyswitch_host(self, ct, n: int, l: int, keys: Sequence[KSK], out, stream=None):
        """n key switches of host ciphertexts ct [n][2][l][N] into host out [n][2][l][N]."""
        assert len(keys) == n
        arr = (_Ksk * n)(*[k._c() for k in keys])
        _ok(lib().pc_keyswitch_host(self._h, _hptr(ct), n, l, arr, _hptr(out), _stream(stream)),
            "pc_keyswitch_host")

    def keyswitch_capture(self, c0, c1, l: int, key: KSK, c0o, c1o) -> "Graph":
        """A CUDA graph of pc_keyswitch on these buffers (replay with Graph.launch)."""
        k = key._c()
        h = ctypes.c_void_p()
        _ok(lib().pc_keyswitch_capture(self._h, _ptr(c0), _ptr(c1), l, ctypes.byref(k), _ptr(c0o), _ptr(c1o),
                                       ctypes.byref(h)), "pc_keyswitch_capture")
        return Graph(h, (c0, c1, key, c0o, c1o))

    def capture(self, fn, keep=()) -> "Graph":
        """Record the library calls fn(stream) makes on a capturing stream into a Graph."""
        cs = ctypes.c_void_p()
        _ok(lib().pc_capture_begin(self._h, ctypes.byref(cs)), "pc_capture_begin")
        try:
            fn(cs.value)
        except BaseException:
            lib().pc_capture_end(self._h, None)
            raise
        h = ctypes.c_void_p()
        _ok(lib().pc_capture_end(self._h, ctypes.byref(h)), "pc_capture_end")
        return Graph(h, keep)

    def relinearize(self, x, y, l: int, key: KSK, out, stream=None):
        k = key._c()
        _ok(lib().pc_relinearize(self._h, _ptr(x), _ptr(y), l, ctypes.byref(k), _ptr(out), _stream(stream)),
            "pc_relinearize")

    def linear_transform_workspace_bytes(self, l: int, n1: int) -> int:
        return int(lib().pc_linear_transform_workspace_bytes(self._h, l, n1))

    def ensure_linear_transform_workspace(self, l: int, n1: int):
        """Allocate (with torch) and set a workspace big enough for a linear transform with n1 baby steps."""
        import torch
        need = self.linear_transform_workspace_bytes(l, n1)
        if self._ws is None or self._ws.numel() * self._ws.element_size() < need:
            self.set_workspace(torch.empty(need, dtype=torch.uint8, device=f"cuda:{self.device}"))
        return self._ws

    def linear_transform(self, c0, c1, l: int, diag, g_baby: Sequence[int], k_baby: Sequence[KSK],
                         g_giant: Sequence[int], k_giant: Sequence[KSK], out, stream=None):
        """pc_linear_transform: diag [n2][n1][l][N] on the device; g_baby/k_baby the n1-1 baby
        rotations, g_giant/k_giant the n2-1 giant rotations; out [2][l][N]."""
        n2, n1 = int(diag.shape[0]), int(diag.shape[1])
        assert len(g_baby) == len(k_baby) == n1 - 1 and len(g_giant) == len(k_giant) == n2 - 1
        gb = (ctypes.c_uint32 * max(1, n1 - 1))(*g_baby)
        kb = (_Ksk * max(1, n1 - 1))(*[k._c() for k in k_baby])
        gg = (ctypes.c_uint32 * max(1, n2 - 1))(*g_giant)
        kg = (_Ksk * max(1, n2 - 1))(*[k._c() for k in k_giant])
        _ok(lib().pc_linear_transform(self._h, _ptr(c0), _ptr(c1), l, n1, gb, kb, n2, gg, kg, _ptr(diag), _ptr(out),
                                      _stream(stream)), "pc_linear_transform")

    def expand_a(self, seed: bytes, l: int, out, stream=None):
        _ok(lib().pc_expand_a(self._h, bytes(seed), l, _ptr(out), _stream(stream)), "pc_expand_a")

    def check(self):
        _ok(lib().pc_check(self._h), "pc_check")

    def set_checks(self, flags: int):
        """pc_set_checks: 0, or CHECK_INPUTS to validate every input residue on the device."""
        _ok(lib().pc_set_checks(self._h, flags), "pc_set_checks")

    def last_error_word(self) -> int:
        return int(lib().pc_last_error_word(self._h))

    def profile_begin(self, max_calls: int, every: int = 1):
        _ok(lib().pc_profile_begin(self._h, max_calls, every), "pc_profile_begin")

    def profile_end(self):
        """-> (dict stage -> summed ms, number of recorded calls)"""
        ms = (ctypes.c_float * len(PROFILE_STAGES))()
        n = ctypes.c_uint32()
        _ok(lib().pc_profile_end(self._h, ms, ctypes.byref(n)), "pc_profile_end")
        return dict(zip(PROFILE_STAGES, [float(v) for v in ms])), int(n.value)

    def timeline_read(self):
        """Per-CTA timeline (library built with --timeline, PC_TIMELINE=1):
        uint64 array [len(TL_ROLES)][TL_CTAS][3] of (start ns, end ns, SM) of
        each role's latest launch (zeros where no CTA ran); the device copy is
        zeroed."""
        import numpy as np
        out = np.zeros((len(TL_ROLES), TL_CTAS, 3), dtype=np.uint64)
        _ok(lib().pc_timeline_read(self._h, out.ctypes.data, out.size), "pc_timeline_read")
        return out
