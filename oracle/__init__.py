"""fp64 CPU oracle for Hybrid Tree Attention (LongSpec verification attention).

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import this package.  The CUDA
library never links, loads or calls it, and it imports nothing from the CUDA
package: the two paths share only the seeded input bytes.

The arithmetic lives in ``hta_oracle.c`` (plain C, single thread, fp64,
libm ``exp``/``log``, no fast-math); this module compiles it with gcc and
marshals numpy arrays through ctypes.  Every entry point is the plain
definition of masked softmax attention over the concatenated
``[prefix; tree]`` keys (LongSpec README, "Introduction", hybrid attention
aggregation; LongSpec paper summary, "Summary", Hybrid Tree Attention bullet),
or a step used to check the method against that definition (prefix-only
partials, tree-only partial, log-sum-exp merge).

Inputs are bf16 bit patterns (``numpy.uint16``); outputs are fp64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hta_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libhta_oracle.so")
_CFLAGS = ["-O2", "-std=c11", "-Wall", "-Wextra", "-ffp-contract=off",
           "-fno-fast-math", "-fPIC", "-shared"]

_lock = threading.Lock()
_lib = None

OK = 0
BAD_DIMS = -1
BAD_PARENT = -2
BAD_PREFIX_LEN = -3
BAD_ROW = -4
NO_MEMORY = -5
NO_VISIBLE_KEY = -6

# planted-mistake codes (see hta_oracle.c); only the pin-sensitivity tests use them
MUTATION_NONE = 0
MUTATION_DROP_SELF_BIT = 1
MUTATION_DROP_TREE = 2
MUTATION_HEAD_MAP = 3
MUTATION_NO_SCALE = 4
MUTATION_BAD_MERGE = 5
MUTATION_SHORT_PREFIX = 6


class OracleError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"oracle {what} failed with code {code}")
        self.code = code


def build(force: bool = False) -> str:
    """Compile hta_oracle.c into oracle/_build/libhta_oracle.so (gcc)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".{os.getpid()}.tmp"
        subprocess.run(["gcc", *_CFLAGS, _SRC, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _Problem(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
        ("D", ctypes.c_int), ("T", ctypes.c_int), ("L_cap", ctypes.c_int),
        ("scale", ctypes.c_double),
        ("q", ctypes.c_void_p), ("k_prefix", ctypes.c_void_p),
        ("v_prefix", ctypes.c_void_p), ("prefix_len", ctypes.c_void_p),
        ("k_tree", ctypes.c_void_p), ("v_tree", ctypes.c_void_p),
        ("parent", ctypes.c_void_p),
    ]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            vp, ci, cd = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
            pp = ctypes.POINTER(_Problem)
            lib.hta_oracle_tree_mask.argtypes = [ci, vp, vp, ci]
            lib.hta_oracle_attention.argtypes = [pp, ci, vp, vp, vp]
            lib.hta_oracle_prefix_partial.argtypes = [pp, ci, ci, ci, vp, vp, vp]
            lib.hta_oracle_tree_partial.argtypes = [pp, ci, vp, vp, vp]
            lib.hta_oracle_lse_merge.argtypes = [ci, ci, ci, vp, vp, vp, vp]
            lib.hta_oracle_set_mutation.argtypes = [ci]
            lib.hta_oracle_set_mutation.restype = None
            lib.hta_oracle_get_mutation.restype = ci
            lib.hta_oracle_bf16_value.argtypes = [ctypes.c_uint16]
            lib.hta_oracle_bf16_value.restype = cd
            _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError(f"expected bf16 bit patterns as uint16, got {a.dtype}")
    return a


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def set_mutation(code: int) -> None:
    """Plant a mistake in the oracle (pin-sensitivity tests only)."""
    _load().hta_oracle_set_mutation(int(code))


def get_mutation() -> int:
    return int(_load().hta_oracle_get_mutation())


def bf16_value(bits: int) -> float:
    return float(_load().hta_oracle_bf16_value(int(bits)))


def tree_mask(parent) -> np.ndarray:
    """Ancestor-or-self bitmask of one tree: uint32 [T][ceil(T/32)]."""
    par = _i32(parent).reshape(-1)
    T = par.shape[0]
    words = max(1, (T + 31) // 32)
    out = np.zeros((T, words), dtype=np.uint32)
    rc = _load().hta_oracle_tree_mask(T, _ptr(par), _ptr(out), words)
    if rc != OK:
        raise OracleError(rc, "tree_mask")
    return out


class Problem:
    """One verification-attention call: shapes plus bf16-bit inputs.

    Shapes: q [B][Hq][T][D], k/v_prefix [B][Hkv][L_cap][D],
    k/v_tree [B][Hkv][T][D], prefix_len [B], parent [B][T].
    """

    def __init__(self, q, k_prefix, v_prefix, prefix_len, k_tree, v_tree,
                 parent, scale: float = 0.0):
        self.q = _u16(q)
        self.k_prefix = _u16(k_prefix)
        self.v_prefix = _u16(v_prefix)
        self.k_tree = _u16(k_tree)
        self.v_tree = _u16(v_tree)
        self.prefix_len = _i32(prefix_len).reshape(-1)
        self.B, self.Hq, self.T, self.D = self.q.shape
        self.Hkv = self.k_tree.shape[1]
        self.L_cap = self.k_prefix.shape[2]
        self.parent = _i32(parent).reshape(self.B, self.T)
        self.scale = float(scale)
        if self.k_prefix.shape != (self.B, self.Hkv, self.L_cap, self.D):
            raise ValueError("k_prefix shape mismatch")
        if self.v_prefix.shape != self.k_prefix.shape:
            raise ValueError("v_prefix shape mismatch")
        if self.k_tree.shape != (self.B, self.Hkv, self.T, self.D):
            raise ValueError("k_tree shape mismatch")
        if self.v_tree.shape != self.k_tree.shape:
            raise ValueError("v_tree shape mismatch")
        if self.prefix_len.shape[0] != self.B:
            raise ValueError("prefix_len shape mismatch")
        self._c = _Problem(self.B, self.Hq, self.Hkv, self.D, self.T,
                           self.L_cap, self.scale, _ptr(self.q),
                           _ptr(self.k_prefix), _ptr(self.v_prefix),
                           _ptr(self.prefix_len), _ptr(self.k_tree),
                           _ptr(self.v_tree), _ptr(self.parent))

    @property
    def n_rows(self) -> int:
        return self.B * self.Hq * self.T

    def _rows(self, rows):
        if rows is None:
            return None, self.n_rows
        r = _i32(rows).reshape(-1, 3)
        return r, r.shape[0]

    def _run(self, fn, what, rows, *extra):
        r, n = self._rows(rows)
        out = np.zeros((n, self.D), dtype=np.float64)
        lse = np.zeros((n,), dtype=np.float64)
        rc = fn(ctypes.byref(self._c), *extra, n,
                None if r is None else _ptr(r), _ptr(out), _ptr(lse))
        if rc != OK:
            raise OracleError(rc, what)
        if rows is None:
            out = out.reshape(self.B, self.Hq, self.T, self.D)
            lse = lse.reshape(self.B, self.Hq, self.T)
        return out, lse

    def attention(self, rows=None):
        """One-pass masked attention over [prefix; tree]: (out, lse).

        rows: None for every (b, h, t) (shapes [B][Hq][T][D] and [B][Hq][T]),
        or an int array of (b, h, t) triples (shapes [n][D] and [n]).
        """
        return self._run(_load().hta_oracle_attention, "attention", rows)

    def prefix_partial(self, key_begin: int, key_end: int, rows=None):
        """Unmasked attention over prefix keys [key_begin, key_end) only."""
        return self._run(_load().hta_oracle_prefix_partial, "prefix_partial",
                         rows, int(key_begin), int(key_end))

    def tree_partial(self, rows=None):
        """Attention over tree keys under the ancestor-or-self mask only."""
        return self._run(_load().hta_oracle_tree_partial, "tree_partial", rows)


def lse_merge(o_parts, lse_parts):
    """Log-sum-exp merge of partials.

    o_parts: [P][n][D] fp64, lse_parts: [P][n] fp64 -> (out [n][D], lse [n]).
    """
    o = np.ascontiguousarray(o_parts, dtype=np.float64)
    l = np.ascontiguousarray(lse_parts, dtype=np.float64)
    P, n, D = o.shape
    if l.shape != (P, n):
        raise ValueError("lse_parts shape mismatch")
    out = np.zeros((n, D), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    rc = _load().hta_oracle_lse_merge(n, P, D, _ptr(o), _ptr(l), _ptr(out),
                                      _ptr(lse))
    if rc != OK:
        raise OracleError(rc, "lse_merge")
    return out, lse
