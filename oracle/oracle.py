"""ctypes front end of the fp64 CPU oracle (``oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the bench's CPU-baseline leg use it; the
product path never does.  Inputs are the raw bf16 bit patterns (numpy uint16) that the CUDA path
receives; outputs are float64 numpy arrays.

Every function here applies the plain attention definition (see the header of ``oracle.c`` for the
passages it follows); the pins that tie it to what the pages and the mathematics fix live in
``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

_u16p = np.ctypeslib.ndpointer(dtype=np.uint16, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_i64p = np.ctypeslib.ndpointer(dtype=np.int64, flags="C_CONTIGUOUS")
_u64p = np.ctypeslib.ndpointer(dtype=np.uint64, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_i64 = ctypes.c_int64
_int = ctypes.c_int
_dbl = ctypes.c_double


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` with gcc into ``liboracle.so`` beside it (plain -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-fno-fast-math",
                               "-o", _LIB, _SRC, "-lm", "-lpthread"])
    return _LIB


class OracleLib:
    """The oracle's entry points bound to one compiled library (the default one, or a test build)."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        lib.oracle_attention.argtypes = [_u16p, _u16p, _u16p, _i64, _i64, _int, _int, _dbl,
                                         _f64p, _f64p, _int]
        lib.oracle_attention_rows.argtypes = [_u16p, _u16p, _u16p, _i64, _int, _int, _dbl, _i64p,
                                              _i64, _f64p, _f64p, _int]
        lib.oracle_attention_probs.argtypes = [_u16p, _u16p, _i64, _int, _int, _dbl, _f64p]
        lib.oracle_flash_alg1.argtypes = [_u16p, _u16p, _u16p, _i64, _int, _int, _dbl, _int, _int,
                                          _f64p, _f64p, _f64p]
        lib.oracle_decode_paged.argtypes = [_u16p, _u16p, _u16p, _i32p, _int, _i32p, _int, _int,
                                            _int, _int, _dbl, _f64p, _f64p, _int]
        lib.oracle_prefill_paged.argtypes = [_u16p, _u16p, _u16p, _i32p, _int, _i32p, _int, _int,
                                             _int, _int, _int, _int, _dbl, _f64p, _f64p, _int]
        lib.oracle_tree_attention.argtypes = [_u16p, _u16p, _u16p, _i32p, _int, _i32p, _u64p,
                                              _int, _int, _int, _int, _int, _dbl, _f64p, _f64p,
                                              _int]
        lib.oracle_tree_attention.restype = ctypes.c_int
        lib.oracle_attention_keyrange.argtypes = [_u16p, _u16p, _u16p, _i64, _i64, _i64, _i64,
                                                  _i64, _int, _int, _dbl, _f64p, _f64p, _int]
        lib.oracle_attention_keyrange.restype = ctypes.c_int
        lib.oracle_merge_partials.argtypes = [_f64p, _f64p, _int, _i64, _int, _f64p, _f64p]
        lib.oracle_merge_partials.restype = ctypes.c_int
        lib.oracle_attention_bwd.argtypes = [_u16p, _u16p, _u16p, _u16p, _i64, _int, _int, _dbl,
                                             _i64p, _i64, _f64p, _f64p, _f64p, _int]
        for f in (lib.oracle_attention, lib.oracle_attention_rows, lib.oracle_attention_probs,
                  lib.oracle_flash_alg1, lib.oracle_decode_paged, lib.oracle_prefill_paged,
                  lib.oracle_attention_bwd):
            f.restype = ctypes.c_int
        self.lib = lib
        self.path = path

    def attention(self, q, k, v, causal: bool, scale: float, nthreads: int | None = None):
        """All rows. q, k, v: uint16 [..., N, d] (bf16 bits). Returns (o [..., N, d], lse [..., N])."""
        q, k, v = _bits(q), _bits(k), _bits(v)
        *lead, N, d = q.shape
        BH = int(np.prod(lead)) if lead else 1
        o = np.empty((BH, N, d), np.float64)
        lse = np.empty((BH, N), np.float64)
        rc = self.lib.oracle_attention(q, k, v, BH, N, d, int(causal), scale, o, lse,
                                       nthreads or default_threads())
        if rc:
            raise ValueError("oracle_attention: bad arguments")
        return o.reshape(*lead, N, d), lse.reshape(*lead, N)

    def attention_rows(self, q, k, v, causal: bool, scale: float, pairs, nthreads: int | None = None):
        """Selected rows. q, k, v: uint16 [..., N, d] (leading dims flattened to bh); pairs: int64
        [n, 2] of (bh, row).  Returns (o [n, d], lse [n])."""
        q, k, v = _bits(q), _bits(k), _bits(v)
        N, d = q.shape[-2], q.shape[-1]
        pairs = np.ascontiguousarray(pairs, dtype=np.int64).reshape(-1, 2)
        n = pairs.shape[0]
        o = np.empty((n, d), np.float64)
        lse = np.empty((n,), np.float64)
        rc = self.lib.oracle_attention_rows(q, k, v, N, d, int(causal), scale, pairs, n, o, lse,
                                            nthreads or default_threads())
        if rc:
            raise ValueError("oracle_attention_rows: bad arguments")
        return o, lse

    def probs(self, q, k, causal: bool, scale: float):
        """Full probability matrix P [N, N] of one head (masked entries 0)."""
        q, k = _bits(q), _bits(k)
        N, d = q.shape
        P = np.empty((N, N), np.float64)
        self.lib.oracle_attention_probs(q, k, N, d, int(causal), scale, P)
        return P

    def flash_alg1(self, q, k, v, causal: bool, scale: float, Br: int, Bc: int):
        """The tiled algorithm with block sizes Br x Bc on one head. Returns (O, l, m)."""
        q, k, v = _bits(q), _bits(k), _bits(v)
        N, d = q.shape
        O = np.empty((N, d), np.float64)
        l = np.empty((N,), np.float64)
        m = np.empty((N,), np.float64)
        rc = self.lib.oracle_flash_alg1(q, k, v, N, d, int(causal), scale, Br, Bc, O, l, m)
        if rc:
            raise ValueError("oracle_flash_alg1: bad arguments")
        return O, l, m

    def attention_keyrange(self, q, k, v, q0: int, k0: int, causal: bool, scale: float,
                           nthreads: int | None = None):
        """Partial attention of queries at positions q0.. over keys at positions k0.. of the same
        sequences.  q [..., Nq, d], k, v [..., Nk, d] (uint16 bf16 bits).  Rows that see no key
        get O = 0, LSE = -inf.  Returns (o [..., Nq, d], lse [..., Nq])."""
        q, k, v = _bits(q), _bits(k), _bits(v)
        *lead, Nq, d = q.shape
        Nk = k.shape[-2]
        BH = int(np.prod(lead)) if lead else 1
        o = np.empty((BH, Nq, d), np.float64)
        lse = np.empty((BH, Nq), np.float64)
        rc = self.lib.oracle_attention_keyrange(q, k, v, BH, Nq, Nk, q0, k0, d, int(causal), scale,
                                                o, lse, nthreads or default_threads())
        if rc:
            raise ValueError("oracle_attention_keyrange: bad arguments")
        return o.reshape(*lead, Nq, d), lse.reshape(*lead, Nq)

    def merge_partials(self, o_parts, lse_parts):
        """o_parts [G, ..., d], lse_parts [G, ...] (float64).  Returns the merged (o, lse)."""
        o_parts = np.ascontiguousarray(o_parts, dtype=np.float64)
        lse_parts = np.ascontiguousarray(lse_parts, dtype=np.float64)
        G, d = o_parts.shape[0], o_parts.shape[-1]
        rows = int(np.prod(o_parts.shape[1:-1]))
        o = np.empty(o_parts.shape[1:], np.float64)
        lse = np.empty(lse_parts.shape[1:], np.float64)
        rc = self.lib.oracle_merge_partials(o_parts, lse_parts, G, rows, d, o, lse)
        if rc:
            raise ValueError("oracle_merge_partials: bad arguments")
        return o, lse

    def tree_attention(self, q, k_pool, v_pool, block_table, seq_lens, tree_mask, scale: float,
                       page: int = 16, nthreads: int | None = None):
        """Tree verification.  q [S,H,T,d] are the tree's nodes, the last T of each sequence's
        cached tokens; tree_mask [S,T] (uint64 bit patterns, any integer dtype): bit u of entry t
        set when node t sees node u.  Returns (o [S,H,T,d], lse [S,H,T])."""
        q, k_pool, v_pool = _bits(q), _bits(k_pool), _bits(v_pool)
        table = np.ascontiguousarray(block_table, dtype=np.int32)
        lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
        mask = np.ascontiguousarray(np.asarray(tree_mask).astype(np.int64).view(np.uint64))
        S, H, T, d = q.shape
        o = np.empty((S, H, T, d), np.float64)
        lse = np.empty((S, H, T), np.float64)
        rc = self.lib.oracle_tree_attention(q, k_pool, v_pool, table, table.shape[1], lens, mask,
                                            S, H, T, d, page, scale, o, lse,
                                            nthreads or default_threads())
        if rc:
            raise ValueError("oracle_tree_attention: bad arguments")
        return o, lse

    def attention_bwd(self, q, k, v, dout, causal: bool, scale: float, heads=None,
                      nthreads: int | None = None):
        """Backward pass.  q, k, v, dout: uint16 [..., N, d] (bf16 bits; leading dims flattened to
        bh).  heads: the bh indices to differentiate (default all).  Returns (dq, dk, dv), each
        float64 [len(heads), N, d] (or [..., N, d] when all heads are taken)."""
        q, k, v, dout = _bits(q), _bits(k), _bits(v), _bits(dout)
        *lead, N, d = q.shape
        BH = int(np.prod(lead)) if lead else 1
        all_heads = heads is None
        heads = np.arange(BH, dtype=np.int64) if all_heads else np.ascontiguousarray(heads, dtype=np.int64)
        if heads.size and (heads.min() < 0 or heads.max() >= BH):
            raise ValueError("head index out of range")
        n = heads.size
        dq, dk, dv = (np.empty((n, N, d), np.float64) for _ in range(3))
        rc = self.lib.oracle_attention_bwd(q, k, v, dout, N, d, int(causal), scale, heads, n, dq, dk,
                                           dv, nthreads or default_threads())
        if rc:
            raise ValueError("oracle_attention_bwd: bad arguments")
        if all_heads:
            return tuple(t.reshape(*lead, N, d) for t in (dq, dk, dv))
        return dq, dk, dv

    def decode_paged(self, q, k_pool, v_pool, block_table, seq_lens, scale: float, page: int = 16,
                     nthreads: int | None = None):
        """q [S,H,d]; pools [P,H,page,d] (uint16 bf16 bits); block_table int32 [S,max_blocks];
        seq_lens int32 [S].  Returns (o [S,H,d], lse [S,H])."""
        q, k_pool, v_pool = _bits(q), _bits(k_pool), _bits(v_pool)
        table = np.ascontiguousarray(block_table, dtype=np.int32)
        lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
        S, H, d = q.shape
        o = np.empty((S, H, d), np.float64)
        lse = np.empty((S, H), np.float64)
        rc = self.lib.oracle_decode_paged(q, k_pool, v_pool, table, table.shape[1], lens, S, H, d,
                                          page, scale, o, lse, nthreads or default_threads())
        if rc:
            raise ValueError("oracle_decode_paged: bad arguments")
        return o, lse


    def prefill_paged(self, q, k_pool, v_pool, block_table, seq_lens, causal: bool, scale: float,
                      page: int = 16, nthreads: int | None = None):
        """Chunked prefill over a paged cache.  q [S,H,Lq,d] are the last Lq positions of each
        sequence's context; pools [P,H,page,d]; block_table int32 [S,max_blocks]; seq_lens int32
        [S] (each >= Lq).  Returns (o [S,H,Lq,d], lse [S,H,Lq])."""
        q, k_pool, v_pool = _bits(q), _bits(k_pool), _bits(v_pool)
        table = np.ascontiguousarray(block_table, dtype=np.int32)
        lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
        S, H, Lq, d = q.shape
        o = np.empty((S, H, Lq, d), np.float64)
        lse = np.empty((S, H, Lq), np.float64)
        rc = self.lib.oracle_prefill_paged(q, k_pool, v_pool, table, table.shape[1], lens, S, H,
                                           Lq, d, page, int(causal), scale, o, lse,
                                           nthreads or default_threads())
        if rc:
            raise ValueError("oracle_prefill_paged: bad arguments")
        return o, lse


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def _bits(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("oracle inputs are bf16 bit patterns (uint16)")
    return a


def default() -> OracleLib:
    """The oracle built from ``oracle.c`` as committed."""
    global _lib
    if _lib is None:
        _lib = OracleLib(build())
    return _lib


def attention(*a, **kw):
    return default().attention(*a, **kw)


def attention_rows(*a, **kw):
    return default().attention_rows(*a, **kw)


def probs(*a, **kw):
    return default().probs(*a, **kw)


def flash_alg1(*a, **kw):
    return default().flash_alg1(*a, **kw)


def decode_paged(*a, **kw):
    return default().decode_paged(*a, **kw)


def prefill_paged(*a, **kw):
    return default().prefill_paged(*a, **kw)


def attention_bwd(*a, **kw):
    return default().attention_bwd(*a, **kw)


def tree_attention(*a, **kw):
    return default().tree_attention(*a, **kw)


def attention_keyrange(*a, **kw):
    return default().attention_keyrange(*a, **kw)


def merge_partials(*a, **kw):
    return default().merge_partials(*a, **kw)
