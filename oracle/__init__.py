"""CPU oracle for the paged-KV attention step (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference leg may import this package.  The product path (the CUDA library
and its binding) never imports it and shares no code with it.

The arithmetic lives in ``pa_oracle.c`` (plain C, fp64, OpenMP over output
rows); this module only compiles it with gcc, loads it with ctypes and
marshals numpy arrays.  bf16 tensors are passed as their uint16 bit patterns.

What it computes, and the passages it follows, are stated in the header of
``pa_oracle.c``: the block-table / slot-mapping semantics of "vLLM 学习笔记 01"
§1.5-§1.6, the computed-vs-total token view of §1.4 and §2.1 (seq_len counts
the tokens scheduled this step; queries are bottom-right causal), and the
block layout of the "Inside vLLM" engine-constructor section.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_ERRORS = {
    1: "bad sizes or null pointers",
    2: "slot outside the pool",
    3: "segment bounds invalid (cu_seqlens not monotone or q_len > seq_len)",
    4: "a block id the segment needs is outside the pool",
    5: "a requested output row does not exist",
    6: "out of host memory",
}


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile pa_oracle.c into liboracle.so next to it (gcc, -O2, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-Wall", "-Wextra", "-shared",
           "-fPIC", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P, I64, I32, D = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
            lib.oracle_reshape_and_cache.restype = ctypes.c_int
            lib.oracle_reshape_and_cache.argtypes = [P, P, P, I64, I32, I32, P, P, I64, I32]
            lib.oracle_attention_varlen.restype = ctypes.c_int
            lib.oracle_attention_varlen.argtypes = [
                P, P, P, P, P, P, I32, I32, I32, I32, I64, I32, I32, D, P, I64, P, I32]
            for name in ("oracle_kv_export", "oracle_kv_import"):
                fn = getattr(lib, name)
                fn.restype = ctypes.c_int
                fn.argtypes = [P, P, I64, I32, I32, I32, P, I32, P, I32, P, P]
            lib.oracle_default_threads.restype = ctypes.c_int
            lib.oracle_default_threads.argtypes = []
            _lib = lib
    return _lib


def default_threads() -> int:
    """Threads the oracle's OpenMP region uses when none are requested."""
    return int(_load().oracle_default_threads())


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _bits(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError(f"bf16 data must be passed as uint16 bit patterns, got {a.dtype}")
    return a


def _check(rc: int):
    if rc != 0:
        raise OracleError(_ERRORS.get(rc, f"oracle error {rc}"))


def reshape_and_cache(k: np.ndarray, v: np.ndarray, slot_mapping: np.ndarray,
                      k_cache: np.ndarray, v_cache: np.ndarray) -> None:
    """Write k[t], v[t] into the caches at slot slot_mapping[t], in place.

    k, v: uint16 [T, Hkv, D]; slot_mapping: int64 [T]; caches: uint16
    [NB, block_size, Hkv, D], modified in place.  Negative slots are skipped.
    """
    k, v = _bits(k), _bits(v)
    if not (k_cache.flags.c_contiguous and v_cache.flags.c_contiguous):
        raise ValueError("caches must be C-contiguous (they are written in place)")
    _bits(k_cache), _bits(v_cache)
    slots = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    T, Hkv, D = k.shape
    NB, B = k_cache.shape[0], k_cache.shape[1]
    if v.shape != k.shape or v_cache.shape != k_cache.shape or k_cache.shape[2:] != (Hkv, D):
        raise ValueError("shape mismatch")
    if slots.shape != (T,):
        raise ValueError("slot_mapping must be [T]")
    _check(_load().oracle_reshape_and_cache(_ptr(k), _ptr(v), _ptr(slots), T, Hkv, D,
                                            _ptr(k_cache), _ptr(v_cache), NB, B))


def attention_varlen(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray,
                     block_tables: np.ndarray, cu_seqlens_q: np.ndarray,
                     seq_lens: np.ndarray, scale: float,
                     rows: np.ndarray | None = None,
                     threads: int = 0) -> np.ndarray:
    """Causal varlen attention over the paged cache, in fp64.

    q: uint16 [T, Hq, D]; caches: uint16 [NB, block_size, Hkv, D];
    block_tables: int32 [S, MB]; cu_seqlens_q: int32 [S+1]; seq_lens: int32 [S].
    Returns float64 [T, Hq, D], or [len(rows), D] when ``rows`` (flat ids
    token * Hq + head) is given.
    """
    q, k_cache, v_cache = _bits(q), _bits(k_cache), _bits(v_cache)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cu = np.ascontiguousarray(cu_seqlens_q, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    T, Hq, D = q.shape
    NB, B, Hkv, D2 = k_cache.shape
    if D2 != D or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch")
    S = sl.shape[0]
    if cu.shape != (S + 1,) or (S and cu[-1] != T):
        raise ValueError("cu_seqlens_q must be [S+1] and end at T")
    if bt.ndim != 2 or bt.shape[0] != S:
        raise ValueError("block_tables must be [S, MB]")
    MB = bt.shape[1]
    if rows is not None:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        out = np.empty((rows.shape[0], D), dtype=np.float64)
        n_rows = rows.shape[0]
    else:
        out = np.empty((T, Hq, D), dtype=np.float64)
        n_rows = 0
    if S == 0:
        cu = np.zeros(1, dtype=np.int32)
    _check(_load().oracle_attention_varlen(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(bt), _ptr(cu), _ptr(sl),
        S, Hq, Hkv, D, NB, MB, B, float(scale), _ptr(rows), n_rows, _ptr(out),
        int(threads)))
    return out


def _kv_args(cache_k, cache_v, block_tables, cu_tokens, buf_k, buf_v):
    NB, B, Hkv, D = cache_k.shape
    if cache_v.shape != cache_k.shape or buf_k.shape != buf_v.shape or tuple(buf_k.shape[1:]) != (Hkv, D):
        raise ValueError("shape mismatch")
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    cu = np.ascontiguousarray(cu_tokens, dtype=np.int32)
    S = bt.shape[0]
    if bt.ndim != 2 or cu.shape != (S + 1,) or cu[-1] != buf_k.shape[0]:
        raise ValueError("block_tables must be [S, MB] and cu_tokens [S+1] ending at N")
    return NB, B, Hkv, D, bt, cu, S


def kv_export(k_cache: np.ndarray, v_cache: np.ndarray, block_tables: np.ndarray,
              cu_tokens: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """K/V of requests gathered from the caches into contiguous buffers.

    Request i's token p (0 <= p < cu_tokens[i+1] - cu_tokens[i]) is read
    from block block_tables[i][p // block_size], row p % block_size, and
    becomes row cu_tokens[i] + p of the returned uint16 [N, Hkv, D] arrays.
    """
    k_cache, v_cache = _bits(k_cache), _bits(v_cache)
    N = int(np.asarray(cu_tokens)[-1])
    k_out = np.zeros((N,) + k_cache.shape[2:], dtype=np.uint16)
    v_out = np.zeros_like(k_out)
    NB, B, Hkv, D, bt, cu, S = _kv_args(k_cache, v_cache, block_tables, cu_tokens, k_out, v_out)
    _check(_load().oracle_kv_export(_ptr(k_cache), _ptr(v_cache), NB, B, Hkv, D, _ptr(bt), bt.shape[1],
                                    _ptr(cu), S, _ptr(k_out), _ptr(v_out)))
    return k_out, v_out


def kv_import(k_in: np.ndarray, v_in: np.ndarray, block_tables: np.ndarray, cu_tokens: np.ndarray,
              k_cache: np.ndarray, v_cache: np.ndarray) -> None:
    """Write contiguous K/V buffers into the caches (in place) through the
    block tables: the inverse of kv_export for the slots the requests use."""
    k_in, v_in = _bits(k_in), _bits(v_in)
    if not (k_cache.flags.c_contiguous and v_cache.flags.c_contiguous):
        raise ValueError("caches must be C-contiguous (they are written in place)")
    _bits(k_cache), _bits(v_cache)
    NB, B, Hkv, D, bt, cu, S = _kv_args(k_cache, v_cache, block_tables, cu_tokens, k_in, v_in)
    _check(_load().oracle_kv_import(_ptr(k_in), _ptr(v_in), NB, B, Hkv, D, _ptr(bt), bt.shape[1],
                                    _ptr(cu), S, _ptr(k_cache), _ptr(v_cache)))
