"""fp64 CPU oracle for paged-KV attention -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  It is independent of the CUDA library: it
shares no code with it and neither imports the other.  Arrays cross this
boundary as numpy arrays holding the stored bit patterns (bf16 as uint16,
fp8 E4M3 as uint8), which the C code decodes exactly to double.

Functions follow "Production Serving: Continuous Batching and PagedAttention"
(The Build, Step 4 "Implement the paged KV cache" and Step 6 "Implement
attention over paged storage") read per query head, and "Continuous batching
and PagedAttention" (How the scheduler works: chunked prefill; PagedAttention:
KV cache memory: copy-on-write).  The C source lists every reading taken
where the pages are silent.
"""
import ctypes as C
import os

import numpy as np

from . import build as _build

BF16, FP8_E4M3 = 0, 1
BLOCK_SIZE = 16

_lib = None


def load(path):
    """Open an oracle shared object at ``path`` and declare its signatures."""
    L = C.CDLL(path)
    p = C.c_void_p
    i32, i64, dbl = C.c_int, C.c_int64, C.c_double
    L.oracle_bf16_to_double.argtypes = [C.c_uint16]
    L.oracle_bf16_to_double.restype = dbl
    L.oracle_e4m3_to_double.argtypes = [C.c_uint8]
    L.oracle_e4m3_to_double.restype = dbl
    L.oracle_e4m3_from_float.argtypes = [C.c_float]
    L.oracle_e4m3_from_float.restype = C.c_uint8
    L.oracle_write_kv.argtypes = [p, p, p, i64, p, p, i32, i64, i32, i32, p, p]
    L.oracle_copy_blocks.argtypes = [p, p, p, i32, i32, i64, i32, i32]
    L.oracle_decode.argtypes = [p, p, p, p, i32, p, p, i32, i32, i32, i32, i32, i64, dbl, p, p, i32]
    L.oracle_decode_split.argtypes = [p, p, p, p, i32, p, p, i32, i32, i32, i32, i32, i64, dbl, p, p,
                                      i32, i32]
    L.oracle_prefill.argtypes = [p, p, p, p, p, i32, i32, i32, i32, i32, p, p, i32, i64, dbl, p, p, i32]
    for f in ("oracle_write_kv", "oracle_copy_blocks", "oracle_decode", "oracle_decode_split",
              "oracle_prefill", "oracle_max_threads"):
        getattr(L, f).restype = i32
    return L


def lib():
    global _lib
    if _lib is None:
        _lib = load(_build.build())
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _dtype_code(cache):
    if cache.dtype == np.uint16:
        return BF16
    if cache.dtype == np.uint8:
        return FP8_E4M3
    raise TypeError("cache must hold uint16 (bf16 bits) or uint8 (E4M3 codes)")


def _scales(dt, k_scale, v_scale, hkv):
    if dt == BF16:
        return None, None
    ks = _c(k_scale, np.float32)
    vs = _c(v_scale, np.float32)
    assert ks.shape == (hkv,) and vs.shape == (hkv,)
    return ks, vs


class OracleError(RuntimeError):
    pass


def _check(rc, what):
    if rc != 0:
        raise OracleError(f"{what}: status {rc} (bad block id / slot or inconsistent arguments)")


def max_threads() -> int:
    return int(lib().oracle_max_threads())


def bf16_to_double(bits: int) -> float:
    return float(lib().oracle_bf16_to_double(int(bits)))


def e4m3_to_double(code: int) -> float:
    return float(lib().oracle_e4m3_to_double(int(code)))


def e4m3_from_float(x: float) -> int:
    return int(lib().oracle_e4m3_from_float(float(np.float32(x))))


def write_kv(k, v, slot_mapping, k_cache, v_cache, k_scale=None, v_scale=None):
    """In-place slot-mapped write of k, v (uint16 bf16 bits, [T, Hkv, D]) into
    the caches ([num_blocks, Hkv, 16, D]); returns nothing."""
    dt = _dtype_code(k_cache)
    nb, hkv, bs, d = k_cache.shape
    assert bs == BLOCK_SIZE and v_cache.shape == k_cache.shape and v_cache.dtype == k_cache.dtype
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    sm = _c(slot_mapping, np.int64)
    assert k.shape == (sm.shape[0], hkv, d) and v.shape == k.shape
    ks, vs = _scales(dt, k_scale, v_scale, hkv)
    _check(lib().oracle_write_kv(_ptr(k), _ptr(v), _ptr(sm), sm.shape[0], _ptr(k_cache), _ptr(v_cache), dt,
                                 nb, hkv, d, _ptr(ks), _ptr(vs)), "write_kv")


def copy_blocks(k_cache, v_cache, pairs):
    """In-place copy of whole physical blocks, pairs int32 [n, 2] = (src, dst)."""
    dt = _dtype_code(k_cache)
    nb, hkv, bs, d = k_cache.shape
    pr = _c(pairs, np.int32).reshape(-1, 2)
    _check(lib().oracle_copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(pr), pr.shape[0], dt, nb, hkv, d),
           "copy_blocks")


def decode(q, k_cache, v_cache, block_tables, seq_lens, scale, k_scale=None, v_scale=None, nthreads=0,
           partition_tokens=None):
    """Paged decode, dense definition.  q uint16 [B, Hq, D]; returns float64
    [B, Hq, D].  With ``partition_tokens`` the split-K form with its
    log-sum-exp merge is evaluated instead."""
    dt = _dtype_code(k_cache)
    nb, hkv, bs, d = k_cache.shape
    q = _c(q, np.uint16)
    b, hq, dq = q.shape
    assert dq == d
    bt = _c(block_tables, np.int32)
    sl = _c(seq_lens, np.int32)
    assert bt.shape[0] == b and sl.shape == (b,)
    ks, vs = _scales(dt, k_scale, v_scale, hkv)
    out = np.zeros((b, hq, d), np.float64)
    if partition_tokens is None:
        rc = lib().oracle_decode(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), dt, _ptr(bt), _ptr(sl), b,
                                 bt.shape[1], hq, hkv, d, nb, float(scale), _ptr(ks), _ptr(vs), int(nthreads))
    else:
        rc = lib().oracle_decode_split(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), dt, _ptr(bt), _ptr(sl),
                                       b, bt.shape[1], hq, hkv, d, nb, float(scale), _ptr(ks), _ptr(vs),
                                       int(partition_tokens), int(nthreads))
    _check(rc, "decode")
    return out


def prefill(q, cu_q, prefix_lens, block_tables, k_cache, v_cache, scale, k_scale=None, v_scale=None,
            nthreads=0):
    """Causal chunked prefill.  q uint16 [sum C, Hq, D]; cu_q int32 [n+1];
    prefix_lens int32 [n]; block_tables int32 [n, max_blocks].  Returns
    float64 [sum C, Hq, D]."""
    dt = _dtype_code(k_cache)
    nb, hkv, bs, d = k_cache.shape
    q = _c(q, np.uint16)
    total, hq, dq = q.shape
    assert dq == d
    cu = _c(cu_q, np.int32)
    pl = _c(prefix_lens, np.int32)
    bt = _c(block_tables, np.int32)
    n = pl.shape[0]
    assert cu.shape == (n + 1,) and cu[-1] == total and bt.shape[0] == n
    ks, vs = _scales(dt, k_scale, v_scale, hkv)
    out = np.zeros((total, hq, d), np.float64)
    _check(lib().oracle_prefill(_ptr(out), _ptr(q), _ptr(cu), _ptr(pl), _ptr(bt), n, bt.shape[1], hq, hkv, d,
                                _ptr(k_cache), _ptr(v_cache), dt, nb, float(scale), _ptr(ks), _ptr(vs),
                                int(nthreads)), "prefill")
    return out
