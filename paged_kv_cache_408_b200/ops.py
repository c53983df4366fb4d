"""Thin ctypes binding of ``libpa.so`` (declared in ``include/pa.h``).

Argument marshalling only: each function checks tensor devices, dtypes and
shapes, turns tensors into raw device pointers and calls the C entry point of
the same name on the current torch stream.  Every step of the computation
runs in the library's CUDA kernels; there is no fallback.  If the library is
missing, ``lib()`` raises immediately.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpa.so")

BLOCK_SIZE = 16
PA_OK = 0
DTYPE_BF16, DTYPE_FP8_E4M3 = 0, 1

DEVERR_BAD_BLOCK, DEVERR_BAD_SLOT, DEVERR_BAD_LEN, DEVERR_BAD_PAIR, DEVERR_TIMEOUT = 0x1, 0x2, 0x4, 0x8, 0x10
DEVERR_LAYOUT = 0x20

EXPORTED = (
    "pa_write_kv", "pa_copy_blocks", "pa_decode_workspace_size", "pa_decode", "pa_prefill_chunk",
    "pa_get_last_device_error", "pa_status_string", "pa_version", "pa_decode_noalloc",
    "pa_decode_cascade_workspace_size", "pa_decode_cascade",
)


class PAError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} failed: {status_string(status)} ({status})")


class CacheDesc(C.Structure):
    _fields_ = [("num_blocks", C.c_int64), ("num_kv_heads", C.c_int32), ("block_size", C.c_int32),
                ("head_dim", C.c_int32), ("dtype", C.c_int32)]


_lib = None


def lib():
    """Load libpa.so once; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libpa.so not found at {LIB_PATH}: build it with "
                               "`python -m paged_kv_cache_408_b200.build` (no CPU fallback exists)")
        L = C.CDLL(LIB_PATH)
        p, i32, i64, f32, sz = C.c_void_p, C.c_int32, C.c_int64, C.c_float, C.c_size_t
        L.pa_write_kv.argtypes = [p, p, p, i64, p, p, p, p, C.POINTER(CacheDesc), p]
        L.pa_copy_blocks.argtypes = [p, p, p, i32, C.POINTER(CacheDesc), p]
        L.pa_decode_workspace_size.argtypes = [i32, i32, i32, i32, i32, C.POINTER(sz)]
        L.pa_decode.argtypes = [p, p, p, p, p, p, i32, i32, i32, f32, p, p, i32, p, sz, C.POINTER(CacheDesc), p]
        L.pa_prefill_chunk.argtypes = [p, p, p, p, p, i32, i32, i32, i32, i32, p, p, f32, p, p,
                                       C.POINTER(CacheDesc), p]
        L.pa_get_last_device_error.argtypes = [C.POINTER(C.c_uint32), p]
        L.pa_decode_noalloc.argtypes = [p, p, p, p, p, p, i32, i32, i32, f32, p, p, i32, C.POINTER(CacheDesc), p]
        L.pa_decode_cascade_workspace_size.argtypes = [i32, i32, i32, i32, C.POINTER(CacheDesc), C.POINTER(sz)]
        L.pa_decode_cascade.argtypes = [p, p, p, p, p, p, i32, i32, i32, f32, p, p, i32, p, sz,
                                        C.POINTER(CacheDesc), p]
        L.pa_status_string.argtypes = [C.c_int]
        L.pa_status_string.restype = C.c_char_p
        for f in EXPORTED:
            if f != "pa_status_string":
                getattr(L, f).restype = C.c_int
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().pa_status_string(int(status)).decode()


def _check(fn, rc):
    if rc != PA_OK:
        raise PAError(fn, rc)


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def _need(t, name, dtype=None, device=None, contiguous=True):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


FP8_TYPES = (torch.uint8, torch.float8_e4m3fn)


def cache_desc(k_cache: torch.Tensor) -> CacheDesc:
    """Descriptor of a cache tensor [num_blocks, Hkv, 16, D] (bf16, or uint8 /
    float8_e4m3fn for E4M3)."""
    if k_cache.dim() != 4 or k_cache.shape[2] != BLOCK_SIZE:
        raise ValueError(f"cache must be [num_blocks, Hkv, {BLOCK_SIZE}, D], got {tuple(k_cache.shape)}")
    if k_cache.dtype == torch.bfloat16:
        dt = DTYPE_BF16
    elif k_cache.dtype in FP8_TYPES:
        dt = DTYPE_FP8_E4M3
    else:
        raise TypeError(f"unsupported cache dtype {k_cache.dtype}")
    nb, hkv, bs, d = k_cache.shape
    return CacheDesc(nb, hkv, bs, d, dt)


def _caches(k_cache, v_cache):
    _need(k_cache, "k_cache", (torch.bfloat16,) + FP8_TYPES)
    _need(v_cache, "v_cache", k_cache.dtype, k_cache.device)
    if v_cache.shape != k_cache.shape:
        raise ValueError("k_cache and v_cache shapes differ")
    return cache_desc(k_cache)


def _scales(desc, k_scale, v_scale, device):
    if desc.dtype != DTYPE_FP8_E4M3:
        return None, None
    if k_scale is None or v_scale is None:
        raise ValueError("an fp8 cache needs k_scale and v_scale")
    _need(k_scale, "k_scale", torch.float32, device)
    _need(v_scale, "v_scale", torch.float32, device)
    if k_scale.numel() != desc.num_kv_heads or v_scale.numel() != desc.num_kv_heads:
        raise ValueError("scales must have one entry per kv head")
    return k_scale, v_scale


def write_kv(k, v, slot_mapping, k_cache, v_cache, k_scale=None, v_scale=None, stream=None):
    """pa_write_kv: k, v bf16 [T, Hkv, D]; slot_mapping int64 [T]."""
    desc = _caches(k_cache, v_cache)
    dev = k_cache.device
    _need(k, "k", torch.bfloat16, dev)
    _need(v, "v", torch.bfloat16, dev)
    _need(slot_mapping, "slot_mapping", torch.int64, dev)
    T = slot_mapping.numel()
    if k.shape != (T, desc.num_kv_heads, desc.head_dim) or v.shape != k.shape:
        raise ValueError(f"k/v must be [T={T}, Hkv, D], got {tuple(k.shape)}")
    ks, vs = _scales(desc, k_scale, v_scale, dev)
    _check("pa_write_kv", lib().pa_write_kv(_ptr(k), _ptr(v), _ptr(slot_mapping), T, _ptr(k_cache), _ptr(v_cache),
                                            _ptr(ks), _ptr(vs), C.byref(desc), _stream(stream)))


def copy_blocks(k_cache, v_cache, pairs, stream=None):
    """pa_copy_blocks: pairs int32 [n, 2] = (src, dst)."""
    desc = _caches(k_cache, v_cache)
    _need(pairs, "pairs", torch.int32, k_cache.device)
    if pairs.numel() % 2:
        raise ValueError("pairs must be [n, 2]")
    _check("pa_copy_blocks", lib().pa_copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(pairs), pairs.numel() // 2,
                                                  C.byref(desc), _stream(stream)))


def decode_workspace_size(num_seqs, num_q_heads, head_dim, max_blocks_per_seq, partition_tokens=0) -> int:
    out = C.c_size_t(0)
    _check("pa_decode_workspace_size", lib().pa_decode_workspace_size(
        int(num_seqs), int(num_q_heads), int(head_dim), int(max_blocks_per_seq), int(partition_tokens),
        C.byref(out)))
    return int(out.value)


def alloc_workspace(num_seqs, num_q_heads, head_dim, max_blocks_per_seq, partition_tokens=0, device=None):
    """Caller-side helper: a torch buffer large enough for pa_decode (it
    needs no particular contents; zero-filled here only to be deterministic)."""
    n = decode_workspace_size(num_seqs, num_q_heads, head_dim, max_blocks_per_seq, partition_tokens)
    return torch.zeros(max(n, 256), dtype=torch.uint8, device=device)


def decode(out, q, k_cache, v_cache, block_tables, seq_lens, scale, k_scale=None, v_scale=None, workspace=None,
           partition_tokens=0, stream=None):
    """pa_decode: q, out bf16 [B, Hq, D]; block_tables int32 [B, max_blocks];
    seq_lens int32 [B]; workspace a uint8 CUDA buffer (see
    decode_workspace_size)."""
    desc = _caches(k_cache, v_cache)
    dev = k_cache.device
    _need(q, "q", torch.bfloat16, dev)
    _need(out, "out", torch.bfloat16, dev)
    _need(block_tables, "block_tables", torch.int32, dev)
    _need(seq_lens, "seq_lens", torch.int32, dev)
    B, Hq, D = q.shape
    if out.shape != q.shape or D != desc.head_dim:
        raise ValueError("out/q shape mismatch")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or seq_lens.shape != (B,):
        raise ValueError("block_tables must be [B, max_blocks] and seq_lens [B]")
    ks, vs = _scales(desc, k_scale, v_scale, dev)
    ws_bytes = 0
    if workspace is not None:
        _need(workspace, "workspace", None, dev)
        ws_bytes = workspace.numel() * workspace.element_size()
    _check("pa_decode", lib().pa_decode(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(seq_lens), B,
        block_tables.shape[1], Hq, float(scale), _ptr(ks), _ptr(vs), int(partition_tokens), _ptr(workspace),
        ws_bytes, C.byref(desc), _stream(stream)))


def decode_noalloc(out, q, k_cache, v_cache, block_tables, seq_lens, scale, k_scale=None, v_scale=None,
                   partition_tokens=0, stream=None):
    """pa_decode_noalloc: pa_decode without a caller workspace, for callers
    that cannot allocate device memory; the library's fixed 16 MiB scratch is
    used instead (shapes that need more raise PAError with
    PA_ERR_WORKSPACE).  Calls must not overlap on the GPU."""
    desc = _caches(k_cache, v_cache)
    dev = k_cache.device
    _need(q, "q", torch.bfloat16, dev)
    _need(out, "out", torch.bfloat16, dev)
    _need(block_tables, "block_tables", torch.int32, dev)
    _need(seq_lens, "seq_lens", torch.int32, dev)
    B, Hq, D = q.shape
    if out.shape != q.shape or D != desc.head_dim:
        raise ValueError("out/q shape mismatch")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or seq_lens.shape != (B,):
        raise ValueError("block_tables must be [B, max_blocks] and seq_lens [B]")
    ks, vs = _scales(desc, k_scale, v_scale, dev)
    _check("pa_decode_noalloc", lib().pa_decode_noalloc(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(seq_lens), B,
        block_tables.shape[1], Hq, float(scale), _ptr(ks), _ptr(vs), int(partition_tokens), C.byref(desc),
        _stream(stream)))


def cascade_workspace_size(num_seqs, num_q_heads, max_blocks_per_seq, prefix_blocks, k_cache) -> int:
    desc = cache_desc(k_cache)
    out = C.c_size_t(0)
    _check("pa_decode_cascade_workspace_size", lib().pa_decode_cascade_workspace_size(
        int(num_seqs), int(num_q_heads), int(max_blocks_per_seq), int(prefix_blocks), C.byref(desc), C.byref(out)))
    return int(out.value)


def alloc_cascade_workspace(num_seqs, num_q_heads, max_blocks_per_seq, prefix_blocks, k_cache):
    """Caller-side helper: a torch buffer large enough for pa_decode_cascade
    (no particular contents needed)."""
    n = cascade_workspace_size(num_seqs, num_q_heads, max_blocks_per_seq, prefix_blocks, k_cache)
    return torch.zeros(max(n, 256), dtype=torch.uint8, device=k_cache.device)


def decode_cascade(out, q, k_cache, v_cache, block_tables, seq_lens, scale, prefix_blocks, workspace,
                   k_scale=None, v_scale=None, stream=None):
    """pa_decode_cascade: pa_decode for sequences whose first prefix_blocks
    block-table entries are the same physical blocks in every row (the
    shared prefix is attended once per kv head on the tensor cores)."""
    desc = _caches(k_cache, v_cache)
    dev = k_cache.device
    _need(q, "q", torch.bfloat16, dev)
    _need(out, "out", torch.bfloat16, dev)
    _need(block_tables, "block_tables", torch.int32, dev)
    _need(seq_lens, "seq_lens", torch.int32, dev)
    _need(workspace, "workspace", None, dev)
    B, Hq, D = q.shape
    if out.shape != q.shape or D != desc.head_dim:
        raise ValueError("out/q shape mismatch")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or seq_lens.shape != (B,):
        raise ValueError("block_tables must be [B, max_blocks] and seq_lens [B]")
    ks, vs = _scales(desc, k_scale, v_scale, dev)
    _check("pa_decode_cascade", lib().pa_decode_cascade(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(seq_lens), B,
        block_tables.shape[1], Hq, float(scale), _ptr(ks), _ptr(vs), int(prefix_blocks), _ptr(workspace),
        workspace.numel() * workspace.element_size(), C.byref(desc), _stream(stream)))


def prefill_chunk(out, q, cu_q_lens, prefix_lens, block_tables, k_cache, v_cache, scale, max_q_len,
                  k_scale=None, v_scale=None, stream=None):
    """pa_prefill_chunk: q, out bf16 [total_q, Hq, D]; cu_q_lens int32 [n+1];
    prefix_lens int32 [n]; block_tables int32 [n, max_blocks]."""
    desc = _caches(k_cache, v_cache)
    dev = k_cache.device
    _need(q, "q", torch.bfloat16, dev)
    _need(out, "out", torch.bfloat16, dev)
    _need(cu_q_lens, "cu_q_lens", torch.int32, dev)
    _need(prefix_lens, "prefix_lens", torch.int32, dev)
    _need(block_tables, "block_tables", torch.int32, dev)
    n = prefix_lens.numel()
    if cu_q_lens.numel() != n + 1 or block_tables.dim() != 2 or block_tables.shape[0] != n:
        raise ValueError("cu_q_lens must be [n+1], block_tables [n, max_blocks]")
    total, Hq, D = q.shape
    if out.shape != q.shape or D != desc.head_dim:
        raise ValueError("out/q shape mismatch")
    ks, vs = _scales(desc, k_scale, v_scale, dev)
    _check("pa_prefill_chunk", lib().pa_prefill_chunk(
        _ptr(out), _ptr(q), _ptr(cu_q_lens), _ptr(prefix_lens), _ptr(block_tables), n, block_tables.shape[1], Hq,
        int(max_q_len), total, _ptr(k_cache), _ptr(v_cache), float(scale), _ptr(ks), _ptr(vs), C.byref(desc),
        _stream(stream)))


def get_last_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    flags = C.c_uint32(0)
    rc = lib().pa_get_last_device_error(C.byref(flags), _stream(stream))
    if rc not in (PA_OK, -5):
        raise PAError("pa_get_last_device_error", rc)
    return int(flags.value)
