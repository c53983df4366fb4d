"""The C-ABI library loads on a machine without a GPU, exports every symbol
include/pa.h declares, and rejects bad arguments on the host before any
device work (no compute call is made here)."""
import ctypes as C
import os
import re

import pytest

from paged_kv_cache_408_b200 import ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = C.c_void_p(0x10000)  # never dereferenced: every call below fails validation first


def header_functions():
    text = open(os.path.join(ROOT, "include", "pa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(pa_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    fns = header_functions()
    for f in ("pa_write_kv", "pa_decode", "pa_decode_workspace_size", "pa_prefill_chunk", "pa_copy_blocks",
              "pa_get_last_device_error", "pa_status_string"):
        assert f in fns


def test_library_exports_every_declared_symbol():
    L = ops.lib()
    for f in header_functions():
        assert hasattr(L, f), f


def test_status_strings_and_version():
    assert ops.status_string(0) == "PA_OK"
    assert ops.status_string(-1) == "PA_ERR_INVALID_ARG"
    assert ops.status_string(-3) == "PA_ERR_WORKSPACE"
    assert ops.lib().pa_version() >= 100


def desc(nb=64, hkv=8, bs=16, d=128, dt=0):
    return ops.CacheDesc(nb, hkv, bs, d, dt)


def call_decode(d, B=4, maxb=8, Hq=32, part=0, ws=None, ws_bytes=0, ptr=FAKE):
    return ops.lib().pa_decode(ptr, ptr, ptr, ptr, ptr, ptr, B, maxb, Hq, 0.1, ptr, ptr, part, ws, ws_bytes,
                               C.byref(d) if d is not None else None, None)


def test_decode_rejects_bad_arguments_on_host():
    assert call_decode(None) == -1
    assert call_decode(desc(bs=8)) == -1
    assert call_decode(desc(d=96)) == -2
    assert call_decode(desc(dt=7)) == -1
    assert call_decode(desc(), Hq=30) == -1          # Hq % Hkv != 0
    assert call_decode(desc(hkv=2), Hq=32) == -2     # group of 16 not built
    assert call_decode(desc(), B=5000) == -1
    assert call_decode(desc(), part=20) == -1        # not a multiple of 16
    assert call_decode(desc(), part=4096) == -1      # above the largest partition
    assert call_decode(desc(), ptr=None) == -1       # null pointers
    # several partitions need a workspace of the reported size
    assert call_decode(desc(), maxb=64, part=256) == -3
    assert call_decode(desc(), B=0) == 0             # nothing to do


def test_workspace_size():
    assert ops.decode_workspace_size(64, 32, 128, 16, 256) == 0  # one partition: no workspace
    n = ops.decode_workspace_size(64, 32, 128, 128, 256)          # 2048 tokens -> 8 partitions
    assert n >= 64 * 32 * 8 * (128 + 1) * 4
    assert ops.decode_workspace_size(64, 32, 128, 128, 512) < n
    with pytest.raises(ops.PAError):
        ops.decode_workspace_size(64, 32, 96, 128)


def test_write_and_copy_reject_bad_arguments_on_host():
    L = ops.lib()
    d = desc()
    assert L.pa_write_kv(FAKE, FAKE, FAKE, 4, FAKE, FAKE, None, None, C.byref(desc(d=80)), None) == -2
    assert L.pa_write_kv(FAKE, FAKE, FAKE, -1, FAKE, FAKE, None, None, C.byref(d), None) == -1
    assert L.pa_write_kv(FAKE, FAKE, FAKE, 0, FAKE, FAKE, None, None, C.byref(d), None) == 0
    assert L.pa_write_kv(FAKE, FAKE, FAKE, 4, FAKE, FAKE, None, None, C.byref(desc(dt=1)), None) == -1  # fp8 needs scales
    assert L.pa_write_kv(None, FAKE, FAKE, 4, FAKE, FAKE, None, None, C.byref(d), None) == -1
    assert L.pa_copy_blocks(FAKE, FAKE, FAKE, -2, C.byref(d), None) == -1
    assert L.pa_copy_blocks(FAKE, FAKE, FAKE, 0, C.byref(d), None) == 0
    assert L.pa_copy_blocks(None, FAKE, FAKE, 3, C.byref(d), None) == -1


def test_prefill_rejects_bad_arguments_on_host():
    L = ops.lib()
    assert L.pa_prefill_chunk(FAKE, FAKE, FAKE, FAKE, FAKE, 2, 8, 32, 64, 100, FAKE, FAKE, 0.1, None, None,
                              C.byref(desc(dt=1)), None) == -1  # an fp8 cache needs its scales
    assert L.pa_prefill_chunk(FAKE, FAKE, FAKE, FAKE, FAKE, 2, 8, 30, 64, 100, FAKE, FAKE, 0.1, None, None,
                              C.byref(desc()), None) == -1
    assert L.pa_prefill_chunk(FAKE, FAKE, FAKE, FAKE, FAKE, 2, 8, 128, 64, 100, FAKE, FAKE, 0.1, None, None,
                              C.byref(desc()), None) == -2  # group of 16 not built
    assert L.pa_prefill_chunk(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 8, 32, 64, 100, FAKE, FAKE, 0.1, None, None,
                              C.byref(desc()), None) == 0


def test_misaligned_pointers_are_rejected():
    odd = C.c_void_p(0x10008)
    L = ops.lib()
    d = desc()
    assert L.pa_write_kv(odd, FAKE, FAKE, 4, FAKE, FAKE, None, None, C.byref(d), None) == -1
    assert L.pa_copy_blocks(odd, FAKE, FAKE, 3, C.byref(d), None) == -1


def call_cascade(d, B=4, maxb=8, Hq=32, pb=4, ws=FAKE, ws_bytes=1 << 30, ptr=FAKE, scales=FAKE):
    return ops.lib().pa_decode_cascade(ptr, ptr, ptr, ptr, ptr, ptr, B, maxb, Hq, 0.1, scales, scales, pb, ws,
                                       ws_bytes, C.byref(d) if d is not None else None, None)


def test_cascade_rejects_bad_arguments_on_host():
    assert call_cascade(None) == -1
    assert call_cascade(desc(d=96)) == -2
    assert call_cascade(desc(), pb=9) == -1          # more shared blocks than the table holds
    assert call_cascade(desc(), pb=-1) == -1
    assert call_cascade(desc(), Hq=30) == -1
    assert call_cascade(desc(hkv=2), Hq=32) == -2    # group of 16 not built
    assert call_cascade(desc(), B=5000) == -1
    assert call_cascade(desc(), ptr=None) == -1
    assert call_cascade(desc(dt=1), scales=None) == -1  # fp8 needs its scales
    assert call_cascade(desc(), ws=None) == -3
    assert call_cascade(desc(), ws_bytes=1024) == -3
    assert call_cascade(desc(), ws=C.c_void_p(0x10010)) == -3  # not 256-byte aligned
    assert call_cascade(desc(), B=0) == 0


def cascade_ws(B, Hq, maxb, pb, dt=0, hkv=8, d=128):
    out = C.c_size_t(0)
    rc = ops.lib().pa_decode_cascade_workspace_size(B, Hq, maxb, pb, C.byref(desc(hkv=hkv, d=d, dt=dt)),
                                                    C.byref(out))
    return rc, out.value


def test_cascade_workspace_size():
    rc, n = cascade_ws(256, 64, 160, 128)
    assert rc == 0
    # split-K pieces of the 32-block suffix (at most 32/16 + 2) plus the prefix piece, fp32 o and lse
    assert n >= 256 * 64 * 5 * (128 + 1) * 4
    rc, n8 = cascade_ws(256, 64, 160, 128, dt=1)
    assert rc == 0 and n8 >= n + 2 * 128 * 8 * 16 * 128 * 2  # fp8: the prefix widened to bf16
    assert cascade_ws(256, 64, 160, 161)[0] == -1
    assert cascade_ws(256, 64, 160, -1)[0] == -1
    assert cascade_ws(256, 64, 160, 0)[1] >= ops.decode_workspace_size(256, 64, 128, 160)


def test_block_table_width_is_bounded():
    """Tables wider than PA_MAX_BLOCKS_PER_SEQ (2^24 entries) are rejected on
    the host by every entry point that takes one, before any size arithmetic
    could overflow; the largest accepted width still sizes its workspace."""
    L = ops.lib()
    big = (1 << 24) + 1
    out = C.c_size_t(0)
    assert L.pa_decode_workspace_size(4, 32, 128, big, 0, C.byref(out)) == -1
    assert L.pa_decode_workspace_size(4, 32, 128, 1 << 24, 0, C.byref(out)) == 0
    assert out.value >= 4 * 32 * ((1 << 24) // 16) * 128 * 4
    assert L.pa_decode_workspace_size(1, 1, 128, 1 << 24, 16, C.byref(out)) == 0  # 2^24 partitions, no wrap
    assert call_decode(desc(), maxb=big) == -1
    assert call_decode(desc(), maxb=(1 << 31) - 1) == -1
    assert call_cascade(desc(), maxb=big, pb=1) == -1
    assert cascade_ws(4, 32, big, 1)[0] == -1
    assert L.pa_prefill_chunk(FAKE, FAKE, FAKE, FAKE, FAKE, 2, big, 32, 64, 100, FAKE, FAKE, 0.1, None, None,
                              C.byref(desc()), None) == -1
    assert L.pa_decode_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, big, 32, 0.1, None, None, 0,
                               C.byref(desc()), None) == -1


def test_device_status_bits_match_the_header():
    """The binding's PA_DEVERR_* bits are the header's."""
    text = open(os.path.join(ROOT, "include", "pa.h")).read()
    bits = {m.group(1): int(m.group(2), 16) for m in re.finditer(r"#define PA_DEVERR_(\w+) (0x[0-9a-fA-F]+)u", text)}
    assert bits == {"BAD_BLOCK": ops.DEVERR_BAD_BLOCK, "BAD_SLOT": ops.DEVERR_BAD_SLOT, "BAD_LEN": ops.DEVERR_BAD_LEN,
                    "BAD_PAIR": ops.DEVERR_BAD_PAIR, "TIMEOUT": ops.DEVERR_TIMEOUT, "LAYOUT": ops.DEVERR_LAYOUT}
    assert len(set(bits.values())) == len(bits) and all(b & (b - 1) == 0 for b in bits.values())
