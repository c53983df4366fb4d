"""pa_decode_noalloc: paged decode for callers that cannot allocate device
memory (a plugin inside an engine whose pool already owns the GPU, or code
that must avoid the implicit synchronisation of cudaMalloc/cudaFree).

It uses the library's fixed device scratch instead of a caller workspace.
The GPU test calls it through the C ABI twice in a row, with different
batches, and checks each result against pa_decode with its own workspace.
This file is collected last on purpose."""
import ctypes as C

import numpy as np
import pytest
import torch

from gpu_util import MAX_ABS, MEAN_ABS, cache_to_device, dev, dev_bf16
from paged_kv_cache_408_b200 import inputs as I
from paged_kv_cache_408_b200 import ops

PA_ERR_WORKSPACE = -3


def _call_noalloc(out, q, kc, vc, bt, lens, scale, partition_tokens):
    desc = ops.cache_desc(kc)
    return ops.lib().pa_decode_noalloc(
        C.c_void_p(out.data_ptr()), C.c_void_p(q.data_ptr()), C.c_void_p(kc.data_ptr()),
        C.c_void_p(vc.data_ptr()), C.c_void_p(bt.data_ptr()), C.c_void_p(lens.data_ptr()), q.shape[0],
        bt.shape[1], q.shape[1], float(scale), None, None, int(partition_tokens), C.byref(desc),
        C.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_oversized_shape_is_rejected_before_any_device_work():
    # 2048 sequences x 32 heads x 2048 blocks needs far more than the 16 MiB scratch
    desc = ops.CacheDesc(4096, 8, 16, 128, 0)
    fake = C.c_void_p(0x10000)  # never dereferenced: the size check fails first
    rc = ops.lib().pa_decode_noalloc(fake, fake, fake, fake, fake, fake, 2048, 2048, 32, 0.1, None, None, 0,
                                     C.byref(desc), None)
    assert rc == PA_ERR_WORKSPACE


@pytest.mark.gpu
def test_noalloc_matches_decode_on_two_calls_in_a_row(cuda_device):
    cases = [(I.batch64_2k(3), 0), (I.make_decode_case(4, [1, 700, 33, 1500, 16, 257], 32, 8, 128), 256)]
    for c, part in cases:
        kc, vc = cache_to_device(c)
        q = dev_bf16(c.q)
        bt = dev(c.block_tables, np.int32)
        lens = dev(c.seq_lens, np.int32)
        ref = torch.empty_like(q)
        ws = ops.alloc_workspace(c.B, c.Hq, c.D, bt.shape[1], part, device=kc.device)
        ops.decode(ref, q, kc, vc, bt, lens, c.scale, workspace=ws, partition_tokens=part)
        got = torch.full_like(q, float("nan"))
        rc = _call_noalloc(got, q, kc, vc, bt, lens, c.scale, part)
        assert rc == 0, ops.status_string(rc)
        torch.cuda.synchronize()
        err = (got.float() - ref.float()).abs()
        assert torch.isfinite(got.float()).all()
        assert err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS, (err.max().item(), err.mean().item())
    assert ops.get_last_device_error() == 0
