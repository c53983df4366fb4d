"""Helpers for the GPU parity tests: move seeded host inputs to the device,
call the library through its binding, and compare with the oracle."""
import numpy as np
import torch

from paged_kv_cache_408_b200 import ops

MAX_ABS = 1e-2   # attention-output tolerance against the fp64 oracle
MEAN_ABS = 1e-3


def dev_bf16(a, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(a, np.uint16).view(np.int16)).view(torch.bfloat16).to(device)


def dev_u8(a, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(a, np.uint8)).to(device)


def dev(a, dtype, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(a, dtype)).to(device)


def host_bits(t):
    """Device bf16 / uint8 tensor -> numpy bit patterns."""
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def to_float(out_bf16):
    return out_bf16.detach().float().cpu().numpy().astype(np.float64)


def cache_to_device(case, device="cuda"):
    if case.fp8:
        return dev_u8(case.k_cache, device), dev_u8(case.v_cache, device)
    return dev_bf16(case.k_cache, device), dev_bf16(case.v_cache, device)


def run_decode(case, kc, vc, seq_lens=None, partition_tokens=0, block_tables=None, q=None):
    lens = case.seq_lens if seq_lens is None else seq_lens
    bt = case.block_tables if block_tables is None else block_tables
    qh = case.q if q is None else q
    qd = dev_bf16(qh)
    out = torch.empty_like(qd)
    B, Hq, D = qh.shape
    ws = ops.alloc_workspace(B, Hq, D, bt.shape[1], partition_tokens, device=kc.device)
    ks = vs = None
    if case.fp8:
        ks, vs = dev(case.k_scale, np.float32), dev(case.v_scale, np.float32)
    ops.decode(out, qd, kc, vc, dev(bt, np.int32), dev(lens, np.int32), case.scale, ks, vs, ws, partition_tokens)
    torch.cuda.synchronize()
    return out


def assert_attn_close(got, ref, what=""):
    err = np.abs(got - ref)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    mx, mean = float(err.max(initial=0.0)), float(err.mean()) if err.size else 0.0
    assert mx <= MAX_ABS and mean <= MEAN_ABS, f"{what}: max-abs {mx:.3e} mean-abs {mean:.3e}"
    return mx, mean


def bf16_round(x):
    """fp64 values rounded to bf16 (nearest even), back as fp64: the closest
    a bf16 output can be to the oracle."""
    t = torch.from_numpy(np.ascontiguousarray(x, np.float64)).to(torch.float32).to(torch.bfloat16)
    return t.to(torch.float64).numpy()
