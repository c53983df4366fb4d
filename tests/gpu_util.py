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


def bf16_step(x):
    """Spacing of bf16 values at magnitude |x| (2^(e-7) for |x| in [2^e, 2^(e+1)))."""
    return np.exp2(np.floor(np.log2(np.maximum(np.abs(x), 1e-300))) - 7)


def assert_attn_close(got, ref, what=""):
    """The attention tolerance: every element within max-abs 1e-2 of the
    fp64 result, or -- where one bf16 step exceeds that (|x| >= 2, rows
    carried by one or two keys) -- less than one bf16 step from it (the
    kernel's fp32 result may lie on the other side of a rounding midpoint);
    mean-abs over all elements <= 1e-3."""
    err = np.abs(got - ref)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    mx, mean = float(err.max(initial=0.0)), float(err.mean()) if err.size else 0.0
    bad = (err > MAX_ABS) & (err >= bf16_step(np.maximum(np.abs(got), np.abs(ref))))
    if bad.any() or not mean <= MEAN_ABS:
        at = np.unravel_index(int(np.argmax(np.where(bad, err, 0.0) if bad.any() else err)), err.shape)
        raise AssertionError(f"{what}: max-abs {mx:.3e} mean-abs {mean:.3e}; worst at {tuple(int(i) for i in at)}: "
                             f"got {float(got[at]):.6f}, expected {float(ref[at]):.6f}; "
                             f"{int(bad.sum())} of {err.size} beyond the tolerance")
    return mx, mean


def bf16_round(x):
    """fp64 values rounded to bf16 (nearest even), back as fp64: the closest
    a bf16 output can be to the oracle."""
    t = torch.from_numpy(np.ascontiguousarray(x, np.float64)).to(torch.float32).to(torch.bfloat16)
    return t.to(torch.float64).numpy()


def assert_attn_close_bf16(got, exact, what=""):
    """For inputs whose softmax is near one-hot (large |q|), where each output
    is close to a single V row of magnitude up to ~5: the output is bf16, and
    where the exact result lies within the kernel's (fp32) error of a bf16
    rounding midpoint, either neighbouring bf16 value is a correct output --
    one bf16 step is 2^-6 at [2, 4) and 2^-5 at [4, 8), above the max-abs
    tolerance.  So an element passes if it is within max-abs 1e-2 of the
    exact result or one of the two bf16 values next to it (less than one
    bf16 step away); the mean-abs bound is taken against the exact result
    rounded to bf16, since rounding alone reaches ~1e-3 on such outputs."""
    err = np.abs(got - exact)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    mag = np.maximum(np.abs(got), np.abs(exact))
    bad = ~((err <= MAX_ABS) | (err < bf16_step(mag)))
    assert not bad.any(), f"{what}: {int(bad.sum())} outputs off by more than max-abs and one bf16 step, " \
                          f"worst {float(err[bad].max()):.3e}"
    mean = float(np.abs(got - bf16_round(exact)).mean())
    assert mean <= MEAN_ABS, f"{what}: mean-abs {mean:.3e} against the bf16-rounded result"
    return float(err.max()), mean
