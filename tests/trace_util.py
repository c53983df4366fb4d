"""Replay of scheduler-planned steps on the GPU and in the oracle.

The GPU side runs every step exactly as the benchmark enqueues it: the
step's metadata uploaded once (``DeviceStep``), then ``StepExecutor.enqueue``
-- copy_blocks, write_kv, decode (or cascade decode) with its merge, and
prefill -- as one programmatic launch chain on one stream, with no host
synchronisation inside the step.  The oracle side applies the same plan to a
host copy of the cache: ``oracle.copy_blocks``, ``oracle.write_kv``, then
``oracle.decode`` and ``oracle.prefill`` over the post-write cache.

After every step the whole cache must be bit-exact and every decode and
prefill output row within the attention tolerance."""
import math

import numpy as np
import torch

import oracle
from gpu_util import assert_attn_close, dev, dev_bf16, dev_u8, host_bits, to_float
from paged_kv_cache_408_b200 import inputs as I
from paged_kv_cache_408_b200 import ops
from paged_kv_cache_408_b200.executor import DeviceStep, StepExecutor


def initial_cache(tr, seed):
    rng = np.random.default_rng(seed)
    shape = (tr.sched.alloc.num_blocks, tr.Hkv, 16, tr.D)
    if tr.fp8:
        kh, ks = I.fp8_cache_from_normal(rng, shape)
        vh, vs = I.fp8_cache_from_normal(rng, shape)
        return kh, vh, ks, vs
    return I.normal_bf16(rng, shape), I.normal_bf16(rng, shape), None, None


def replay(tr, n_steps, seed=0, attend_prefill=False, cascade=True, expect_cascade=None, check_prefill_rows=None):
    """Run n_steps planned steps of trace ``tr`` on the GPU and in the oracle,
    comparing after each.  Returns per-step statistics."""
    plans = tr.plans(n_steps)
    kh, vh, ks, vs = initial_cache(tr, seed)
    if tr.fp8:
        kd, vd = dev_u8(kh), dev_u8(vh)
        ksd, vsd = dev(ks, np.float32), dev(vs, np.float32)
    else:
        kd, vd = dev_bf16(kh), dev_bf16(vh)
        ksd = vsd = None
    scale = 1.0 / math.sqrt(tr.D)
    ex = StepExecutor(kd, vd, tr.Hq, scale, ksd, vsd, attend_prefill=attend_prefill, cascade=cascade)
    ex.reserve(plans)
    rng = np.random.default_rng(seed + 1)
    stats = []
    for plan in plans:
        ds = DeviceStep(plan, torch, kd.device, cascade=cascade)
        if expect_cascade is not None:
            assert bool(ds.pb) == expect_cascade, (plan.step, ds.pb)
        T, B, NP = len(plan.slots), plan.num_decode, plan.num_prefill_tokens
        nk = I.normal_bf16(rng, (max(T, 1), tr.Hkv, tr.D))
        nv = I.normal_bf16(rng, (max(T, 1), tr.Hkv, tr.D))
        q = I.normal_bf16(rng, (max(B, 1), tr.Hq, tr.D))
        pq = I.normal_bf16(rng, (max(NP, 1), tr.Hq, tr.D))
        qd, pqd = dev_bf16(q), dev_bf16(pq)
        out = torch.full_like(qd, float("nan"))
        pout = torch.full_like(pqd, float("nan"))
        ex.enqueue(ds, qd, out, dev_bf16(nk), dev_bf16(nv), pqd, pout)
        # the oracle applies the same plan to its copy of the cache
        if len(plan.copies):
            oracle.copy_blocks(kh, vh, plan.copies)
        if T:
            oracle.write_kv(nk[:T], nv[:T], plan.slots, kh, vh, ks, vs)
        torch.cuda.synchronize()
        assert ops.get_last_device_error() == 0, f"step {plan.step}: device status word set"
        assert np.array_equal(host_bits(kd), kh), f"step {plan.step}: K cache differs"
        assert np.array_equal(host_bits(vd), vh), f"step {plan.step}: V cache differs"
        st = {"step": plan.step, "decode": B, "prefill_tokens": NP, "copies": len(plan.copies), "cascade": ds.pb,
              "admitted": len(plan.admitted), "retired": len(plan.retired)}
        if B:
            ref = oracle.decode(q[:B], kh, vh, plan.decode_tables, plan.decode_lens, scale, ks, vs)
            st["decode_err"] = assert_attn_close(to_float(out[:B]), ref, f"step {plan.step} decode")
        if attend_prefill and NP:
            ref = oracle.prefill(pq[:NP], plan.prefill_cu, plan.prefill_prefix, plan.prefill_tables, kh, vh, scale,
                                 ks, vs)
            st["prefill_err"] = assert_attn_close(to_float(pout[:NP]), ref, f"step {plan.step} prefill")
        stats.append(st)
    return stats
