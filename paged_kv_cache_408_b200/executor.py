"""Device execution of scheduler steps.

A ``StepPlan`` from :mod:`paged_kv_cache_408_b200.runtime` holds one step's
metadata as numpy arrays.  ``DeviceStep`` uploads it (one copy of a packed
pinned buffer, or one copy per field); ``StepExecutor.enqueue`` runs the
step's kernels on the current stream, in the order the step needs them:

1. ``pa_copy_blocks`` -- the copy-on-write pairs the allocator emitted ("Continuous
   batching and PagedAttention", PagedAttention: KV cache memory: a shared
   block is copied before a sharer's first divergent write), so it runs
   before the writes;
2. ``pa_write_kv`` -- every new token's K/V: one per decoding sequence, then
   the prefill chunks' tokens ("Production Serving: Continuous Batching and
   PagedAttention", Step 4);
3. ``pa_decode`` (or ``pa_decode_cascade`` when the decode rows share leading
   blocks) -- one query per decoding sequence over its cache, its own new
   token included (write first, then attend);
4. ``pa_prefill_chunk`` -- the prefill chunks, causal over their prefixes
   ("Continuous batching and PagedAttention", How the scheduler works: the
   budget left after decode is filled with prefill chunks).

Every call goes through the C ABI (:mod:`ops`); the kernels of one step are
programmatic dependents of one another, so the host enqueues the whole step
without a synchronisation.
"""
from __future__ import annotations

import math

import numpy as np

from . import ops
from .runtime import BLOCK_SIZE, StepPlan

# cascade decode pays off once enough rows share enough leading blocks
CASCADE_MIN_ROWS = 8
CASCADE_MIN_TOKENS = 256


def cascade_blocks(plan: StepPlan, enabled: bool = True) -> int:
    """Shared prefix blocks a step's decode attends through cascade decode:
    the leading table entries that every decode row shares (the same
    physical blocks, e.g. sequences forked from one prompt) and fills, for a
    batch and prefix large enough to pay for the extra launches; else 0
    (plain decode)."""
    if not enabled:
        return 0
    pb = plan.shared_decode_blocks
    return pb if plan.num_decode >= CASCADE_MIN_ROWS and pb * BLOCK_SIZE >= CASCADE_MIN_TOKENS else 0


class DeviceStep:
    """One planned step's metadata as device tensors, or (pin=True) packed
    into one pinned host buffer that ``to()`` moves with a single copy."""
    FIELDS = (("slots", np.int64), ("copies", np.int32), ("tables", np.int32), ("lens", np.int32),
              ("p_cu", np.int32), ("p_prefix", np.int32), ("p_tables", np.int32))

    def __init__(self, plan: StepPlan, torch, device, pin=False, cascade=True):
        arrs = {"copies": plan.copies, "slots": plan.slots, "tables": plan.decode_tables,
                "lens": plan.decode_lens, "p_cu": plan.prefill_cu, "p_prefix": plan.prefill_prefix,
                "p_tables": plan.prefill_tables}
        self.plan = plan
        self.packed = None
        if pin:
            # one byte buffer, every field at a 16-byte aligned offset
            self.layout, off = [], 0
            for k, dt in self.FIELDS:
                a = np.ascontiguousarray(arrs[k], dt)
                self.layout.append((k, dt, off, a.shape))
                off += (a.nbytes + 15) // 16 * 16
            host = np.zeros(max(off, 16), np.uint8)
            for k, dt, o, shape in self.layout:
                a = np.ascontiguousarray(arrs[k], dt)
                host[o:o + a.nbytes] = a.view(np.uint8).reshape(-1)
            self.packed = torch.from_numpy(host).pin_memory()
        else:
            for k, dt in self.FIELDS:
                setattr(self, k, torch.from_numpy(np.ascontiguousarray(arrs[k], dt)).to(device))
        self.T = len(plan.slots)
        self.B = plan.num_decode
        self.nchunks = len(plan.prefill_ids)
        self.n_prefill = plan.num_prefill_tokens
        self.max_chunk = plan.max_chunk
        self.pb = cascade_blocks(plan, cascade)  # 0: plain decode

    def to(self, device, non_blocking=True, out=None):
        """Device copy of a packed step: one host-to-device copy (into `out`,
        a uint8 device tensor of at least ``nbytes()``, if given), then views."""
        import torch
        d = object.__new__(DeviceStep)
        d.__dict__.update(self.__dict__)
        if out is None:
            buf = self.packed.to(device, non_blocking=non_blocking)
        else:
            buf = out[:self.packed.numel()]
            buf.copy_(self.packed, non_blocking=non_blocking)
        tdt = {np.int32: torch.int32, np.int64: torch.int64}
        for k, dt, o, shape in self.layout:
            n = int(np.prod(shape)) * np.dtype(dt).itemsize
            setattr(d, k, buf[o:o + n].view(tdt[dt]).view(shape))
        d.packed = None
        return d

    def nbytes(self):
        if self.packed is not None:
            return self.packed.numel()
        return sum(getattr(self, k).numel() * getattr(self, k).element_size() for k, _ in self.FIELDS)


class StepExecutor:
    """Runs planned steps on one paged cache through the C ABI.

    k_cache, v_cache  device tensors [num_blocks, Hkv, 16, D] (bf16, or uint8
                      E4M3 with k_scale / v_scale fp32 [Hkv]);
    Hq                query heads; scale the softmax scale (default 1/sqrt(D));
    attend_prefill    run the prefill chunks' attention (False: their K/V are
                      written, e.g. to materialise a prompt's cache, but not
                      attended);
    cascade           use cascade decode where the decode rows share blocks;
    partition_tokens  pa_decode's split (0: balanced).
    ``reserve(plans)`` sizes the one decode workspace for every step first.
    """

    def __init__(self, k_cache, v_cache, Hq, scale=None, k_scale=None, v_scale=None, attend_prefill=True,
                 cascade=True, partition_tokens=0):
        self.k_cache, self.v_cache = k_cache, v_cache
        self.k_scale, self.v_scale = k_scale, v_scale
        self.Hq = int(Hq)
        self.D = int(k_cache.shape[3])
        self.scale = float(scale) if scale is not None else 1.0 / math.sqrt(self.D)
        self.attend_prefill = attend_prefill
        self.cascade = cascade
        self.partition = int(partition_tokens)
        self.ws = None

    def workspace_bytes(self, plan: StepPlan) -> int:
        """Workspace a step needs: for plain decode of its tables, and for the
        cascade where it takes one (the larger of the two, so that the same
        step can also run through plain decode)."""
        maxb = plan.decode_tables.shape[1]
        B = max(plan.num_decode, 1)
        n = ops.decode_workspace_size(B, self.Hq, self.D, maxb, self.partition)
        pb = cascade_blocks(plan, self.cascade)
        if pb:
            n = max(n, ops.cascade_workspace_size(B, self.Hq, maxb, pb, self.k_cache))
        return n

    def reserve(self, plans):
        import torch
        n = max([self.workspace_bytes(p) for p in plans] + [256])
        if self.ws is None or self.ws.numel() < n:
            self.ws = torch.zeros(n, dtype=torch.uint8, device=self.k_cache.device)

    def copy_and_write(self, ds: DeviceStep, new_k, new_v) -> int:
        """The step's copy-on-write copies, then its new K/V."""
        n = 0
        if ds.copies.shape[0]:
            ops.copy_blocks(self.k_cache, self.v_cache, ds.copies)
            n += 1
        if ds.T:
            ops.write_kv(new_k[:ds.T], new_v[:ds.T], ds.slots, self.k_cache, self.v_cache, self.k_scale, self.v_scale)
            n += 1
        return n

    def decode(self, ds: DeviceStep, q, out) -> int:
        """One query per decoding sequence (cascade where the rows share blocks)."""
        if not ds.B:
            return 0
        kc, vc, ks, vs = self.k_cache, self.v_cache, self.k_scale, self.v_scale
        if ds.pb:
            ops.decode_cascade(out[:ds.B], q[:ds.B], kc, vc, ds.tables, ds.lens, self.scale, ds.pb, self.ws, ks, vs)
            return 4 if ks is not None else 3  # (fp8 widening) + prefix attention + suffix decode + merge
        ops.decode(out[:ds.B], q[:ds.B], kc, vc, ds.tables, ds.lens, self.scale, ks, vs, self.ws, self.partition)
        return 2  # decode + merge

    def prefill(self, ds: DeviceStep, pq, pout) -> int:
        """The step's prefill chunks, causal over their prefixes."""
        if not (self.attend_prefill and ds.nchunks and ds.n_prefill):
            return 0
        nt = ds.n_prefill
        ops.prefill_chunk(pout[:nt], pq[:nt], ds.p_cu, ds.p_prefix, ds.p_tables, self.k_cache, self.v_cache,
                          self.scale, ds.max_chunk, self.k_scale, self.v_scale)
        return 1

    def enqueue(self, ds: DeviceStep, q, out, new_k, new_v, pq=None, pout=None) -> int:
        """Enqueue one whole step; returns the number of kernels launched.

        q, out        bf16 [>= ds.B, Hq, D]: the decode queries and outputs;
        new_k, new_v  bf16 [>= ds.T, Hkv, D]: the step's new K/V, decode
                      tokens first, then the prefill chunks' tokens;
        pq, pout      bf16 [>= prefill tokens, Hq, D]: the chunks' queries and
                      outputs (needed when the step has chunks to attend)."""
        return self.copy_and_write(ds, new_k, new_v) + self.decode(ds, q, out) + self.prefill(ds, pq, pout)
