"""Host-side logic of bench.py, on the CPU: which decode path a step takes,
how the roofline of a cascade call is assembled, the binding roof of the
decode kernel, and the packed per-step metadata of the end-to-end run."""
import types

import numpy as np
import pytest
import torch

import bench
from paged_kv_cache_408_b200 import runtime as R
from paged_kv_cache_408_b200 import traces


def plan_with(tables, lens):
    t = np.asarray(tables, np.int32)
    return R.StepPlan(0, np.zeros((0, 2), np.int32), np.zeros(0, np.int64), np.arange(len(t)), t,
                      np.asarray(lens, np.int32), np.zeros(0, np.int64), np.zeros(1, np.int32),
                      np.zeros(0, np.int32), np.zeros((0, t.shape[1]), np.int32))


def test_cascade_is_taken_for_a_large_shared_prefix_only():
    args = types.SimpleNamespace(no_cascade=False)
    shared = np.tile(np.arange(20), (8, 1))
    assert bench.cascade_blocks(plan_with(shared, [320] * 8), args) == 20
    assert bench.cascade_blocks(plan_with(shared, [255] * 8), args) == 0        # < 16 blocks covered by every row
    assert bench.cascade_blocks(plan_with(shared[:7], [320] * 7), args) == 0    # fewer than 8 rows
    diverge = shared.copy()
    diverge[3, 10] = 99
    assert bench.cascade_blocks(plan_with(diverge, [320] * 8), args) == 0       # only 10 shared blocks
    assert bench.cascade_blocks(plan_with(shared, [320] * 8), types.SimpleNamespace(no_cascade=True)) == 0


def test_every_step_of_the_shared_prefix_trace_takes_the_cascade():
    args = types.SimpleNamespace(no_cascade=False)
    for plan in traces.prefix_share_fp8(0).plans(4):
        assert bench.cascade_blocks(plan, args) >= 128


def test_decode_math_location():
    assert not bench.decode_math_on_cuda_cores(64, 8, True)     # fp8 GQA 8: tensor cores
    assert bench.decode_math_on_cuda_cores(64, 8, False)
    assert bench.decode_math_on_cuda_cores(32, 8, True)


def test_cascade_roofline_reports_the_longer_stage_with_consistent_fractions():
    c = {"call_ms": 0.1, "suffix_ms": 0.06, "prefix_flops": 17.2e9, "suffix_flops": 2e9, "suffix_bytes": 138e6,
         "unique_bytes": 142e6, "prefix_blocks": [128]}
    r = bench.cascade_roofline(c, 6541.0, "measured", 74.4, 1965.0, "none", cuda_core_math=False)
    assert r["kernel"].startswith("decode_kernel") and r["bound"] == "hbm"
    assert r["achieved"] == pytest.approx(138e6 / 0.06e-3 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"])
    pre = r["stages"]["prefix"]
    assert pre["bound"] == "tensor" and pre["ms_per_launch"] == pytest.approx(0.04)
    assert pre["frac"] == pytest.approx(pre["achieved"] / pre["peak"])
    call = r["stages"]["call"]
    assert call["roof_ms"] == pytest.approx((17.2e9 / (pre["peak"] * 1e12) + 138e6 / 6541e9) * 1e3)
    c["suffix_ms"] = 0.03  # now the prefix stage is the longer one
    assert bench.cascade_roofline(c, 6541.0, "measured", 74.4, 1965.0, "none", False)["bound"] == "tensor"


def test_packed_step_metadata_round_trips(monkeypatch):
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self: self)  # no CUDA here
    for plan in traces.batch64_2k(0).plans(3) + traces.mixed(0).plans(2):
        plain = bench.DeviceStep(plan, torch, "cpu")
        moved = bench.DeviceStep(plan, torch, "cpu", pin=True).to("cpu")
        for k, _ in bench.DeviceStep.FIELDS:
            a, b = getattr(plain, k), getattr(moved, k)
            assert a.dtype == b.dtype and a.shape == b.shape and torch.equal(a, b), k


def test_roof_time_reproduces_the_pages_batching_model():
    """The two-roof bound bench.py uses, checked against the batching table of
    the third page (pass time and tokens/s for B sequences sharing one read of
    the weights; tests/golden/batching_model.json cites it).  Summing the two
    roofs instead of taking the slower, or swapping bytes and FLOPs, breaks
    the small-batch rows or the plateau."""
    import json
    import os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "batching_model.json")))
    m = g["model"]
    for row in g["rows"]:
        B = row["batch"]
        t = bench.roof_time(m["weight_bytes"], m["hbm_bytes_per_s"], B * m["flops_per_token"],
                            m["usable_fraction"] * m["peak_flops_per_s"])
        assert abs(t * 1e3 - row["pass_ms"]) <= 0.06, (B, t)   # printed to 0.1 ms
        assert B / t == pytest.approx(row["tokens_per_s"], rel=0.01)
    # the crossover: memory-bound up to 26 sequences, compute-bound beyond
    w = m["weight_bytes"] / m["hbm_bytes_per_s"]
    per = m["flops_per_token"] / (m["usable_fraction"] * m["peak_flops_per_s"])
    assert int(w // per) == 25 and w / per < 26
