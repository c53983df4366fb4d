"""Pins of the fp64 CPU oracle against things other than itself.

Every check here ties the oracle to a fact the pages or mathematics fix:
hand-worked closed forms (tests/golden/hand_examples.json), special cases with
a closed-form answer (seq_len 1 -> v0, equal keys -> mean of V), invariances
(block permutation, garbage past the sequence end, partition size of the
log-sum-exp merge, chunk splitting), an independent library routine
(torch scaled_dot_product_attention in fp64 on a contiguous gather; torch's
float8_e4m3fn conversion) and exhaustive enumeration (all 256 E4M3 codes).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_408_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------- helpers
def bits(vals):
    return I.bf16_bits(np.asarray(vals, np.float32))


def one_seq_cache(k_rows, v_rows, num_blocks=4, perm_seed=None, Hkv=1):
    """Lay out a single sequence's K/V rows ([n, D] float, exactly
    representable in bf16) into a paged cache with one kv head."""
    k_rows = np.asarray(k_rows, np.float32)
    v_rows = np.asarray(v_rows, np.float32)
    n, D = k_rows.shape
    nb_need = I.blocks_for(n)
    order = np.arange(num_blocks) if perm_seed is None else np.random.default_rng(perm_seed).permutation(num_blocks)
    table = np.full((1, max(nb_need, 1)), -1, np.int32)
    table[0, :nb_need] = order[:nb_need]
    kc = np.zeros((num_blocks, Hkv, 16, D), np.uint16)
    vc = np.zeros_like(kc)
    for t in range(n):
        blk, off = table[0, t // 16], t % 16
        kc[blk, 0, off] = bits(k_rows[t])
        vc[blk, 0, off] = bits(v_rows[t])
    return kc, vc, table


def contiguous_sdpa(case_q, kc, vc, table, seq_len, Hq, k_scale=None, v_scale=None, causal_rows=None):
    """Gather one sequence's tokens into a contiguous [len, Hkv, D] cache (the
    padded per-request layout that paging replaces) with numpy indexing and
    run torch's fp64 scaled_dot_product_attention per head."""
    nb, Hkv, bs, D = kc.shape
    t = np.arange(seq_len)
    phys = table[t // 16]
    if kc.dtype == np.uint8:
        kf = torch.from_numpy(kc[phys, :, t % 16, :]).view(torch.float8_e4m3fn).double()
        vf = torch.from_numpy(vc[phys, :, t % 16, :]).view(torch.float8_e4m3fn).double()
        kf = kf * torch.from_numpy(k_scale).double().view(1, Hkv, 1)
        vf = vf * torch.from_numpy(v_scale).double().view(1, Hkv, 1)
    else:
        kf = torch.from_numpy(I.bf16_values(kc[phys, :, t % 16, :])).double()
        vf = torch.from_numpy(I.bf16_values(vc[phys, :, t % 16, :])).double()
    g = Hq // Hkv
    kf = kf.permute(1, 0, 2).repeat_interleave(g, 0)  # [Hq, len, D]
    vf = vf.permute(1, 0, 2).repeat_interleave(g, 0)
    qf = torch.from_numpy(I.bf16_values(case_q)).double()  # [rows, Hq, D]
    qf = qf.permute(1, 0, 2)  # [Hq, rows, D]
    mask = None
    if causal_rows is not None:  # row r may see keys 0..causal_rows[r]
        lim = torch.from_numpy(np.asarray(causal_rows))
        mask = torch.arange(seq_len).view(1, -1) <= lim.view(-1, 1)
    o = torch.nn.functional.scaled_dot_product_attention(qf, kf, vf, attn_mask=mask, scale=1.0 / math.sqrt(D))
    return o.permute(1, 0, 2).numpy()


# ----------------------------------------------------------- number formats
def test_bf16_widening_matches_torch():
    rng = np.random.default_rng(1)
    b = rng.integers(0, 1 << 16, 4000).astype(np.uint16)
    b = b[~np.isnan(I.bf16_values(b))]
    ref = I.bf16_values(b).astype(np.float64)
    got = np.array([oracle.bf16_to_double(x) for x in b])
    assert np.array_equal(got, ref)


def test_e4m3_decode_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    got = np.array([oracle.e4m3_to_double(c) for c in codes])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert nan.sum() == 2  # S.1111.111 only
    assert np.array_equal(got[~nan], ref[~nan])
    # spec landmarks: largest finite, smallest normal, smallest subnormal, one
    assert got[0x7E] == 448.0 and got[0x08] == 2.0 ** -6 and got[0x01] == 2.0 ** -9
    assert got[0x38] == 1.0 and got[0xB8] == -1.0 and math.copysign(1, got[0x80]) == -1


def test_e4m3_encode_roundtrip_every_code():
    for c in range(256):
        x = oracle.e4m3_to_double(c)
        if math.isnan(x):
            continue
        assert oracle.e4m3_from_float(x) == c, hex(c)


def test_e4m3_encode_ties_to_even_and_matches_torch_in_range():
    codes = np.arange(256, dtype=np.uint8)
    vals = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    pos = np.sort(vals[(~np.isnan(vals)) & (vals >= 0)])
    pos = np.unique(pos)
    mids = (pos[:-1] + pos[1:]) / 2  # exact ties (float32 holds them)
    rng = np.random.default_rng(7)
    rand = rng.uniform(-464, 464, 20000).astype(np.float32)
    xs = np.concatenate([mids, -mids, rand, np.float32([0.0, -0.0, 1e-30, -1e-30, 464.0, -464.0])]).astype(np.float32)
    ref = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_from_float(x) for x in xs], np.uint8)
    assert np.array_equal(got, ref)
    # ties go to the even mantissa: 1.0625 sits between 1.0 (0x38) and 1.125 (0x39)
    assert oracle.e4m3_from_float(1.0625) == 0x38
    assert oracle.e4m3_from_float(1.1875) == 0x3A  # between 1.125 and 1.25 -> 1.25 (even)


def test_e4m3_encode_saturates_and_keeps_nan():
    for x in (448.0, 449.0, 465.0, 480.0, 1e6, 3.0e38, float("inf")):
        assert oracle.e4m3_from_float(x) == 0x7E
        assert oracle.e4m3_from_float(-x) == 0xFE
    assert oracle.e4m3_from_float(float("nan")) & 0x7F == 0x7F


# ------------------------------------------------------------------ decode
@pytest.mark.parametrize("idx", [0, 1, 2])
def test_decode_hand_examples(idx):
    case = json.load(open(os.path.join(GOLDEN, "hand_examples.json")))["cases"][idx]
    D = case["head_dim"]
    if isinstance(case["k"], str):
        k = np.zeros((17, D))
        k[16] = [8, 0]
        v = np.array([[t, 1] for t in range(17)], float)
    else:
        k, v = np.array(case["k"]), np.array(case["v"])
    kc, vc, table = one_seq_cache(k, v, num_blocks=3, perm_seed=5)
    q = bits(np.array(case["q"]).reshape(1, 1, D))
    out = oracle.decode(q, kc, vc, table, np.array([len(k)], np.int32), case["scale"])
    np.testing.assert_allclose(out[0, 0], case["out"], rtol=0, atol=1e-12)


def test_decode_seq_len_one_returns_v0_exactly():
    c = I.make_decode_case(3, [1, 1, 1], 8, 2, 64, num_blocks=8)
    out = oracle.decode(c.q, c.k_cache, c.v_cache, c.block_tables, c.seq_lens, c.scale)
    for b in range(3):
        blk = c.block_tables[b, 0]
        for h in range(8):
            v0 = I.bf16_values(c.v_cache[blk, h // 4, 0]).astype(np.float64)
            assert np.array_equal(out[b, h], v0)


def test_decode_gqa_maps_consecutive_query_heads_to_one_kv_head():
    # Hq = 6, Hkv = 3: heads (0,1) -> kv 0, (2,3) -> kv 1, (4,5) -> kv 2
    D = 8
    kc = np.zeros((2, 3, 16, D), np.uint16)
    vc = np.zeros_like(kc)
    for kvh in range(3):
        vc[1, kvh, 0] = bits(np.full(D, kvh + 1.0))
    table = np.array([[1]], np.int32)
    q = bits(np.ones((1, 6, D)))
    out = oracle.decode(q, kc, vc, table, np.array([1], np.int32), 0.5)
    assert np.array_equal(out[0, :, 0], [1, 1, 2, 2, 3, 3])


@pytest.mark.parametrize("scale_zero", [False, True])
def test_decode_equal_scores_give_mean_of_v(scale_zero):
    rng = np.random.default_rng(11)
    n, D = 37, 16
    k = np.tile(I.bf16_values(bits(rng.standard_normal(D))), (n, 1))
    if scale_zero:
        k = I.bf16_values(bits(rng.standard_normal((n, D))))
    v = I.bf16_values(bits(rng.standard_normal((n, D))))
    kc, vc, table = one_seq_cache(k, v, num_blocks=5, perm_seed=2)
    q = bits(rng.standard_normal((1, 1, D)))
    out = oracle.decode(q, kc, vc, table, np.array([n], np.int32), 0.0 if scale_zero else 0.3)
    np.testing.assert_allclose(out[0, 0], v.astype(np.float64).mean(0), rtol=0, atol=1e-12)


def test_decode_zero_length_gives_zeros():
    c = I.make_decode_case(4, [0, 5], 4, 4, 64, num_blocks=4)
    out = oracle.decode(c.q, c.k_cache, c.v_cache, c.block_tables, c.seq_lens, c.scale)
    assert not out[0].any() and out[1].any()


def test_decode_invariant_under_block_permutation():
    c = I.make_decode_case(5, [3, 16, 17, 40, 64], 8, 4, 64, num_blocks=24)
    ref = oracle.decode(c.q, c.k_cache, c.v_cache, c.block_tables, c.seq_lens, c.scale)
    p = np.random.default_rng(9).permutation(c.num_blocks)  # new position of block i
    kc2 = np.empty_like(c.k_cache)
    vc2 = np.empty_like(c.v_cache)
    kc2[p] = c.k_cache
    vc2[p] = c.v_cache
    bt2 = np.where(c.block_tables >= 0, p[np.maximum(c.block_tables, 0)], -1).astype(np.int32)
    out = oracle.decode(c.q, kc2, vc2, bt2, c.seq_lens, c.scale)
    assert np.array_equal(out, ref)


def test_decode_ignores_everything_past_the_sequence_end():
    c = I.make_decode_case(6, [5, 21, 33], 4, 2, 64, num_blocks=12)
    ref = oracle.decode(c.q, c.k_cache, c.v_cache, c.block_tables, c.seq_lens, c.scale)
    kc, vc = c.k_cache.copy(), c.v_cache.copy()
    used = set()
    for b, n in enumerate(c.seq_lens):
        for t in range(n):
            used.add((int(c.block_tables[b, t // 16]), t % 16))
    huge = bits(np.float32(3.0e38))
    for blk in range(c.num_blocks):
        for s in range(16):
            if (blk, s) not in used:
                kc[blk, :, s] = huge
                vc[blk, :, s] = huge
    out = oracle.decode(c.q, kc, vc, c.block_tables, c.seq_lens, c.scale)
    assert np.array_equal(out, ref)


@pytest.mark.parametrize("fp8", [False, True])
def test_decode_matches_torch_sdpa_on_contiguous_gather(fp8):
    c = I.make_decode_case(12, [1, 7, 16, 33, 100, 257], 8, 2, 64, fp8=fp8)
    out = oracle.decode(c.q, c.k_cache, c.v_cache, c.block_tables, c.seq_lens, c.scale, c.k_scale, c.v_scale)
    for b, n in enumerate(c.seq_lens):
        ref = contiguous_sdpa(c.q[b:b + 1], c.k_cache, c.v_cache, c.block_tables[b], int(n), c.Hq,
                              c.k_scale, c.v_scale)
        np.testing.assert_allclose(out[b], ref[0], rtol=0, atol=1e-12)


@pytest.mark.parametrize("P", [16, 48, 64, 512, 4096])
def test_split_merge_equals_single_pass(P):
    c = I.make_decode_case(13, [1, 15, 16, 17, 511, 512, 513, 1500], 8, 4, 64)
    ref = oracle.decode(c.q, c.k_cache, c.v_cache, c.block_tables, c.seq_lens, c.scale)
    out = oracle.decode(c.q, c.k_cache, c.v_cache, c.block_tables, c.seq_lens, c.scale, partition_tokens=P)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_decode_rejects_block_ids_outside_the_pool():
    c = I.make_decode_case(14, [20], 4, 4, 64, num_blocks=4)
    bt = c.block_tables.copy()
    bt[0, 1] = 99
    with pytest.raises(oracle.OracleError):
        oracle.decode(c.q, c.k_cache, c.v_cache, bt, c.seq_lens, c.scale)


# ----------------------------------------------------------------- prefill
def _prefill_case(seed=21, chunks=(1, 5, 16, 40), prefixes=(0, 3, 32, 17), Hq=8, Hkv=2, D=64):
    pc = I.make_prefill_case(seed, list(chunks), list(prefixes), Hq, Hkv, D)
    oracle.write_kv(pc.new_k, pc.new_v, pc.slot_mapping, pc.k_cache, pc.v_cache)
    return pc


def test_prefill_matches_causal_sdpa():
    pc = _prefill_case()
    out = oracle.prefill(pc.q, pc.cu_q, pc.prefix_lens, pc.block_tables, pc.k_cache, pc.v_cache, pc.scale)
    for c in range(len(pc.prefix_lens)):
        a, b = pc.cu_q[c], pc.cu_q[c + 1]
        P, C = int(pc.prefix_lens[c]), int(b - a)
        ref = contiguous_sdpa(pc.q[a:b], pc.k_cache, pc.v_cache, pc.block_tables[c], P + C, pc.Hq,
                              causal_rows=P + np.arange(C))
        np.testing.assert_allclose(out[a:b], ref, rtol=0, atol=1e-12)


def test_prefill_last_query_equals_decode_of_full_length():
    pc = _prefill_case(seed=22)
    out = oracle.prefill(pc.q, pc.cu_q, pc.prefix_lens, pc.block_tables, pc.k_cache, pc.v_cache, pc.scale)
    last = pc.cu_q[1:] - 1
    lens = (pc.prefix_lens + pc.chunk_lens).astype(np.int32)
    dec = oracle.decode(pc.q[last], pc.k_cache, pc.v_cache, pc.block_tables, lens, pc.scale)
    assert np.array_equal(out[last], dec)


def test_prefill_chunk_split_in_two_gives_same_rows():
    pc = _prefill_case(seed=23, chunks=(40,), prefixes=(9,))
    out = oracle.prefill(pc.q, pc.cu_q, pc.prefix_lens, pc.block_tables, pc.k_cache, pc.v_cache, pc.scale)
    cu2 = np.array([0, 13, 40], np.int32)
    pl2 = np.array([9, 9 + 13], np.int32)
    bt2 = np.repeat(pc.block_tables, 2, axis=0)
    out2 = oracle.prefill(pc.q, cu2, pl2, bt2, pc.k_cache, pc.v_cache, pc.scale)
    assert np.array_equal(out, out2)


def test_prefill_first_token_without_prefix_returns_its_own_v():
    pc = _prefill_case(seed=24, chunks=(1,), prefixes=(0,), Hq=4, Hkv=4)
    out = oracle.prefill(pc.q, pc.cu_q, pc.prefix_lens, pc.block_tables, pc.k_cache, pc.v_cache, pc.scale)
    assert np.array_equal(out[0], I.bf16_values(pc.new_v[0]).astype(np.float64))


# ------------------------------------------------------------- write, copy
def test_write_kv_bf16_places_bits_at_slots_and_touches_nothing_else():
    c = I.tiny_decode(0)
    kc, vc = c.k_cache.copy(), c.v_cache.copy()
    sm = c.slot_mapping.copy()
    sm[2] = -1  # padding slot is skipped
    oracle.write_kv(c.new_k, c.new_v, sm, kc, vc)
    expect_k, expect_v = c.k_cache.copy(), c.v_cache.copy()
    for t, s in enumerate(sm):
        if s >= 0:
            expect_k[s // 16, :, s % 16] = c.new_k[t]
            expect_v[s // 16, :, s % 16] = c.new_v[t]
    assert np.array_equal(kc, expect_k) and np.array_equal(vc, expect_v)


def test_write_kv_fp8_codes_match_torch_conversion():
    rng = np.random.default_rng(31)
    nb, Hkv, D, T = 6, 4, 32, 20
    kc = np.zeros((nb, Hkv, 16, D), np.uint8)
    vc = np.zeros_like(kc)
    k = I.bf16_bits(rng.standard_normal((T, Hkv, D), dtype=np.float32) * 3)
    v = I.bf16_bits(rng.standard_normal((T, Hkv, D), dtype=np.float32) * 3)
    ks = rng.uniform(0.005, 0.05, Hkv).astype(np.float32)
    vs = rng.uniform(0.005, 0.05, Hkv).astype(np.float32)
    slots = rng.permutation(nb * 16)[:T].astype(np.int64)
    oracle.write_kv(k, v, slots, kc, vc, ks, vs)
    # fp32 multiply by the fp32 reciprocal, then nearest-even E4M3
    kx = (I.bf16_values(k) * (np.float32(1) / ks).reshape(1, -1, 1)).astype(np.float32)
    vx = (I.bf16_values(v) * (np.float32(1) / vs).reshape(1, -1, 1)).astype(np.float32)
    in_range = (np.abs(kx) <= 464).all() and (np.abs(vx) <= 464).all()
    kref = torch.from_numpy(kx).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    vref = torch.from_numpy(vx).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    sat_k = np.abs(kx) > 464
    kref[sat_k] = np.where(kx[sat_k] > 0, 0x7E, 0xFE)
    sat_v = np.abs(vx) > 464
    vref[sat_v] = np.where(vx[sat_v] > 0, 0x7E, 0xFE)
    assert (sat_k.any() or sat_v.any()) or in_range
    for t, s in enumerate(slots):
        assert np.array_equal(kc[s // 16, :, s % 16], kref[t])
        assert np.array_equal(vc[s // 16, :, s % 16], vref[t])


def test_copy_blocks_copies_whole_blocks_in_order():
    rng = np.random.default_rng(41)
    kc = rng.integers(0, 65535, (10, 3, 16, 8)).astype(np.uint16)
    vc = rng.integers(0, 65535, (10, 3, 16, 8)).astype(np.uint16)
    k0, v0 = kc.copy(), vc.copy()
    pairs = np.array([[1, 7], [4, 2], [9, 0]], np.int32)
    oracle.copy_blocks(kc, vc, pairs)
    ek, ev = k0.copy(), v0.copy()
    for s, d in pairs:
        ek[d] = k0[s]
        ev[d] = v0[s]
    assert np.array_equal(kc, ek) and np.array_equal(vc, ev)
