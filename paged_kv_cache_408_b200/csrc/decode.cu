// decode.cu -- paged decode attention for sm_100a, with split-K pieces and
// a log-sum-exp merge kernel launched as a programmatic dependent.
//
// What is computed ("Production Serving: Continuous Batching and
// PagedAttention", The Build, Step 6 "Implement attention over paged
// storage", read per query head):
//     out[b][h] = sum_{t < len_b} softmax_t(scale * q[b][h] . k_t) v_t
// where token t of sequence b lives in slot t%16 of physical block
// block_tables[b][t/16], kv head floor(h*Hkv/Hq).
//
// How (B200 design):
//  * The unit of work is a warp.  Every warp streams 16-token blocks of ONE
//    (sequence, kv head) at a time and computes the whole GQA group of that
//    kv head, so each K/V byte is read from HBM exactly once per step.
//    Warps are independent: no CTA barrier inside the main loop, so one
//    warp's per-item latencies (q load, epilogue, merge) are hidden by the
//    other warps of the SM.
//  * Work split (host selects with partition_tokens):
//      balanced -- the (sequence, kv head) segments of the batch form one
//        line in cost units: one unit per 16-token block plus kSegmentCost
//        units charged at the head of every segment for its per-item work
//        (q load, epilogue, output write); warp g takes the contiguous share
//        [g*S, (g+1)*S) with S = ceil(total / warps), so warps get the same
//        time's work whatever the length mix;
//      fixed -- every (sequence, kv head) is cut into partitions of P tokens,
//        dealt round-robin to warps (full partitions first); split points
//        depend only on token positions, so results are batch-invariant.
//    Every CTA rebuilds the split from seq_lens with a block-wide scan in
//    shared memory: no host sync, no empty CTAs for short sequences.
//  * One CTA of 12 warps per SM.  With several CTAs per SM the warp
//    schedulers favour the CTA that arrived first, so equal shares finished
//    up to 15% apart; warps of one CTA are served evenly.  (GQA groups of 8
//    keep two CTAs of 4 warps: their arithmetic per byte is twice as high
//    and there the uneven service measured faster.)
//  * Each warp runs its own NSTAGE-deep shared-memory ring filled by 1-D
//    bulk async copies (the TMA engine; K and V of one block of one kv head
//    are 4 KB contiguous each) that complete on mbarriers.  The rings of an
//    SM's warps fill kRingBytes of shared memory.  The producer runs ahead
//    across item boundaries and keeps block-table entries in registers (a
//    sliding window, plus the next item's first entries).
//  * Math on CUDA cores for bf16 caches and for groups of up to 4 heads
//    (4-8 query rows are far below a tcgen05 tile, and the path is
//    HBM-bound), on the tensor cores with warp-level MMAs for an fp8 cache
//    with groups of 8 (see mma_items).  CUDA-core path: lanes form token
//    groups of LPT lanes; a lane owns
//    DPL head dims (16-byte shared-memory reads, bank-conflict-free), keeps
//    q for them in fp32 registers pre-scaled by scale*log2(e), and
//    accumulates with packed fp32x2 FMAs.  Partial dot products are
//    completed by a select-free shuffle reduce-scatter, exponentiated by the
//    owning lane and all-gathered for P.V.
//  * Online softmax with a lazily moved running max (it only moves when a
//    score exceeds it by more than 8 in log2 units); the final division uses
//    the sum taken against the same max, so the result is the exact softmax.
//  * A (sequence, kv head) covered by one piece is written as bf16 straight
//    from registers.  Otherwise each piece writes its fp32 output and its
//    log2-sum-exp to the workspace with plain stores: no fence and no
//    atomic on the streaming warps (a gpu-scope fence waits for the store
//    acknowledgements, microseconds while HBM is saturated).  A second
//    kernel, launched as a programmatic dependent so that its launch
//    overlaps the decode kernel, merges the pieces by log-sum-exp once the
//    decode grid has completed.
#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace pa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: p <= 256 before a rescale
constexpr int kSegmentCost = 2;            // balanced split: cost units charged per segment
constexpr size_t kRingBytes = 192 * 1024;  // K/V staging rings of all warps of an SM
constexpr unsigned kFull = 0xffffffffu;

template <int D_, int G_, bool FP8_>
struct Cfg {
    static constexpr int D = D_, G = G_;
    static constexpr bool FP8 = FP8_;
    static constexpr int EB = FP8 ? 1 : 2;           // bytes per element
    static constexpr int DPL = (G >= 4) ? 8 : 16;     // head dims owned by a lane
    static constexpr int LPT = D / DPL;               // lanes per token
    static constexpr int NGRP = 32 / LPT;             // token groups per warp
    static constexpr int TPG = 16 / NGRP;             // tokens per group per block
    static constexpr int TSUB = (TPG * G > 16) ? (16 / G > 0 ? 16 / G : 1) : TPG;  // tokens per sub-step
    static constexpr int NSUB = TPG / TSUB;
    static constexpr int NCH = DPL / 8;               // 8-element chunks per lane per row
    static constexpr int CHB = 8 * EB;                // bytes per chunk
    static constexpr int ROWB = D * EB;               // bytes per token row
    static constexpr int BLKB = 16 * ROWB;            // bytes of one block of one head (K or V)
    static constexpr int P2 = DPL / 2;                // fp32 pairs per lane per head
    static constexpr int NS = TSUB * G;               // partial scores per lane per sub-step
    static constexpr bool RS = NS >= LPT;             // reduce-scatter (else all-reduce)
    static constexpr int VPL = RS ? NS / LPT : NS;    // scores a lane owns after the reduction
    // CTAS CTAs of NW warps per SM share the register file (G = 8 needs ~255
    // registers a thread, so 8 warps an SM; otherwise ~168, so 12) and a
    // kRingBytes shared-memory ring, split into NSTAGE stages per warp.
    // fp8 with GQA 8 runs its products on the tensor cores (mma_items)
    static constexpr bool MMA = FP8 && G == 8;
    static constexpr int CTAS = (G >= 8 && !MMA) ? 2 : 1;  // CTAs per SM
    static constexpr int NW = (G >= 8 && !MMA) ? 4 : 12;   // warps per CTA
    static constexpr int NT = NW * 32;
    static constexpr int NSTAGE = (int)(kRingBytes / ((size_t)CTAS * NW * 2 * BLKB));  // ring depth per warp
    static constexpr int MIN_CTAS = CTAS;
    static constexpr size_t STAGE_BYTES = (size_t)NW * NSTAGE * 2 * BLKB;
    static_assert(NSTAGE >= 2 && NSTAGE <= 32, "ring depth");
    static_assert(LPT >= 1 && LPT <= 32 && 32 % LPT == 0, "bad lane split");
    static_assert(TPG * NGRP == 16 && TSUB * NSUB == TPG, "bad token split");
    static_assert(!RS || NS % LPT == 0, "reduce-scatter needs NS divisible by LPT");
};

template <class C>
size_t smem_bytes(int B) {
    size_t s = C::STAGE_BYTES;
    s += (size_t)C::NW * C::NSTAGE * 8;   // mbarriers
    s += (size_t)C::NW * C::NSTAGE * 4;   // valid-token count per stage
    s += (size_t)2 * C::NW * 4;           // scan scratch
    s += (size_t)(3 * B + 2) * 4;         // lens and two exclusive scans
    return s;
}

// Largest b in [0, n) with arr[b] <= u, for non-decreasing arr with arr[0] = 0.
PA_DEVICE int upper_index(const int *arr, int n, int u) {
    int lo = 0, hi = n;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (arr[mid] <= u) lo = mid; else hi = mid;
    }
    return lo;
}

// ---- compile-time butterflies over the LPT lanes of a token group.
//
// Lane `sub` of a group stores partial score idx (= token*G + head within a
// sub-step) at register position idx ^ S, S = sub*VPL.  With that lane-
// dependent layout a reduce-scatter is select-free: at every level a lane
// keeps positions [0, N) and adds the partner's positions [N, 2N), and after
// the last level positions [0, VPL) hold the lane's own complete scores
// (idx = S + i).  The all-gather walks back the same way.  The layout costs
// nothing: the XOR on the head bits permutes which q head sits in which
// register slot (chosen once, at the q load), the XOR on the token bits
// permutes which shared-memory row a lane reads.
template <int MASK, int N, int NS>
PA_DEVICE void rs_level(float (&v)[NS]) {
    if constexpr (MASK >= 1) {
#pragma unroll
        for (int k = 0; k < N; ++k) v[k] += __shfl_xor_sync(kFull, v[k + N], MASK);
        rs_level<MASK / 2, N / 2, NS>(v);
    }
}

template <int MASK, int LPT, int N, int NS>
PA_DEVICE void ag_level(float (&v)[NS]) {
    if constexpr (MASK < LPT) {
#pragma unroll
        for (int k = 0; k < N; ++k) v[k + N] = __shfl_xor_sync(kFull, v[k], MASK);
        ag_level<MASK * 2, LPT, N * 2, NS>(v);
    }
}

// Butterfly all-reduce (sum) of NS values over lanes whose index differs in
// bits below LPT (used when every lane keeps every score).
template <int MASK, int NS>
PA_DEVICE void allreduce_level(float (&v)[NS]) {
    if constexpr (MASK >= 1) {
#pragma unroll
        for (int k = 0; k < NS; ++k) v[k] += __shfl_xor_sync(kFull, v[k], MASK);
        allreduce_level<MASK / 2, NS>(v);
    }
}

// All-reduce of per-head values kept in permuted head slots: slot h of lane
// sub is head h ^ (sub*VPL % G), so the partner across MASK keeps my head in
// slot h ^ (MASK*VPL % G).  MAX selects max, otherwise sum.
template <int MASK, int VPL, int G, bool MAX>
PA_DEVICE void perm_allreduce(float (&v)[G]) {
    if constexpr (MASK >= 1) {
        constexpr int X = (MASK * VPL) % G;
        float r[G];
#pragma unroll
        for (int h = 0; h < G; ++h) r[h] = __shfl_xor_sync(kFull, v[h ^ X], MASK);
#pragma unroll
        for (int h = 0; h < G; ++h) v[h] = MAX ? fmaxf(v[h], r[h]) : v[h] + r[h];
        perm_allreduce<MASK / 2, VPL, G, MAX>(v);
    }
}

// Merge the (m, l, acc) states of token groups: partners differ in the group
// bits (MASK = LPT, 2*LPT, ... 16).  Groups of opposite parity visit their
// two 16-byte chunks in swapped order, so at MASK == LPT the partner's
// register holding my chunk is at the other half (k ^ 4).
template <int MASK, int LPT, int G, int P2, bool SWAP>
PA_DEVICE void group_merge(float (&m)[G], float (&l)[G], float2 (&acc)[G][P2]) {
    if constexpr (MASK < 32) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float mo = __shfl_xor_sync(kFull, m[h], MASK);
            const float lo = __shfl_xor_sync(kFull, l[h], MASK);
            const float M = fmaxf(m[h], mo);
            const float am = (m[h] == -INFINITY) ? 0.f : ex2(m[h] - M);
            const float ao = (mo == -INFINITY) ? 0.f : ex2(mo - M);
            l[h] = l[h] * am + lo * ao;
            m[h] = M;
            float2 rx[P2];
#pragma unroll
            for (int k = 0; k < P2; ++k) {
                constexpr bool sw = SWAP && MASK == LPT;
                const int ks = sw ? (k ^ 4) : k;
                rx[k].x = __shfl_xor_sync(kFull, acc[h][ks].x, MASK);
                rx[k].y = __shfl_xor_sync(kFull, acc[h][ks].y, MASK);
            }
#pragma unroll
            for (int k = 0; k < P2; ++k)
                acc[h][k] = ffma2(acc[h][k], make_float2(am, am), make_float2(rx[k].x * ao, rx[k].y * ao));
        }
        group_merge<MASK * 2, LPT, G, P2, SWAP>(m, l, acc);
    }
}

// A unit of work: blocks [blk0, blk0 + nblk) of sequence b, kv head kvh.
// It is piece `piece` of the npieces pieces that cover that (sequence, kv
// head); a single piece writes the output, several pieces are merged.
struct Item {
    int b, kvh, piece, npieces, len, blk0, nblk;
};

// The work split, rebuilt by every CTA from seq_lens in shared memory.
struct Schedule {
    const int *len;   // [B]
    const int *pre0;  // balanced: segment offset [B+1]; fixed: full-partition prefix [B+1]
    const int *pre1;  // fixed: tail prefix [B+1]
    int B, Hkv, P;
    int total;        // balanced: blocks in the line; fixed: number of items
    int S;            // balanced: share per warp, in blocks
    int NF;           // fixed: number of full-partition entries (per kv head)

    PA_DEVICE Item fixed_item(int i) const {
        Item it;
        it.kvh = i % Hkv;
        int u = i / Hkv;
        if (u < NF) {
            it.b = upper_index(pre0, B, u);
            it.piece = u - pre0[it.b];
        } else {
            u -= NF;
            it.b = upper_index(pre1, B, u);
            it.piece = pre0[it.b + 1] - pre0[it.b];
        }
        it.len = len[it.b];
        it.npieces = (pre0[it.b + 1] - pre0[it.b]) + (pre1[it.b + 1] - pre1[it.b]);
        const int t0 = it.piece * P, t1 = min(t0 + P, it.len);
        it.blk0 = t0 >> 4;
        it.nblk = ((t1 + 15) >> 4) - it.blk0;
        return it;
    }

    // balanced: the piece of the segment holding line position pos, cut at
    // `end`.  A segment is kSegmentCost cost units, then one unit per block;
    // its pieces are the warp shares that hold its block units.  Returns the
    // line position after the piece (nblk <= 0: the share ends before the
    // segment's first block).
    PA_DEVICE int balanced_item(int pos, int end, Item &it) const {
        it.b = upper_index(pre0, B, pos);
        it.len = len[it.b];
        const int nb = (it.len + 15) >> 4, U = nb + kSegmentCost;
        const int u = pos - pre0[it.b];
        it.kvh = u / U;
        const int seg0 = pre0[it.b] + it.kvh * U, r0 = seg0 + kSegmentCost, seg1 = seg0 + U;
        const int p = max(pos, r0), stop = min(seg1, end);
        it.blk0 = p - r0;
        it.nblk = stop - p;
        it.piece = p / S - r0 / S;
        it.npieces = (seg1 - 1) / S - r0 / S + 1;
        return stop;
    }
};

// Walks the items of one warp (global warp index gw of GW) in order.
struct ItemIter {
    int cur, end, step;

    PA_DEVICE void start(const Schedule &sc, int gw, int GW) {
        if (sc.P == 0) {
            cur = min(sc.total, gw * sc.S);
            end = min(sc.total, cur + sc.S);
            step = 0;
        } else {
            cur = gw;
            end = sc.total;
            step = GW;
        }
    }
    PA_DEVICE bool next(const Schedule &sc, Item &it) {
        if (sc.P == 0) {
            while (cur < end) {
                cur = sc.balanced_item(cur, end, it);
                if (it.nblk > 0) return true;
            }
            return false;
        }
        if (cur >= end) return false;
        it = sc.fixed_item(cur);
        cur += step;
        return true;
    }
};

// Per-warp producer: lane 0 issues the two bulk copies (K and V block of one
// kv head) for the next block of the warp's stream.  The warp keeps a
// 64-entry window of the current item's block-table entries in registers
// (lane l holds entries base+l and base+32+l), slid 32 entries ahead of use,
// plus the first 64 entries of the next item, loaded while the current one
// streams.
template <class C>
struct Producer {
    ItemIter iter;
    Item cur, nxt;
    bool has_cur, has_nxt;
    int j, base;
    int t0, t1, nt0, nt1;
    uint32_t issued;

    PA_DEVICE int load32(const DecodeArgs &a, const Item &it, int lane, int off) {
        const int32_t *row = a.block_tables + (size_t)it.b * a.max_blocks + a.prefix_blocks + it.blk0;
        return (off + lane < it.nblk) ? row[off + lane] : -1;
    }

    PA_DEVICE void fetch_next(const Schedule &sc, const DecodeArgs &a, int lane) {
        has_nxt = iter.next(sc, nxt);
        if (has_nxt) {
            nt0 = load32(a, nxt, lane, 0);
            nt1 = load32(a, nxt, lane, 32);
        }
    }

    PA_DEVICE void advance(const Schedule &sc, const DecodeArgs &a, int lane) {
        cur = nxt;
        has_cur = has_nxt;
        t0 = nt0;
        t1 = nt1;
        j = 0;
        base = 0;
        fetch_next(sc, a, lane);
    }

    PA_DEVICE void init(const Schedule &sc, const DecodeArgs &a, int gw, int GW, int lane) {
        issued = 0;
        iter.start(sc, gw, GW);
        fetch_next(sc, a, lane);
        advance(sc, a, lane);
    }

    PA_DEVICE void produce(const Schedule &sc, const DecodeArgs &a, int lane, const uint8_t *kc, const uint8_t *vc,
                           uint8_t *stg, uint64_t *bars, int *valid_of) {
        while (has_cur && j >= cur.nblk) advance(sc, a, lane);
        if (!has_cur) return;
        if (j - base == 32) {  // slide the window: refill 32 entries ahead
            t0 = t1;
            t1 = load32(a, cur, lane, base + 64);
            base += 32;
        }
        int phys = __shfl_sync(kFull, t0, j - base);
        if (lane == 0) {
            const int blk = cur.blk0 + j;
            int valid = min(16, cur.len - blk * 16);
            if (phys < 0 || phys >= a.num_blocks) {
                flag_error(a.err, PA_DEVERR_BAD_BLOCK);
                phys = 0;
                valid = 0;
            }
            const int s = issued % C::NSTAGE;
            valid_of[s] = valid;
            mbar_arrive_expect_tx(&bars[s], 2 * C::BLKB);
            const size_t src = ((size_t)phys * sc.Hkv + cur.kvh) * C::BLKB;
            uint8_t *dst = stg + (size_t)s * 2 * C::BLKB;
            bulk_g2s(dst, kc + src, C::BLKB, &bars[s]);
            bulk_g2s(dst + C::BLKB, vc + src, C::BLKB, &bars[s]);
        }
        ++issued;
        ++j;
    }
};

// After a wait of this warp's ring ran past the launch deadline: record the
// timeout, stop streaming, and wait (with a short fresh budget) for the
// copies this warp has issued but not consumed, so that none lands in
// shared memory after the warp has exited.  Each of those stages has exactly
// one copy in flight (a stage is refilled only after it was consumed).
template <class C>
PA_DEVICE void give_up(const DecodeArgs &a, uint64_t *bars, uint32_t consumed, uint32_t issued, int lane) {
    if (lane == 0) flag_error(a.err, PA_DEVERR_TIMEOUT);
    const uint64_t dd = drain_deadline();
    for (uint32_t c = consumed; c < issued; ++c)
        if (!mbar_wait(&bars[c % C::NSTAGE], (c / C::NSTAGE) & 1, dd)) break;
    __syncwarp();
}

// Load this lane's chunks of one token row from shared memory and widen to fp32 pairs.
template <class C>
PA_DEVICE void load_row(const uint8_t *row, const int (&choff)[C::NCH], float2 (&f)[C::P2]) {
#pragma unroll
    for (int c = 0; c < C::NCH; ++c) {
        if constexpr (!C::FP8) {
            const uint4 u = *reinterpret_cast<const uint4 *>(row + choff[c] * C::CHB);
            f[4 * c + 0] = bf16x2_to_float2(u.x);
            f[4 * c + 1] = bf16x2_to_float2(u.y);
            f[4 * c + 2] = bf16x2_to_float2(u.z);
            f[4 * c + 3] = bf16x2_to_float2(u.w);
        } else {
            const uint2 u = *reinterpret_cast<const uint2 *>(row + choff[c] * C::CHB);
            f[4 * c + 0] = e4m3x2_to_float2((uint16_t)(u.x & 0xffff));
            f[4 * c + 1] = e4m3x2_to_float2((uint16_t)(u.x >> 16));
            f[4 * c + 2] = e4m3x2_to_float2((uint16_t)(u.y & 0xffff));
            f[4 * c + 3] = e4m3x2_to_float2((uint16_t)(u.y >> 16));
        }
    }
}

// Raw inputs of one item that the consumer loads ahead of time: its q rows
// (this lane's chunks, head slot h = head h ^ sh) and the fp8 scales.
template <class C>
struct QPrefetch {
    uint4 q[C::G][C::NCH];
    float ks, vs;

    PA_DEVICE void load(const DecodeArgs &a, const Item &it, const int (&choff)[C::NCH], int sh) {
        const __nv_bfloat16 *qrow =
            static_cast<const __nv_bfloat16 *>(a.q) + ((size_t)it.b * a.Hq + (size_t)it.kvh * C::G) * C::D;
#pragma unroll
        for (int h = 0; h < C::G; ++h)
#pragma unroll
            for (int c = 0; c < C::NCH; ++c)
                q[h][c] = *reinterpret_cast<const uint4 *>(qrow + (h ^ sh) * C::D + choff[c] * 8);
        ks = C::FP8 ? a.k_scale[it.kvh] : 1.0f;
        vs = C::FP8 ? a.v_scale[it.kvh] : 1.0f;
    }
};

// ---- tensor-core decode (fp8 cache, GQA groups of 8) ----------------------
//
// With an fp8 cache and 8 q heads per kv head, q.k and p.v on CUDA cores
// cost 16 FLOP per cached byte, more than the fp32 pipes deliver at HBM
// speed.  This path moves both products onto the tensor cores with the
// warp-level mma.sync m16n8k16 (f16 operands, fp32 accumulators), one block
// (16 tokens) at a time:
//     S^T [16 tokens x 8 heads]  = K [16 x D] . q^T [D x 8]      (D/16 MMAs)
//     O^T [D x 8 heads]         += V^T [D x 16] . P^T [16 x 8]   (D/16 MMAs)
// so no operand is padded.  E4M3 codes widen to f16 exactly; q is scaled
// by a power of two 2^e so that its largest magnitude lies in [2^14, 2^15)
// (exact for every bf16 value in f16's normal range; 2^-e is folded into
// the softmax scale).  P is rounded to f16 for the MMA (the normaliser
// sums the fp32 values).
//
// Index maps (a reduction index may be permuted freely as long as both
// operands use the same map): lane (r = lane/4, c = lane%4) reads, of K,
// rows r and r+8 at dims [c*D/4, (c+1)*D/4), so its k-indices
// {2c, 2c+1, 2c+8, 2c+9} of MMA step kk are dims c*D/4 + 4kk + {0,1,2,3}:
// one 32-bit shared-memory word per row and step; q uses the same map.  Of
// V it reads tokens {2c, 2c+1, 2c+8, 2c+9} at dims [r*D/8, (r+1)*D/8): row
// m = r of output tile mt is dim r*D/8 + mt, row r+8 is r*D/8 + D/16 + mt,
// so the lane's output for one head is D/8 contiguous dims.  The S^T
// accumulator tile, transposed by movmatrix, is exactly P^T's B fragment.
PA_DEVICE void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

PA_DEVICE uint32_t movmatrix_trans(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

PA_DEVICE uint32_t f2_to_h2(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

PA_DEVICE uint32_t prmt(uint32_t x, uint32_t y, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(x), "r"(y), "r"(sel));
    return d;
}

// q of one item for the tensor-core path: head r, dims [c*D/4, (c+1)*D/4).
template <class C>
struct QPrefetchMma {
    static constexpr int NQ4 = C::D / 32;  // uint4 (8 bf16) per lane
    uint4 q[NQ4];
    float ks, vs;

    PA_DEVICE void load(const DecodeArgs &a, const Item &it, int r, int c) {
        const __nv_bfloat16 *qrow = static_cast<const __nv_bfloat16 *>(a.q) +
                                    ((size_t)it.b * a.Hq + (size_t)it.kvh * C::G + r) * C::D + c * (C::D / 4);
#pragma unroll
        for (int i = 0; i < NQ4; ++i) q[i] = reinterpret_cast<const uint4 *>(qrow)[i];
        ks = a.k_scale[it.kvh];
        vs = a.v_scale[it.kvh];
    }
};

template <class C>
PA_DEVICE void mma_items(const DecodeArgs &a, const Schedule &sc, Producer<C> &prod, ItemIter &items,
                         uint8_t *my_stages, uint64_t *my_bars, int *my_valid, int lane, const uint8_t *kc,
                         const uint8_t *vc, uint64_t deadline) {
    constexpr int D = C::D, G = C::G, NK = D / 16, NM = D / 16, KW = D / 16, VB = D / 8;
    static_assert(C::FP8 && G == 8, "tensor-core decode: fp8 cache, GQA 8");
    const int r = lane >> 2, c = lane & 3, Hkv = sc.Hkv;
    uint32_t consumed = 0;
    Item it, nx;
    bool have = items.next(sc, it);
    bool have_nx = have && items.next(sc, nx);
    QPrefetchMma<C> qp;
    if (have) qp.load(a, it, r, c);
    while (have) {
        const float vscale = qp.vs;
        // ---- q^T fragments in f16 with a power-of-two scale 2^e
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < QPrefetchMma<C>::NQ4; ++i) {
            const uint32_t ws[4] = {qp.q[i].x, qp.q[i].y, qp.q[i].z, qp.q[i].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = bf16x2_to_float2(ws[e]);
                amax = fmax3(amax, fabsf(f.x), fabsf(f.y));
            }
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, o));
        int ex = 0;
        if (amax > 0.f) ex = min(max(14 - ((int)((__float_as_uint(amax) >> 23) & 0xff) - 127), -60), 60);
        const float qsc = __uint_as_float((uint32_t)(127 + ex) << 23);
        const float sl2 = a.scale * kLog2e * qp.ks * __uint_as_float((uint32_t)(127 - ex) << 23);
        uint32_t qf[NK][2];
#pragma unroll
        for (int kk = 0; kk < NK; ++kk) {
            const uint4 u = qp.q[kk / 2];
            const uint32_t w0 = (kk & 1) ? u.z : u.x, w1 = (kk & 1) ? u.w : u.y;
            const float2 f0 = bf16x2_to_float2(w0), f1 = bf16x2_to_float2(w1);
            qf[kk][0] = f2_to_h2(f0.x * qsc, f0.y * qsc);
            qf[kk][1] = f2_to_h2(f1.x * qsc, f1.y * qsc);
        }
        float o[NM][4];
#pragma unroll
        for (int mt = 0; mt < NM; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
        float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // heads 2c, 2c+1

        for (int j = 0; j < it.nblk; ++j) {
            const int s = consumed % C::NSTAGE;
            // the lanes waited separately: agree (and converge) before the warp-wide MMAs
            if (!__all_sync(kFull, mbar_wait(&my_bars[s], (consumed / C::NSTAGE) & 1, deadline))) {
                give_up<C>(a, my_bars, consumed, prod.issued, lane);
                return;
            }
            const int valid = my_valid[s];
            const uint8_t *Kb = my_stages + (size_t)s * 2 * C::BLKB, *Vb = Kb + C::BLKB;
            // ---- S^T = K q^T
            uint32_t kr[KW], kr8[KW];
#pragma unroll
            for (int i = 0; i < KW / 4; ++i) {
                const uint4 u = *reinterpret_cast<const uint4 *>(Kb + r * D + c * (D / 4) + 16 * i);
                const uint4 u8 = *reinterpret_cast<const uint4 *>(Kb + (r + 8) * D + c * (D / 4) + 16 * i);
                kr[4 * i] = u.x, kr[4 * i + 1] = u.y, kr[4 * i + 2] = u.z, kr[4 * i + 3] = u.w;
                kr8[4 * i] = u8.x, kr8[4 * i + 1] = u8.y, kr8[4 * i + 2] = u8.z, kr8[4 * i + 3] = u8.w;
            }
            float st[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int kk = 0; kk < NK; ++kk)
                mma_f16(st, e4m3x2_to_h2(kr[kk]), e4m3x2_to_h2(kr8[kk]), e4m3x2_to_h2(kr[kk] >> 16),
                        e4m3x2_to_h2(kr8[kk] >> 16), qf[kk][0], qf[kk][1]);
            // V rows of this lane's tokens, loaded now so they overlap the softmax
            uint32_t vw[4][VB / 4];
            {
                const int tok[4] = {2 * c, 2 * c + 1, 2 * c + 8, 2 * c + 9};
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const uint8_t *src = Vb + tok[t] * D + r * VB;
                    if constexpr (VB == 16) {
                        const uint4 u = *reinterpret_cast<const uint4 *>(src);
                        vw[t][0] = u.x, vw[t][1] = u.y, vw[t][2] = u.z, vw[t][3] = u.w;
                    } else {
                        const uint2 u = *reinterpret_cast<const uint2 *>(src);
                        vw[t][0] = u.x, vw[t][1] = u.y;
                    }
                }
                if (valid < 16) {  // rows past the end may hold any bytes (NaN codes): zero them
#pragma unroll
                    for (int t = 0; t < 4; ++t)
                        if (tok[t] >= valid)
#pragma unroll
                            for (int i = 0; i < VB / 4; ++i) vw[t][i] = 0u;
                }
            }
            // ---- online softmax over the block's tokens, heads 2c and 2c+1
            const bool ok0 = r < valid, ok8 = r + 8 < valid;
            const float t0 = ok0 ? st[0] * sl2 : -INFINITY, t1 = ok0 ? st[1] * sl2 : -INFINITY;
            const float t2 = ok8 ? st[2] * sl2 : -INFINITY, t3 = ok8 ? st[3] * sl2 : -INFINITY;
            const bool need = fmaxf(t0, t2) > m0 + kRescaleThreshold || fmaxf(t1, t3) > m1 + kRescaleThreshold;
            if (__any_sync(kFull, need)) {
                float b0 = fmaxf(t0, t2), b1 = fmaxf(t1, t3);
#pragma unroll
                for (int x = 4; x <= 16; x <<= 1) {
                    b0 = fmaxf(b0, __shfl_xor_sync(kFull, b0, x));
                    b1 = fmaxf(b1, __shfl_xor_sync(kFull, b1, x));
                }
                const float n0 = fmaxf(m0, b0), n1 = fmaxf(m1, b1);
                const float al0 = (n0 == -INFINITY) ? 1.f : ex2(m0 - n0), al1 = (n1 == -INFINITY) ? 1.f : ex2(m1 - n1);
                m0 = n0, m1 = n1;
                l0 *= al0, l1 *= al1;
#pragma unroll
                for (int mt = 0; mt < NM; ++mt) {
                    o[mt][0] *= al0, o[mt][2] *= al0;
                    o[mt][1] *= al1, o[mt][3] *= al1;
                }
            }
            const float mb0 = (m0 == -INFINITY) ? 0.f : m0, mb1 = (m1 == -INFINITY) ? 0.f : m1;
            const float p0 = ex2(t0 - mb0), p1 = ex2(t1 - mb1), p2 = ex2(t2 - mb0), p3 = ex2(t3 - mb1);
            l0 += p0 + p2;
            l1 += p1 + p3;
            // P^T fragments: the accumulator tile (tokens x heads) transposed
            const uint32_t pb0 = movmatrix_trans(f2_to_h2(p0, p1)), pb1 = movmatrix_trans(f2_to_h2(p2, p3));
            // ---- O^T += V^T P^T, two output tiles per byte-pair permute
#pragma unroll
            for (int mt = 0; mt < NM; mt += 2) {
                const int w = mt / 4, bsel = mt % 4;
                const uint32_t sel = bsel | ((4 + bsel) << 4) | ((bsel + 1) << 8) | ((5 + bsel) << 12);
                constexpr int HW = (D / 16) / 4;  // word offset of the rows r+8 dims
                const uint32_t x0 = prmt(vw[0][w], vw[1][w], sel);            // tokens 2c, 2c+1, row r
                const uint32_t x1 = prmt(vw[0][w + HW], vw[1][w + HW], sel);  // tokens 2c, 2c+1, row r+8
                const uint32_t x2 = prmt(vw[2][w], vw[3][w], sel);            // tokens 2c+8, 2c+9, row r
                const uint32_t x3 = prmt(vw[2][w + HW], vw[3][w + HW], sel);
                mma_f16(o[mt], e4m3x2_to_h2(x0), e4m3x2_to_h2(x1), e4m3x2_to_h2(x2), e4m3x2_to_h2(x3), pb0, pb1);
                mma_f16(o[mt + 1], e4m3x2_to_h2(x0 >> 16), e4m3x2_to_h2(x1 >> 16), e4m3x2_to_h2(x2 >> 16),
                        e4m3x2_to_h2(x3 >> 16), pb0, pb1);
            }
            __syncwarp();
            ++consumed;
            prod.produce(sc, a, lane, kc, vc, my_stages, my_bars, my_valid);
        }
        if (have_nx) qp.load(a, nx, r, c);

        // ---- epilogue: the normalisers over the lanes of each head
#pragma unroll
        for (int x = 4; x <= 16; x <<= 1) {
            l0 += __shfl_xor_sync(kFull, l0, x);
            l1 += __shfl_xor_sync(kFull, l1, x);
        }
        const size_t row0 = (size_t)it.b * a.Hq + (size_t)it.kvh * G;
        const float inv0 = (l0 > 0.f) ? vscale / l0 : 0.f, inv1 = (l1 > 0.f) ? vscale / l1 : 0.f;
        // head 2c: o[.][0] (dims r*VB + mt) then o[.][2] (dims r*VB + NM + mt); head 2c+1: [1], [3]
        if (it.npieces == 1 && !a.prefix_blocks) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const float inv = hh ? inv1 : inv0;
                uint32_t wds[VB / 2];
#pragma unroll
                for (int i = 0; i < VB / 2; ++i) {
                    const int d0 = 2 * i, d1 = 2 * i + 1;  // dims r*VB + d
                    const float v0 = d0 < NM ? o[d0][hh] : o[d0 - NM][2 + hh];
                    const float v1 = d1 < NM ? o[d1][hh] : o[d1 - NM][2 + hh];
                    const __nv_bfloat162 bb = __floats2bfloat162_rn(v0 * inv, v1 * inv);
                    wds[i] = *reinterpret_cast<const uint32_t *>(&bb);
                }
                uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.out) +
                                                       (row0 + 2 * c + hh) * D + r * VB);
#pragma unroll
                for (int i = 0; i < VB / 8; ++i) dst[i] = make_uint4(wds[4 * i], wds[4 * i + 1], wds[4 * i + 2], wds[4 * i + 3]);
            }
            if (lane == 0 && a.ws_np) a.ws_np[(size_t)it.b * Hkv + it.kvh] = 1;
        } else {
            const int piece = it.piece + a.prefix_pieces;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const float inv = hh ? inv1 : inv0;
                float4 *dst = reinterpret_cast<float4 *>(a.ws_o + ((row0 + 2 * c + hh) * a.max_parts + piece) * D + r * VB);
#pragma unroll
                for (int i = 0; i < VB / 4; ++i) {
                    float v[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int d = 4 * i + e;
                        v[e] = (d < NM ? o[d][hh] : o[d - NM][2 + hh]) * inv;
                    }
                    dst[i] = make_float4(v[0], v[1], v[2], v[3]);
                }
            }
            if (r == 0) {
                a.ws_lse[(row0 + 2 * c) * a.max_parts + piece] = (l0 > 0.f) ? m0 + lg2(l0) : -INFINITY;
                a.ws_lse[(row0 + 2 * c + 1) * a.max_parts + piece] = (l1 > 0.f) ? m1 + lg2(l1) : -INFINITY;
            }
            if (lane == 0 && it.piece == 0) a.ws_np[(size_t)it.b * Hkv + it.kvh] = it.npieces + a.prefix_pieces;
        }
        it = nx;
        have = have_nx;
        have_nx = have && items.next(sc, nx);
    }
}

template <class C>
__global__ void __launch_bounds__(C::NT, C::MIN_CTAS) decode_kernel(const DecodeArgs a) {
    constexpr int D = C::D, G = C::G, NW = C::NW, NS = C::NS, VPL = C::VPL, P2 = C::P2, LPT = C::LPT;
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t *stages = smem;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::STAGE_BYTES);
    int *stage_valid = reinterpret_cast<int *>(bars + NW * C::NSTAGE);
    int *wsum = stage_valid + NW * C::NSTAGE;  // [2*NW]
    int *s_len = wsum + 2 * NW;                // [B]
    int *s_pre0 = s_len + a.B;                 // [B+1]
    int *s_pre1 = s_pre0 + a.B + 1;            // [B+1]

    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int g = lane / LPT, sub = lane % LPT;
    const int B = a.B, Hkv = a.Hkv, P = a.partition_tokens;  // P == 0: balanced split
    const int gw = blockIdx.x * NW + w, GW = gridDim.x * NW;
    pdl_trigger();  // the merge kernel may be scheduled now; it waits for this grid
    pdl_wait();     // the preceding kernel (e.g. the K/V write) has completed
    const uint64_t deadline = wait_deadline();  // shared by every wait of this launch
    {
        // bring the block tables and q into L2 while the split is built: the
        // first bulk copies wait on table entries, the first items on q
        const size_t tb = (size_t)B * a.max_blocks * sizeof(int32_t), qb = (size_t)B * a.Hq * D * 2;
        const size_t step = (size_t)gridDim.x * C::NT * 128, o0 = ((size_t)blockIdx.x * C::NT + tid) * 128;
        for (size_t o = o0; o < tb; o += step) prefetch_l2(reinterpret_cast<const char *>(a.block_tables) + o);
        for (size_t o = o0; o < qb; o += step) prefetch_l2(static_cast<const char *>(a.q) + o);
    }

    // ---- lengths, then exclusive scans over sequences: the balanced split
    // needs each sequence's offset in the line (Hkv segments of cost units),
    // the fixed one the numbers of full partitions and of ragged tails.
    const int cap = a.max_blocks * 16, skip = a.prefix_blocks * 16;  // cascade: attend tokens [skip, len)
    for (int b = tid; b < B; b += C::NT) {
        int len = a.seq_lens[b];
        if (len < skip || len > cap) {
            flag_error(a.err, PA_DEVERR_BAD_LEN);
            len = skip;
        }
        s_len[b] = len - skip;
    }
    if (lane < C::NSTAGE) mbar_init(&bars[w * C::NSTAGE + lane], 1);
    fence_mbar_init();
    __syncthreads();
    {
        auto count0 = [&](int len) {
            return P == 0 ? (len > 0 ? Hkv * (((len + 15) >> 4) + kSegmentCost) : 0) : len / P;
        };
        auto count1 = [&](int len) { return P == 0 ? 0 : (int)((len % P) != 0); };
        const int per = (B + C::NT - 1) / C::NT;  // each thread scans a run of sequences
        const int b0 = min(B, tid * per), b1 = min(B, b0 + per);
        int f = 0, t = 0;
        for (int b = b0; b < b1; ++b) {
            f += count0(s_len[b]);
            t += count1(s_len[b]);
        }
        int fi = f, ti = t;  // inclusive warp scan
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int fu = __shfl_up_sync(kFull, fi, o), tu = __shfl_up_sync(kFull, ti, o);
            if (lane >= o) {
                fi += fu;
                ti += tu;
            }
        }
        if (lane == 31) {
            wsum[w] = fi;
            wsum[NW + w] = ti;
        }
        __syncthreads();
        int fb = 0, tb = 0;
        for (int i = 0; i < w; ++i) {
            fb += wsum[i];
            tb += wsum[NW + i];
        }
        int fx = fb + fi - f, tx = tb + ti - t;  // exclusive prefix of this thread's run
        for (int b = b0; b < b1; ++b) {
            s_pre0[b] = fx;
            s_pre1[b] = tx;
            fx += count0(s_len[b]);
            tx += count1(s_len[b]);
        }
        if (tid == C::NT - 1) {
            s_pre0[B] = fx;
            s_pre1[B] = tx;
        }
        __syncthreads();
    }
    Schedule sc;
    sc.len = s_len;
    sc.pre0 = s_pre0;
    sc.pre1 = s_pre1;
    sc.B = B;
    sc.Hkv = Hkv;
    sc.P = P;
    if (P == 0) {
        sc.total = s_pre0[B];
        sc.S = max((sc.total + GW - 1) / GW, kMinShareBlocks);
        sc.NF = 0;
    } else {
        sc.NF = s_pre0[B];
        sc.total = (sc.NF + s_pre1[B]) * Hkv;
        sc.S = 0;
    }
    // empty sequences produce all-zero rows (no item covers them); in a
    // cascade their output is the shared-prefix piece alone
    for (int b = blockIdx.x; b < B; b += gridDim.x)
        if (s_len[b] == 0) {
            if (a.prefix_blocks)
                for (int k = tid; k < Hkv; k += C::NT) a.ws_np[(size_t)b * Hkv + k] = a.prefix_pieces;
            else
                for (int i = tid; i < a.Hq * D; i += C::NT)
                    static_cast<__nv_bfloat16 *>(a.out)[(size_t)b * a.Hq * D + i] = __float2bfloat16_rn(0.f);
        }

    const uint8_t *kc = static_cast<const uint8_t *>(a.k_cache);
    const uint8_t *vc = static_cast<const uint8_t *>(a.v_cache);
    uint8_t *my_stages = stages + (size_t)w * C::NSTAGE * 2 * C::BLKB;
    uint64_t *my_bars = bars + w * C::NSTAGE;
    int *my_valid = stage_valid + w * C::NSTAGE;

    Producer<C> prod;
    prod.init(sc, a, gw, GW, lane);

    // ---- per-lane constants: which 16-byte chunks of a row this lane reads.
    // Odd token groups visit their chunks in the other order so that lanes
    // of neighbouring groups never hit the same banks in the same access.
    int choff[C::NCH];
#pragma unroll
    for (int c = 0; c < C::NCH; ++c) choff[c] = sub + LPT * ((c + g) % C::NCH);
    // register layout of the partial scores (see rs_level)
    const int S = C::RS ? sub * VPL : 0;
    const int sh = S % G;  // head slot h holds head h ^ sh
    const int sj = S / G;  // token slot j reads token j ^ sj of the sub-step
    uint32_t consumed = 0;

    for (int prime = 0; prime < C::NSTAGE; ++prime) prod.produce(sc, a, lane, kc, vc, my_stages, my_bars, my_valid);

    ItemIter items;
    items.start(sc, gw, GW);
    if constexpr (C::MMA) {
        mma_items<C>(a, sc, prod, items, my_stages, my_bars, my_valid, lane, kc, vc, deadline);
    } else {
        Item it, nx;
        bool have = items.next(sc, it);
        bool have_nx = have && items.next(sc, nx);
        QPrefetch<C> qp;
        if (have) qp.load(a, it, choff, sh);
        while (have) {
            const float vscale = qp.vs;
            const float qs = a.scale * kLog2e * qp.ks;
            const size_t row0 = (size_t)it.b * a.Hq + (size_t)it.kvh * G;  // first q head of the group

            // q of the GQA group in fp32, pre-scaled into log2 units; slot h = head h ^ sh
            float2 q2[G][P2], acc2[G][P2];
            float m[G], l[G];
    #pragma unroll
            for (int h = 0; h < G; ++h) {
    #pragma unroll
                for (int c = 0; c < C::NCH; ++c) {
                    const uint32_t ws[4] = {qp.q[h][c].x, qp.q[h][c].y, qp.q[h][c].z, qp.q[h][c].w};
    #pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = bf16x2_to_float2(ws[e]);
                        q2[h][4 * c + e] = make_float2(f.x * qs, f.y * qs);
                        acc2[h][4 * c + e] = make_float2(0.f, 0.f);
                    }
                }
                m[h] = -INFINITY;
                l[h] = 0.f;
            }

            for (int j = 0; j < it.nblk; ++j) {
                const int s = consumed % C::NSTAGE;
                if (!__all_sync(kFull, mbar_wait(&my_bars[s], (consumed / C::NSTAGE) & 1, deadline))) {
                    give_up<C>(a, my_bars, consumed, prod.issued, lane);
                    return;
                }
                const int valid = my_valid[s];
                const uint8_t *Kb = my_stages + (size_t)s * 2 * C::BLKB, *Vb = Kb + C::BLKB;

    #pragma unroll
                for (int sb = 0; sb < C::NSUB; ++sb) {
                    const int t_base = g + C::NGRP * sb * C::TSUB;
                    // --- q . k: partial dot products over this lane's dims
                    float part[NS];
    #pragma unroll
                    for (int jj = 0; jj < C::TSUB; ++jj) {
                        float2 kf[P2];
                        load_row<C>(Kb + (t_base + C::NGRP * (jj ^ sj)) * C::ROWB, choff, kf);
    #pragma unroll
                        for (int h = 0; h < G; ++h) {
                            float2 d2 = make_float2(0.f, 0.f);
    #pragma unroll
                            for (int k = 0; k < P2; ++k) d2 = ffma2(q2[h][k], kf[k], d2);
                            part[jj * G + h] = d2.x + d2.y;
                        }
                    }
                    // --- complete the scores across the LPT lanes of the group
                    if constexpr (C::RS)
                        rs_level<LPT / 2, NS / 2, NS>(part);
                    else
                        allreduce_level<LPT / 2, NS>(part);
                    // --- owned score i: head slot i % G, token slot i / G.
                    // Mask tokens past the end; move the running max only when a
                    // score exceeds it by more than the threshold.
                    float sco[VPL];
                    bool need = false;
    #pragma unroll
                    for (int i = 0; i < VPL; ++i) {
                        const int t = t_base + C::NGRP * ((i / G) ^ sj);
                        sco[i] = (t < valid) ? part[i] : -INFINITY;
                        need |= sco[i] > m[i % G] + kRescaleThreshold;
                    }
                    if (__any_sync(kFull, need)) {
                        float bm[G];
    #pragma unroll
                        for (int h = 0; h < G; ++h) bm[h] = -INFINITY;
    #pragma unroll
                        for (int i = 0; i < VPL; ++i) bm[i % G] = fmaxf(bm[i % G], sco[i]);
                        if constexpr (C::RS) perm_allreduce<LPT / 2, VPL, G, true>(bm);
    #pragma unroll
                        for (int h = 0; h < G; ++h) {
                            const float mn = fmaxf(m[h], bm[h]);
                            const float alpha = (mn == -INFINITY) ? 1.f : ex2(m[h] - mn);
                            m[h] = mn;
                            l[h] *= alpha;
    #pragma unroll
                            for (int k = 0; k < P2; ++k) acc2[h][k] = fmul2(acc2[h][k], make_float2(alpha, alpha));
                        }
                    }
                    // --- probabilities of the owned scores, then all-gather them
                    float pr[NS];
    #pragma unroll
                    for (int i = 0; i < VPL; ++i) {
                        const float p = (sco[i] == -INFINITY) ? 0.f : ex2(sco[i] - m[i % G]);
                        l[i % G] += p;
                        pr[i] = p;
                    }
                    if constexpr (C::RS) ag_level<1, LPT, VPL, NS>(pr);
                    // --- acc += p * v over this group's tokens
    #pragma unroll
                    for (int jj = 0; jj < C::TSUB; ++jj) {
                        const int t = t_base + C::NGRP * (jj ^ sj);
                        if (t < valid) {
                            float2 vf[P2];
                            load_row<C>(Vb + t * C::ROWB, choff, vf);
    #pragma unroll
                            for (int h = 0; h < G; ++h) {
                                const float p = pr[jj * G + h];
                                const float2 pp = make_float2(p, p);
    #pragma unroll
                                for (int k = 0; k < P2; ++k) acc2[h][k] = ffma2(pp, vf[k], acc2[h][k]);
                            }
                        }
                    }
                }
                __syncwarp();
                ++consumed;
                prod.produce(sc, a, lane, kc, vc, my_stages, my_bars, my_valid);
            }

            // ---- the next item's q and scales are needed right after this
            // epilogue: start their loads now so the latency overlaps it
            if (have_nx) qp.load(a, nx, choff, sh);

            // ---- epilogue: complete the normaliser per head across the group,
            // then merge the token groups (same dims, different tokens)
            if constexpr (C::RS) perm_allreduce<LPT / 2, VPL, G, false>(l);
            group_merge<LPT, LPT, G, P2, C::NCH == 2>(m, l, acc2);

            // every group now holds the warp's result; group 0 writes it
            if (it.npieces == 1 && !a.prefix_blocks) {
                if (g == 0) {
    #pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const float inv = (l[h] > 0.f) ? vscale / l[h] : 0.f;
                        __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(a.out) + (row0 + (h ^ sh)) * D;
    #pragma unroll
                        for (int c = 0; c < C::NCH; ++c) {
                            uint32_t wds[4];
    #pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const __nv_bfloat162 bb =
                                    __floats2bfloat162_rn(acc2[h][4 * c + e].x * inv, acc2[h][4 * c + e].y * inv);
                                wds[e] = *reinterpret_cast<const uint32_t *>(&bb);
                            }
                            *reinterpret_cast<uint4 *>(dst + choff[c] * 8) = make_uint4(wds[0], wds[1], wds[2], wds[3]);
                        }
                    }
                }
                if (lane == 0 && a.ws_np) a.ws_np[(size_t)it.b * Hkv + it.kvh] = 1;  // nothing to merge
            } else {
                // ---- split-K: this piece's normalised output and log2-sum-exp;
                // piece 0 also records how many pieces the merge kernel combines
                // (in a cascade the pieces follow the shared prefix's pieces)
                const int piece = it.piece + a.prefix_pieces;
                if (g == 0) {
    #pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const float inv = (l[h] > 0.f) ? vscale / l[h] : 0.f;
                        float *dst = a.ws_o + ((row0 + (h ^ sh)) * a.max_parts + piece) * D;
    #pragma unroll
                        for (int c = 0; c < C::NCH; ++c) {
                            float4 *d4 = reinterpret_cast<float4 *>(dst + choff[c] * 8);
                            d4[0] = make_float4(acc2[h][4 * c].x * inv, acc2[h][4 * c].y * inv,
                                                acc2[h][4 * c + 1].x * inv, acc2[h][4 * c + 1].y * inv);
                            d4[1] = make_float4(acc2[h][4 * c + 2].x * inv, acc2[h][4 * c + 2].y * inv,
                                                acc2[h][4 * c + 3].x * inv, acc2[h][4 * c + 3].y * inv);
                        }
                        if (sub == 0)  // sub 0 has sh == 0: slot h is head h
                            a.ws_lse[(row0 + h) * a.max_parts + piece] = (l[h] > 0.f) ? m[h] + lg2(l[h]) : -INFINITY;
                    }
                }
                if (lane == 0 && it.piece == 0)
                    a.ws_np[(size_t)it.b * Hkv + it.kvh] = it.npieces + a.prefix_pieces;
            }
            it = nx;
            have = have_nx;
            have_nx = have && items.next(sc, nx);
        }
    }
}

// Log-sum-exp merge of the split-K pieces, one warp per (sequence, q head):
//     out = sum_p w_p o_p / sum_p w_p,   w_p = 2^(lse_p - max_p lse_p)
// where o_p is piece p's normalised output and lse_p its log2-sum-exp.  Runs
// as a programmatic dependent of the decode kernel: its CTAs may become
// resident while the decode grid drains, and griddepcontrol.wait returns
// once that grid has completed with its memory visible.  Lane l owns head
// dims [l*E, l*E + E).  The length, the piece count and the first
// merge_spec pieces are loaded together (their addresses do not depend on
// the count), so a row of up to merge_spec pieces costs one L2 round trip;
// the launcher picks merge_spec so that those slots are written for every
// row that needs a merge (a cascade's prefix pieces and its first suffix
// piece; 2 in plain decode), so the look-ahead never reads a stale slot
// (after an L2 flush, from DRAM).  The rest of a row's pieces are loaded
// once its count is known.
// Pieces a merge warp loads at a time (its first round trip holds at most
// this many; a larger count is merged in further chunks).  4 keeps the
// kernel at 47 registers, 40 warps an SM; with 8 it took 64 registers and
// a 256-sequence cascade's 16,384-row merge ran ~1 us longer.
constexpr int kMergeFirst = 4;

template <int D>
__global__ void __launch_bounds__(128) merge_kernel(const DecodeArgs a) {
    constexpr int E = D / 32, kFirst = kMergeFirst;
    pdl_trigger();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * 4 + (threadIdx.x >> 5);  // b * Hq + h
    if (row >= (long long)a.B * a.Hq) return;
    const int b = (int)(row / a.Hq), h = (int)(row % a.Hq), kvh = h / (a.Hq / a.Hkv);
    const float *lse = a.ws_lse + (size_t)row * a.max_parts;
    const float *op = a.ws_o + (size_t)row * a.max_parts * D + lane * E;
    auto load_o = [&](int p, float (&v)[E]) {
        if constexpr (E == 4) {
            const float4 x = __ldcg(reinterpret_cast<const float4 *>(op + (size_t)p * D));
            v[0] = x.x;
            v[1] = x.y;
            v[2] = x.z;
            v[3] = x.w;
        } else {
            const float2 x = __ldcg(reinterpret_cast<const float2 *>(op + (size_t)p * D));
            v[0] = x.x;
            v[1] = x.y;
        }
    };
    const int len = __ldcg(a.seq_lens + b);
    const int np = __ldcg(a.ws_np + (size_t)b * a.Hkv + kvh);
    const int spec = a.merge_spec;  // <= min(kFirst, max_parts)
    float lp[kFirst], v[kFirst][E];
#pragma unroll
    for (int u = 0; u < kFirst; ++u)
        if (u < spec) {
            lp[u] = __ldcg(lse + u);
            load_o(u, v[u]);
        }
    if (len <= 0 || len > a.max_blocks * 16) return;  // empty or rejected: the decode kernel wrote the row
    if (np <= (a.prefix_blocks ? 0 : 1)) return;       // one piece: the decode kernel wrote the row
    if (np > a.max_parts) {
        if (lane == 0) flag_error(a.err, PA_DEVERR_BAD_LEN);
        return;
    }
    // chunks of kFirst pieces, each chunk's loads in flight together; the
    // running max moves between chunks
    float M = -INFINITY, L = 0.f, acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
    for (int p0 = 0; p0 < np; p0 += kFirst) {
#pragma unroll
        for (int u = 0; u < kFirst; ++u)
            if (p0 + u < np && (p0 > 0 || u >= spec)) {
                lp[u] = __ldcg(lse + p0 + u);
                load_o(p0 + u, v[u]);
            }
        float mc = M;
#pragma unroll
        for (int u = 0; u < kFirst; ++u)
            if (p0 + u < np) mc = fmaxf(mc, lp[u]);  // slots past np may hold anything: never read
        if (mc == -INFINITY) continue;
        const float sc = (M == -INFINITY) ? 0.f : ex2(M - mc);
        M = mc;
        L *= sc;
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] *= sc;
#pragma unroll
        for (int u = 0; u < kFirst; ++u)
            if (p0 + u < np && lp[u] != -INFINITY) {
                const float w = ex2(lp[u] - M);
                L += w;
#pragma unroll
                for (int e = 0; e < E; ++e) acc[e] = fmaf(w, v[u][e], acc[e]);
            }
    }
    const float inv = (L > 0.f) ? 1.f / L : 0.f;
    __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(a.out) + (size_t)row * D + lane * E;
#pragma unroll
    for (int e = 0; e < E; e += 2)
        *reinterpret_cast<__nv_bfloat162 *>(out + e) = __floats2bfloat162_rn(acc[e] * inv, acc[e + 1] * inv);
}

template <class C>
cudaError_t run(const DecodeArgs &a, cudaStream_t st) {
    // Per device: opt in to the large shared-memory carve-out once, and
    // remember SM count and occupancy per shared-memory size (B decides it).
    struct Occ {
        int smem_key = -1, ctas = 0;
    };
    static std::mutex mu;
    static bool ready[64] = {};
    static int sms[64] = {};
    static Occ occ[64][4];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    const size_t smem = smem_bytes<C>(a.B);
    int ctas = 0;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!ready[dev]) {
            e = cudaFuncSetAttribute(decode_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)smem_bytes<C>(kMaxDecodeSeqs));
            if (e != cudaSuccess) return e;
            e = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
            if (e != cudaSuccess) return e;
            ready[dev] = true;
        }
        Occ *slot = nullptr;
        for (auto &o : occ[dev])
            if (o.smem_key == (int)smem) slot = &o;
        if (!slot) {
            int n = 0;
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_kernel<C>, C::NT, smem);
            if (e != cudaSuccess) return e;
            slot = &occ[dev][(smem / 16) % 4];
            slot->smem_key = (int)smem;
            slot->ctas = n < 1 ? 1 : n;
        }
        ctas = slot->ctas * sms[dev];
    }
    // enough CTAs to cover every warp-sized unit of work, at most one wave
    // (balanced: a segment costs its blocks plus kSegmentCost units)
    const long long units = a.partition_tokens == 0
                                ? (long long)a.Hkv * a.B * (a.max_blocks + kSegmentCost) / kMinShareBlocks + 1
                                : (long long)a.Hkv * a.B * a.max_parts;
    const long long grid = std::max<long long>(1, std::min<long long>((units + C::NW - 1) / C::NW, ctas));
    e = launch_pdl(decode_kernel<C>, dim3((unsigned)grid), dim3(C::NT), smem, st, a);
    if (e != cudaSuccess || !a.ws_np) return e;  // no workspace: every (sequence, kv head) is one piece
    const long long rows = (long long)a.B * a.Hq;
    DecodeArgs m = a;
    // pieces every merged row is sure to have: a cascade row has its prefix
    // pieces and (unless its suffix is empty) one suffix piece; a plain row
    // that needs a merge has at least two
    m.merge_spec = std::min({kMergeFirst, a.max_parts, a.prefix_blocks ? a.prefix_pieces + 1 : 2});
    return launch_pdl(merge_kernel<C::D>, dim3((unsigned)((rows + 3) / 4)), dim3(128), 0, st, m);
}

template <int D, bool FP8>
cudaError_t by_group(const DecodeArgs &a, cudaStream_t st) {
    switch (a.Hq / a.Hkv) {
        case 1: return run<Cfg<D, 1, FP8>>(a, st);
        case 2: return run<Cfg<D, 2, FP8>>(a, st);
        case 4: return run<Cfg<D, 4, FP8>>(a, st);
        case 8: return run<Cfg<D, 8, FP8>>(a, st);
        default: return cudaErrorNotSupported;
    }
}

}  // namespace

namespace {
size_t round256(size_t n) { return (n + 255) & ~(size_t)255; }
size_t ws_np_bytes(int B, int Hq) { return round256((size_t)B * Hq * sizeof(int)); }  // >= B * Hkv
size_t ws_o_bytes(int B, int Hq, int D, int max_parts) {
    return round256((size_t)B * Hq * max_parts * D * sizeof(float));
}
}  // namespace

size_t decode_ws_bytes(int B, int Hq, int D, int max_parts) {
    return ws_np_bytes(B, Hq) + ws_o_bytes(B, Hq, D, max_parts) + round256((size_t)B * Hq * max_parts * sizeof(float));
}

void decode_ws_carve(void *base, int B, int Hq, int D, int max_parts, DecodeArgs &a) {
    char *p = static_cast<char *>(base);
    a.ws_np = reinterpret_cast<int *>(p);
    a.ws_o = reinterpret_cast<float *>(p + ws_np_bytes(B, Hq));
    a.ws_lse = reinterpret_cast<float *>(p + ws_np_bytes(B, Hq) + ws_o_bytes(B, Hq, D, max_parts));
}

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t st) {
    if (a.D == 128) return a.fp8 ? by_group<128, true>(a, st) : by_group<128, false>(a, st);
    if (a.D == 64) return a.fp8 ? by_group<64, true>(a, st) : by_group<64, false>(a, st);
    return cudaErrorNotSupported;
}

}  // namespace pa
