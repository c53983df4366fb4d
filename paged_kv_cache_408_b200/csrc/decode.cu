// decode.cu -- paged decode attention for sm_100a, with split-K partials and
// a log-sum-exp merge.
//
// What is computed ("Production Serving: Continuous Batching and
// PagedAttention", The Build, Step 6 "Implement attention over paged
// storage", read per query head):
//     out[b][h] = sum_{t < len_b} softmax_t(scale * q[b][h] . k_t) v_t
// where token t of sequence b lives in slot t%16 of physical block
// block_tables[b][t/16], kv head floor(h*Hkv/Hq).
//
// How (B200 design):
//  * Work unit ("item") = (sequence, kv head, partition of `P` tokens).  One
//    CTA processes a whole GQA group for its item, so each K/V byte is read
//    from HBM exactly once per step.  Partitions depend only on token index:
//    a sequence's result never depends on the rest of the batch.
//  * Persistent grid: every CTA rebuilds the item list from seq_lens in
//    shared memory (a block-wide scan) and walks items
//    blockIdx.x, blockIdx.x + gridDim.x, ...; full partitions come first, the
//    ragged tails last.  No empty CTAs for short sequences, no host sync.
//  * Each warp streams its own 16-token blocks (blocks w, w+4, ... of the
//    item) through an NSTAGE-deep shared-memory ring filled by 1-D bulk
//    async copies (the TMA engine, 4 KB contiguous per K or V block) that
//    complete on mbarriers.  The producer runs ahead across item boundaries
//    and prefetches the next item's block-table entries into registers.
//  * Math on CUDA cores (the contraction per step is 4-8 query rows, far
//    below a tensor-core tile): lanes are split into token groups of LPT
//    lanes; a lane owns DPL head dims (16-byte shared-memory reads, bank-
//    conflict-free), holds q for those dims in fp32 registers pre-scaled by
//    scale*log2(e), and accumulates with packed fp32x2 FMAs.  Partial dot
//    products are combined by a shuffle reduce-scatter, exponentiated by the
//    owning lane, and all-gathered for the P.V step.
//  * Online softmax with a lazily updated running max: the max only moves
//    when a new score exceeds it by more than 2^8 (ratio), so the common
//    block needs no max shuffles; final normalisation divides by the sum
//    taken against the same max, so the result is the exact softmax.
//  * Each token group keeps its own (m, l, acc); groups, then warps, are
//    combined once per item.  A sequence with one partition writes bf16
//    output directly; longer ones write fp32 partials and log2-sum-exp to
//    the workspace, merged by merge_kernel.
#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace pa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: p <= 256 before a rescale
constexpr unsigned kFull = 0xffffffffu;

PA_DEVICE float lg2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

template <int D_, int G_, bool FP8_>
struct Cfg {
    static constexpr int D = D_, G = G_;
    static constexpr bool FP8 = FP8_;
    static constexpr int EB = FP8 ? 1 : 2;           // bytes per element
    static constexpr int DPL = (G >= 8) ? 8 : 16;     // head dims owned by a lane
    static constexpr int LPT = D / DPL;               // lanes per token
    static constexpr int NGRP = 32 / LPT;             // token groups per warp
    static constexpr int TPG = 16 / NGRP;             // tokens per group per block
    static constexpr int TSUB = (TPG * G > 32) ? 32 / G : TPG;  // tokens per group per sub-step
    static constexpr int NSUB = TPG / TSUB;
    static constexpr int NCH = DPL / 8;               // 8-element chunks per lane per row
    static constexpr int CHB = 8 * EB;                // bytes per chunk
    static constexpr int ROWB = D * EB;               // bytes per token row
    static constexpr int BLKB = 16 * ROWB;            // bytes of one block of one head (K or V)
    static constexpr int P2 = DPL / 2;                // fp32 pairs per lane per head
    static constexpr int NS = TSUB * G;               // partial scores per lane per sub-step
    static constexpr bool RS = NS >= LPT;             // reduce-scatter (else all-reduce)
    static constexpr int VPL = RS ? NS / LPT : NS;    // scores a lane owns after the reduction
    static constexpr int NW = 4;                      // warps per CTA
    static constexpr int NT = NW * 32;
    static constexpr int NSTAGE = 3;                  // ring depth per warp
    static constexpr size_t STAGE_BYTES = (size_t)NW * NSTAGE * 2 * BLKB;
    static constexpr size_t RED_FLOATS = (size_t)NW * G * (D + 2);
    static_assert(LPT >= 1 && LPT <= 32 && 32 % LPT == 0, "bad lane split");
    static_assert(TPG * NGRP == 16 && TSUB * NSUB == TPG, "bad token split");
};

template <class C>
size_t smem_bytes(int B) {
    size_t s = C::STAGE_BYTES;
    s += (size_t)C::NW * C::NSTAGE * 8;   // mbarriers
    s += (size_t)C::NW * C::NSTAGE * 4;   // valid-token count per stage
    s = (s + 15) & ~(size_t)15;
    s += C::RED_FLOATS * 4;               // cross-warp combine
    s += (size_t)(3 * B + 2) * 4;         // lens, full-partition scan, tail scan
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

struct Item {
    int b, kvh, part, len, blk0, nblk, nparts;
};

template <class C>
__global__ void __launch_bounds__(C::NT) decode_kernel(const DecodeArgs a) {
    constexpr int D = C::D, G = C::G, NW = C::NW, NS = C::NS, VPL = C::VPL, P2 = C::P2, LPT = C::LPT;
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t *stages = smem;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::STAGE_BYTES);
    int *stage_valid = reinterpret_cast<int *>(bars + NW * C::NSTAGE);
    size_t off = C::STAGE_BYTES + (size_t)NW * C::NSTAGE * 12;
    off = (off + 15) & ~(size_t)15;
    float *red_acc = reinterpret_cast<float *>(smem + off);  // [NW][G][D]
    float *red_m = red_acc + NW * G * D;                      // [NW][G]
    float *red_l = red_m + NW * G;                            // [NW][G]
    int *s_len = reinterpret_cast<int *>(red_l + NW * G);     // [B]
    int *s_full = s_len + a.B;                                // [B+1]
    int *s_tail = s_full + a.B + 1;                           // [B+1]

    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int g = lane / LPT, sub = lane % LPT;
    const int B = a.B, Hkv = a.Hkv, P = a.partition_tokens;

    // ---- lengths, then scans of full partitions and tails per sequence
    const int cap = a.max_blocks * 16;
    for (int b = tid; b < B; b += C::NT) {
        int len = a.seq_lens[b];
        if (len < 0 || len > cap) {
            flag_error(a.err, PA_DEVERR_BAD_LEN);
            len = 0;
        }
        s_len[b] = len;
    }
    if (lane < C::NSTAGE) mbar_init(&bars[w * C::NSTAGE + lane], 1);
    fence_mbar_init();
    __syncthreads();
    {
        // each thread scans a contiguous run of sequences, then a block scan
        const int per = (B + C::NT - 1) / C::NT;
        const int b0 = min(B, tid * per), b1 = min(B, b0 + per);
        int f = 0, t = 0;
        for (int b = b0; b < b1; ++b) {
            f += s_len[b] / P;
            t += (s_len[b] % P) != 0;
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
        int *wsum = reinterpret_cast<int *>(red_acc);  // scratch: 2*NW ints
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
            s_full[b] = fx;
            s_tail[b] = tx;
            fx += s_len[b] / P;
            tx += (s_len[b] % P) != 0;
        }
        if (tid == C::NT - 1) {
            s_full[B] = fx;
            s_tail[B] = tx;
        }
        __syncthreads();
    }
    const int NF = s_full[B];
    const int n_items = (NF + s_tail[B]) * Hkv;

    auto get_item = [&](int i) {
        Item it;
        it.kvh = i % Hkv;
        int u = i / Hkv;
        if (u < NF) {
            it.b = upper_index(s_full, B, u);
            it.part = u - s_full[it.b];
        } else {
            u -= NF;
            it.b = upper_index(s_tail, B, u);
            it.part = s_full[it.b + 1] - s_full[it.b];
        }
        it.len = s_len[it.b];
        it.nparts = (s_full[it.b + 1] - s_full[it.b]) + (s_tail[it.b + 1] - s_tail[it.b]);
        const int t0 = it.part * P, t1 = min(t0 + P, it.len);
        it.blk0 = t0 >> 4;
        it.nblk = ((t1 + 15) >> 4) - it.blk0;
        return it;
    };
    auto warp_blocks = [&](const Item &it) { return it.nblk > w ? (it.nblk - w + NW - 1) / NW : 0; };

    // ---- producer: one lane issues bulk copies; the warp prefetches table entries
    const uint8_t *kc = static_cast<const uint8_t *>(a.k_cache);
    const uint8_t *vc = static_cast<const uint8_t *>(a.v_cache);
    auto stage_k = [&](int s) { return stages + ((size_t)(w * C::NSTAGE + s) * 2) * C::BLKB; };
    auto stage_v = [&](int s) { return stage_k(s) + C::BLKB; };

    auto load_tbl = [&](int item, int &e0, int &e1) {
        e0 = e1 = -1;
        if (item >= n_items) return;
        const Item it = get_item(item);
        const int nbw = warp_blocks(it);
        const int32_t *row = a.block_tables + (size_t)it.b * a.max_blocks + it.blk0 + w;
        if (lane < nbw) e0 = row[NW * lane];
        if (lane + 32 < nbw) e1 = row[NW * (lane + 32)];
    };

    int p_item = blockIdx.x, p_j = 0, p_nbw = 0, p_kvh = 0, p_blk0 = 0, p_len = 0;
    int p_t0, p_t1, n_t0, n_t1;  // table entries of the current and of the next item
    load_tbl(p_item, p_t0, p_t1);
    load_tbl(p_item + gridDim.x, n_t0, n_t1);
    if (p_item < n_items) {
        const Item it = get_item(p_item);
        p_nbw = warp_blocks(it);
        p_kvh = it.kvh;
        p_blk0 = it.blk0;
        p_len = it.len;
    }
    uint32_t issued = 0, consumed = 0;

    auto produce = [&]() {
        while (p_item < n_items && p_j >= p_nbw) {
            p_item += gridDim.x;
            p_j = 0;
            p_t0 = n_t0;
            p_t1 = n_t1;
            load_tbl(p_item + gridDim.x, n_t0, n_t1);
            if (p_item < n_items) {
                const Item it = get_item(p_item);
                p_nbw = warp_blocks(it);
                p_kvh = it.kvh;
                p_blk0 = it.blk0;
                p_len = it.len;
            }
        }
        if (p_item >= n_items) return;
        int phys = __shfl_sync(kFull, p_j < 32 ? p_t0 : p_t1, p_j & 31);
        if (lane == 0) {
            const int blk = p_blk0 + w + NW * p_j;
            int valid = min(16, p_len - blk * 16);
            if (phys < 0 || phys >= a.num_blocks) {
                flag_error(a.err, PA_DEVERR_BAD_BLOCK);
                phys = 0;
                valid = 0;
            }
            const int s = issued % C::NSTAGE;
            stage_valid[w * C::NSTAGE + s] = valid;
            uint64_t *bar = &bars[w * C::NSTAGE + s];
            mbar_arrive_expect_tx(bar, 2 * C::BLKB);
            const size_t src = ((size_t)phys * Hkv + p_kvh) * C::BLKB;
            bulk_g2s(stage_k(s), kc + src, C::BLKB, bar);
            bulk_g2s(stage_v(s), vc + src, C::BLKB, bar);
        }
        ++issued;
        ++p_j;
    };

    // ---- per-lane constants: which 16-byte chunks of a row this lane reads.
    // Odd token groups visit their chunks in the other order so that lanes
    // of neighbouring groups never hit the same banks in the same access.
    int choff[C::NCH];
#pragma unroll
    for (int c = 0; c < C::NCH; ++c) choff[c] = sub + LPT * ((c + g) % C::NCH);

    auto load_row = [&](const uint8_t *row, float2 (&f)[P2]) {
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
    };

    // scores this lane owns after the reduction: sub-step token j and head h
    int own_j[VPL], own_h[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        const int idx = (C::RS ? sub * VPL : 0) + i;
        own_j[i] = idx / G;
        own_h[i] = idx % G;
    }

    for (int prime = 0; prime < C::NSTAGE; ++prime) produce();

    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        const Item it = get_item(item);
        const int nbw = warp_blocks(it);
        const float kscale = C::FP8 ? a.k_scale[it.kvh] : 1.0f;
        const float vscale = C::FP8 ? a.v_scale[it.kvh] : 1.0f;
        const float qs = a.scale * kLog2e * kscale;

        float2 q2[G][P2], acc2[G][P2];
        float m[G], m_own[VPL], l_own[VPL];
        {
            const __nv_bfloat16 *qrow =
                static_cast<const __nv_bfloat16 *>(a.q) + ((size_t)it.b * a.Hq + (size_t)it.kvh * G) * D;
#pragma unroll
            for (int h = 0; h < G; ++h) {
#pragma unroll
                for (int c = 0; c < C::NCH; ++c) {
                    const uint4 u = *reinterpret_cast<const uint4 *>(qrow + h * D + choff[c] * 8);
                    const uint32_t ws[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = bf16x2_to_float2(ws[e]);
                        q2[h][4 * c + e] = make_float2(f.x * qs, f.y * qs);
                        acc2[h][4 * c + e] = make_float2(0.f, 0.f);
                    }
                }
                m[h] = -INFINITY;
            }
#pragma unroll
            for (int i = 0; i < VPL; ++i) {
                m_own[i] = -INFINITY;
                l_own[i] = 0.f;
            }
        }

        for (int j = 0; j < nbw; ++j) {
            const int s = consumed % C::NSTAGE;
            if (!mbar_wait(&bars[w * C::NSTAGE + s], (consumed / C::NSTAGE) & 1) && lane == 0)
                flag_error(a.err, PA_DEVERR_TIMEOUT);
            const int valid = stage_valid[w * C::NSTAGE + s];
            const uint8_t *Kb = stage_k(s), *Vb = stage_v(s);

#pragma unroll
            for (int sb = 0; sb < C::NSUB; ++sb) {
                // --- q . k for this group's TSUB tokens, all G heads
                float part[NS];
#pragma unroll
                for (int jj = 0; jj < C::TSUB; ++jj) {
                    const int t = g + C::NGRP * (sb * C::TSUB + jj);
                    float2 kf[P2];
                    load_row(Kb + t * C::ROWB, kf);
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        float2 d2 = make_float2(0.f, 0.f);
#pragma unroll
                        for (int k = 0; k < P2; ++k) d2 = ffma2(q2[h][k], kf[k], d2);
                        part[jj * G + h] = d2.x + d2.y;
                    }
                }
                // --- combine partial dot products across the LPT lanes of the group
                if constexpr (C::RS) {
                    int n = NS;
#pragma unroll
                    for (int mask = LPT / 2; mask >= 1; mask >>= 1) {
                        n >>= 1;
                        const bool hi = (sub & mask) != 0;
#pragma unroll
                        for (int k = 0; k < NS / 2; ++k) {
                            if (k < n) {
                                const float send = hi ? part[k] : part[k + n];
                                const float keep = hi ? part[k + n] : part[k];
                                part[k] = keep + __shfl_xor_sync(kFull, send, mask);
                            }
                        }
                    }
                } else {
#pragma unroll
                    for (int mask = LPT / 2; mask >= 1; mask >>= 1)
#pragma unroll
                        for (int k = 0; k < NS; ++k) part[k] += __shfl_xor_sync(kFull, part[k], mask);
                }
                // --- mask tokens past the end, check whether the running max must move
                float sc[VPL];
                bool need = false;
#pragma unroll
                for (int i = 0; i < VPL; ++i) {
                    const int t = g + C::NGRP * (sb * C::TSUB + own_j[i]);
                    sc[i] = (t < valid) ? part[i] : -INFINITY;
                    need |= sc[i] > m_own[i] + kRescaleThreshold;
                }
                if (__any_sync(kFull, need)) {
                    float bm[G];
#pragma unroll
                    for (int h = 0; h < G; ++h) bm[h] = -INFINITY;
#pragma unroll
                    for (int i = 0; i < VPL; ++i)
#pragma unroll
                        for (int h = 0; h < G; ++h)
                            if (own_h[i] == h) bm[h] = fmaxf(bm[h], sc[i]);
                    if constexpr (C::RS) {
#pragma unroll
                        for (int mask = LPT / 2; mask >= 1; mask >>= 1)
#pragma unroll
                            for (int h = 0; h < G; ++h) bm[h] = fmaxf(bm[h], __shfl_xor_sync(kFull, bm[h], mask));
                    }
                    float alpha[G];
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const float mn = fmaxf(m[h], bm[h]);
                        alpha[h] = (mn == -INFINITY) ? 1.f : ex2(m[h] - mn);
                        m[h] = mn;
#pragma unroll
                        for (int k = 0; k < P2; ++k)
                            acc2[h][k] = fmul2(acc2[h][k], make_float2(alpha[h], alpha[h]));
                    }
#pragma unroll
                    for (int i = 0; i < VPL; ++i) {
#pragma unroll
                        for (int h = 0; h < G; ++h)
                            if (own_h[i] == h) {
                                l_own[i] *= alpha[h];
                                m_own[i] = m[h];
                            }
                    }
                }
                // --- probabilities of the owned scores, then all-gather them
                float pr[NS];
#pragma unroll
                for (int i = 0; i < VPL; ++i) {
                    const float p = (sc[i] == -INFINITY) ? 0.f : ex2(sc[i] - m_own[i]);
                    l_own[i] += p;
                    pr[i] = p;
                }
                if constexpr (C::RS) {
                    int n = VPL;
#pragma unroll
                    for (int mask = 1; mask < LPT; mask <<= 1) {
                        const bool hi = (sub & mask) != 0;
#pragma unroll
                        for (int k = 0; k < NS / 2; ++k) {
                            if (k < n) {
                                const float r = __shfl_xor_sync(kFull, pr[k], mask);
                                const float mine = pr[k];
                                pr[k] = hi ? r : mine;
                                pr[k + n] = hi ? mine : r;
                            }
                        }
                        n <<= 1;
                    }
                }
                // --- acc += p * v for this group's tokens
#pragma unroll
                for (int jj = 0; jj < C::TSUB; ++jj) {
                    const int t = g + C::NGRP * (sb * C::TSUB + jj);
                    if (t < valid) {
                        float2 vf[P2];
                        load_row(Vb + t * C::ROWB, vf);
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
            produce();
        }

        // ---- epilogue: normaliser per head within the group
        float l[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
            l[h] = 0.f;
#pragma unroll
            for (int i = 0; i < VPL; ++i)
                if (own_h[i] == h) l[h] += l_own[i];
        }
        if constexpr (C::RS) {
#pragma unroll
            for (int mask = 1; mask < LPT; mask <<= 1)
#pragma unroll
                for (int h = 0; h < G; ++h) l[h] += __shfl_xor_sync(kFull, l[h], mask);
        }
        // ---- combine token groups of this warp (same dims, different tokens)
#pragma unroll
        for (int mask = LPT; mask < 32; mask <<= 1) {
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float mo = __shfl_xor_sync(kFull, m[h], mask);
                const float lo = __shfl_xor_sync(kFull, l[h], mask);
                const float M = fmaxf(m[h], mo);
                const float am = (m[h] == -INFINITY) ? 0.f : ex2(m[h] - M);
                const float ao = (mo == -INFINITY) ? 0.f : ex2(mo - M);
                l[h] = l[h] * am + lo * ao;
                m[h] = M;
                // Groups of opposite parity visit their chunks in swapped
                // order: pull the partner's register that holds my chunk.
                constexpr bool swap = (C::NCH == 2);
                float2 rx[P2];
#pragma unroll
                for (int k = 0; k < P2; ++k) {
                    const int ks = (swap && mask == LPT) ? (k ^ 4) : k;
                    rx[k].x = __shfl_xor_sync(kFull, acc2[h][ks].x, mask);
                    rx[k].y = __shfl_xor_sync(kFull, acc2[h][ks].y, mask);
                }
#pragma unroll
                for (int k = 0; k < P2; ++k)
                    acc2[h][k] = ffma2(acc2[h][k], make_float2(am, am), make_float2(rx[k].x * ao, rx[k].y * ao));
            }
        }
        // ---- combine warps through shared memory
        if (g == 0) {
#pragma unroll
            for (int h = 0; h < G; ++h) {
#pragma unroll
                for (int c = 0; c < C::NCH; ++c) {
                    float *dst = red_acc + ((size_t)w * G + h) * D + choff[c] * 8;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        dst[2 * e] = acc2[h][4 * c + e].x;
                        dst[2 * e + 1] = acc2[h][4 * c + e].y;
                    }
                }
                if (sub == 0) {
                    red_m[w * G + h] = m[h];
                    red_l[w * G + h] = l[h];
                }
            }
        }
        __syncthreads();
        const bool single = it.nparts == 1;
        for (int idx = tid; idx < G * D; idx += C::NT) {
            const int h = idx / D, d = idx % D;
            float M = -INFINITY;
#pragma unroll
            for (int v = 0; v < NW; ++v) M = fmaxf(M, red_m[v * G + h]);
            float L = 0.f, O = 0.f;
#pragma unroll
            for (int v = 0; v < NW; ++v) {
                const float mv = red_m[v * G + h];
                const float f = (mv == -INFINITY) ? 0.f : ex2(mv - M);
                L += red_l[v * G + h] * f;
                O += red_acc[((size_t)v * G + h) * D + d] * f;
            }
            const float o = (L > 0.f) ? (O / L) * vscale : 0.f;
            const size_t row = (size_t)it.b * a.Hq + (size_t)it.kvh * G + h;
            if (single) {
                static_cast<__nv_bfloat16 *>(a.out)[row * D + d] = __float2bfloat16_rn(o);
            } else {
                a.ws_o[(row * a.max_parts + it.part) * D + d] = o;
                if (d == 0) a.ws_lse[row * a.max_parts + it.part] = (L > 0.f) ? M + lg2(L) : -INFINITY;
            }
        }
        __syncthreads();
    }
}

// One warp per (sequence, query head): log-sum-exp merge of the partials of
// sequences with more than one partition; zero rows for empty sequences.
template <int D>
__global__ void __launch_bounds__(128) merge_kernel(const DecodeArgs a) {
    constexpr int E = D / 32;  // dims per lane
    const int b = blockIdx.x, h = blockIdx.y * 4 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (h >= a.Hq) return;
    int len = a.seq_lens[b];
    if (len < 0 || len > a.max_blocks * 16) len = 0;
    const int P = a.partition_tokens;
    const int nparts = (len + P - 1) / P;
    if (nparts == 1) return;
    const size_t row = (size_t)b * a.Hq + h;
    __nv_bfloat16 *out = static_cast<__nv_bfloat16 *>(a.out) + row * D + lane * E;
    float acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
    if (nparts > 1) {
        const float *lse = a.ws_lse + row * a.max_parts;
        const float *o = a.ws_o + row * a.max_parts * D + lane * E;
        float M = -INFINITY;
        for (int p = lane; p < nparts; p += 32) M = fmaxf(M, lse[p]);
#pragma unroll
        for (int mask = 16; mask >= 1; mask >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, mask));
        float L = 0.f;
        for (int p = 0; p < nparts; ++p) {
            const float lp = lse[p];
            const float wgt = (lp == -INFINITY) ? 0.f : ex2(lp - M);
            L += wgt;
            if constexpr (E == 4) {
                const float4 v = *reinterpret_cast<const float4 *>(o + (size_t)p * D);
                acc[0] += wgt * v.x;
                acc[1] += wgt * v.y;
                acc[2] += wgt * v.z;
                acc[3] += wgt * v.w;
            } else {
                const float2 v = *reinterpret_cast<const float2 *>(o + (size_t)p * D);
                acc[0] += wgt * v.x;
                acc[1] += wgt * v.y;
            }
        }
        const float inv = (L > 0.f) ? 1.f / L : 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] *= inv;
    }
#pragma unroll
    for (int e = 0; e < E; e += 2)
        *reinterpret_cast<__nv_bfloat162 *>(out + e) = __floats2bfloat162_rn(acc[e], acc[e + 1]);
}

template <class C>
cudaError_t run(const DecodeArgs &a, cudaStream_t st) {
    // Opt in to the large dynamic shared-memory carve-out once per device.
    static std::mutex mu;
    static bool ready[64] = {};
    int dev = 0, sms = 0, occ = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!ready[dev]) {
            e = cudaFuncSetAttribute(decode_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)smem_bytes<C>(2048));
            if (e != cudaSuccess) return e;
            ready[dev] = true;
        }
    }
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const size_t smem = smem_bytes<C>(a.B);
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, decode_kernel<C>, C::NT, smem);
    if (e != cudaSuccess) return e;
    if (occ < 1) occ = 1;
    const long long upper = (long long)a.Hkv * a.B * a.max_parts;
    const long long grid = std::min<long long>(upper, (long long)sms * occ);
    if (grid > 0) decode_kernel<C><<<(unsigned)grid, C::NT, smem, st>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    dim3 mgrid(a.B, (a.Hq + 3) / 4);
    merge_kernel<C::D><<<mgrid, 128, 0, st>>>(a);
    return cudaGetLastError();
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

size_t decode_ws_o_bytes(int B, int Hq, int D, int max_parts) {
    const size_t o = (size_t)B * Hq * max_parts * D * sizeof(float);
    return (o + 255) & ~(size_t)255;
}

size_t decode_ws_bytes(int B, int Hq, int D, int max_parts) {
    const size_t lse = (size_t)B * Hq * max_parts * sizeof(float);
    return decode_ws_o_bytes(B, Hq, D, max_parts) + ((lse + 255) & ~(size_t)255);
}

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t st) {
    if (a.D == 128) return a.fp8 ? by_group<128, true>(a, st) : by_group<128, false>(a, st);
    if (a.D == 64) return a.fp8 ? by_group<64, true>(a, st) : by_group<64, false>(a, st);
    return cudaErrorNotSupported;
}

}  // namespace pa
