// prefill.cu -- causal chunked-prefill attention over a paged prefix, on the
// sm_100a tensor cores (tcgen05, TMEM accumulators, TMA tensor copies).
//
// What is computed ("Continuous batching and PagedAttention", How the
// scheduler works: chunked prefill; "Continuous batching and
// PagedAttention: serving many users from one GPU", Prefill gets in the
// way): row i of chunk c sits at position prefix_lens[c] + i and attends,
// per query head, to keys 0 .. prefix_lens[c] + i of its sequence through
// the block table -- the prefix already in the cache and the chunk's own
// keys, written there first.
//
// Design (warp-specialised, two query tiles per CTA):
//  * A query tile is 128 accumulator rows = 128/G positions x the G query
//    heads of one kv head (row = position*G + head), so every K/V tile is
//    fetched once per GQA group.  A CTA holds two query tiles of the same
//    (chunk, kv head) that share every K/V tile.
//  * Warp roles: warps 0-7 and 8-15 are the softmax warpgroups of query
//    tiles 0 and 1 (two threads per accumulator row = TMEM lane, each with
//    half of the row's keys and of its O columns); warp 16 gathers K/V
//    tiles of 128 keys (8 paged blocks) through the block table with 2-D
//    TMA tensor copies (64-column boxes, 128-byte swizzle, no multicast)
//    into rings of K and V slots (an E4M3 cache: warps 16-17 gather the
//    codes and widen them to f16); one lane of the last warp issues the
//    tcgen05 MMAs (kind::f16, fp32 accumulate) and commits them to
//    mbarriers.
//  * Start-up: the first loader thread initialises the barriers, requests
//    the two query tiles (bf16: one 3-D TMA box per 64-column atom, 64
//    columns x G heads x 128/G positions of q) and goes straight on to the
//    block table and the first K tile, without waiting for the other
//    warps, so the query tiles, the table entries and the first K tile are
//    in flight together.  (An E4M3 cache's query rows are loaded and scaled
//    by the softmax warps.)
//  * Per K/V tile j and query tile t: S_t = Q_t K_j^T into TMEM; softmax
//    warpgroup t loads S_t, computes P_t and hands it to O_t += P_t V_j.
//  * bf16 cache: P_t goes to shared memory (128-byte swizzled, the A operand
//    of the P.V MMA), so S_t(j+1) is issued into S_t's TMEM columns as soon
//    as softmax t has loaded S_t(j) ("S free") and the tensor core computes
//    the next scores while the exponentials run; softmax t writes P_t(j)
//    once P_t(j-1).V has completed, which also makes a rescale of its O row
//    in TMEM safe.  K_{j+1} is requested a tile period ahead (2 K slots),
//    V_j once P(j-1).V is done (1 V slot).
//  * E4M3 cache: P_t (f16) is written over the first half of S_t's TMEM
//    columns and O_t += P_t V_j reads it from TMEM; S_t(j+1) is issued only
//    after that P.V has completed.  The MMA warp issues, per tile in turn,
//    P.V as soon as P arrives and then the tile's next S, so a tile never
//    waits for the other tile's softmax.
//  * Softmax applies the causal mask only on tiles that reach past the
//    row's position, moves the running max only when it grows by more than
//    8 (log2 units), and computes P with one packed FMA and one
//    exponential per score (MUFU; kEmuPairs of every 8 pairs can go to the
//    FMA pipe, fastexp.cuh).  The row sum l adds the fp32 probabilities for
//    a bf16 cache and the f16-rounded ones for an E4M3 cache.
//  * Every mbarrier is waited on in phase order and never falls two phases
//    behind its producer (a parity wait cannot tell phase k from k+2); the
//    protocol was checked against that rule, and for deadlock, by a
//    discrete simulation over random schedules.
//  * Key rows past the sequence end in the last V tile are zeroed in shared
//    memory before P.V, so stale cache contents can never reach the output.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "fastexp.cuh"
#include "tc.cuh"

namespace pa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;
// Named barrier that releases the CTA once the barriers are initialised and
// TMEM is allocated (the softmax warps' barriers use ids 1..4*NQ).
constexpr int kStartBar = 15;
// Of every 8 pairs of scores a softmax thread exponentiates, kEmuPairs go
// through the FMA-pipe exponential (fastexp.cuh) and the rest through MUFU:
// with head_dim 128 MUFU alone needs as many clocks per tile as the two
// MMAs of a query tile, which would leave the tensor core waiting.
constexpr int kEmuPairs = 0;

template <int D_, int G_, bool FP8_>
struct PCfg {
    static constexpr int D = D_, G = G_;
    static constexpr bool FP8 = FP8_;             // E4M3 cache: f16 operands, K/V widened by the loader warps
    // bf16 cache: P goes to shared memory and the P.V MMA reads it from
    // there, so S_t(j+1) may be issued into S_t's TMEM columns as soon as
    // the softmax has loaded S_t(j).  E4M3 cache: P is written over S_t's
    // TMEM columns, and S_t(j+1) waits for P_t(j).V_j to complete.
    static constexpr bool PSMEM = !FP8_;
    static constexpr int M = 128;                 // accumulator rows of a query tile
    static constexpr int QPOS = M / G;            // query positions per query tile
    static constexpr int NQ = 2;                  // query tiles per CTA
    static constexpr int KT = 128;                // keys per K/V tile (8 blocks)
    static constexpr int NATOM = D / 64;          // 128-byte column atoms along D
    static constexpr int QATOM = M * 128;         // bytes of one atom column of a query tile
    static constexpr int KATOM = KT * 128;        // bytes of one atom column of a K/V tile
    static constexpr int QTILE = NATOM * QATOM;
    static constexpr int KTILE = NATOM * KATOM;
    // K and V ring depths.  With P in shared memory and head_dim 128 the
    // budget leaves 2 K slots and 1 V slot: K_{j+1} is requested a tile
    // period ahead (the next scores need it early), V_j once P(j-1).V is
    // done (P.V needs it late), so the two copies do not compete for the
    // TMA bandwidth.  (One ring of three slots filled in read order --
    // K_{j+1}, V_j, ... -- requests both early and measured 2.5% slower;
    // two V slots with one P buffer shared by the query tiles, 8% slower.)
    static constexpr int NSK = PSMEM ? (D == 128 ? 2 : 3) : 2;
    static constexpr int NSV = PSMEM ? (D == 128 ? 1 : 3) : 2;
    static constexpr int NPB = PSMEM ? NQ : 0;     // P buffers: one per query tile
    static constexpr int PATOM = M * 128;         // P: one atom column = 64 keys of 128 rows
    static constexpr int PTILE = (KT / 64) * PATOM;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + NQ * QTILE;
    static constexpr int OFF_V = OFF_K + NSK * KTILE;
    static constexpr int OFF_P = OFF_V + NSV * KTILE;
    static constexpr int NSPLIT = 2;              // softmax threads per accumulator row
    static constexpr int SCOL = KT / NSPLIT;      // S columns (keys) per softmax thread
    static constexpr int OCOL = D / NSPLIT;       // O columns per softmax thread
    // E4M3 cache: a K or V tile arrives as KT rows of D codes (row-major, by
    // TMA) in a staging area and is widened there into its f16 slot.  With
    // head_dim 128 the staging area is the slot's own second atom column: the
    // thread that widens row i writes that column's row i exactly over row i
    // of the codes, which it has read first.  With head_dim 64 the slot has
    // one atom column, so the codes get a ring of their own.
    static constexpr int STG_BYTES = KT * D;      // one tile of codes
    static constexpr bool STG_IN_PLACE = FP8 && D == 128;
    static constexpr int OFF_STG = OFF_P + NPB * PTILE;
    static constexpr int STG_RING = (FP8 && !STG_IN_PLACE) ? (NSK + NSV) * STG_BYTES : 0;
    // row max exchange of a row's threads (two parities), and for an E4M3
    // cache the row sums and query magnitudes: fp32.  With P in shared
    // memory the maxima travel as bf16 rounded up (both threads of a row
    // take the same rounded values, so they agree on the row's reference
    // point) and the sums go through the query tile's buffer once O is
    // final (every MMA that read it has completed).
    static constexpr int OFF_X = OFF_STG + STG_RING;
    static constexpr int X_BYTES = PSMEM ? 2 * NQ * NSPLIT * 128 * 2 : 3 * NQ * NSPLIT * 128 * 4;
    static constexpr int OFF_BAR = OFF_X + X_BYTES;
    // K/V full+empty; S full, P full, O done, O final; (P in shared memory)
    // S free; end; (E4M3) K/V codes loaded; (bf16) query tiles loaded
    static constexpr int NBAR = 2 * NSK + 2 * NSV + 4 * NQ + (PSMEM ? NQ : 0) + 1 + (FP8 ? NSK + NSV : 1);
    static constexpr int USED = OFF_BAR + NBAR * 8 + 16;  // + the TMEM address slot
    // the tiles need a 1024-byte aligned base: slack to align it where the
    // budget allows, else the launch requires the base aligned (it is: the
    // dynamic shared memory of a CTA starts on a 1 KB boundary) and checks it
    static constexpr int SLACK = USED + 1024 <= 227 * 1024 ? 1024 : 0;
    static constexpr int SMEM = USED + SLACK;
    static constexpr int NSMW = NQ * 4 * NSPLIT;  // softmax warps
    // loader warps: one TMA warp (bf16 cache), or two warps that gather
    // E4M3 K/V codes and widen them into the operand tiles
    static constexpr int NLOAD = FP8 ? 2 : 1;
    static constexpr int W_LOAD = NSMW, W_MMA = NSMW + NLOAD;
    static constexpr int NT = (NSMW + NLOAD + 1) * 32;
    static constexpr uint32_t FULL_ARRIVALS = FP8 ? NLOAD * 32 : 1;  // arrivals that fill a K or V slot
    // TMEM columns: S_t at t * KT (and for an E4M3 cache P_t in its first
    // KT/2 columns); O_t at COL_O + t * D
    static constexpr uint32_t COL_O = NQ * KT;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t TX_BYTES = KTILE;   // one K or V tile
    static_assert(M % G == 0, "group must divide 128");
    static_assert(COL_O + NQ * D <= TMEM_COLS, "TMEM columns");
    static_assert(SMEM <= 227 * 1024, "shared memory");
    static_assert(SCOL % 64 == 0 && OCOL % 32 == 0, "whole TMEM column groups per thread");
    static_assert(!FP8 || NSK == NSV, "the E4M3 loader fills K and V slots in pairs");
    static_assert(NSPLIT * 128 * 4 <= QTILE, "row sums fit in a query tile's buffer");
};

template <class C>
__global__ void __launch_bounds__(C::NT, 1)
    prefill_kernel(const PrefillArgs a, const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                   const __grid_constant__ CUtensorMap tmQ) {
    constexpr int D = C::D, G = C::G, KT = C::KT, NSK = C::NSK, NSV = C::NSV, NQ = C::NQ;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *sQ = smem + C::OFF_Q;
    uint8_t *sK = smem + C::OFF_K;
    uint8_t *sV = smem + C::OFF_V;
    uint8_t *sP = smem + C::OFF_P;  // P_t (bf16 cache): 128 rows x KT keys, 128-byte swizzle
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *kfull = bars, *kempty = kfull + NSK, *vfull = kempty + NSK, *vempty = vfull + NSV;
    uint64_t *sfull = vempty + NSV, *pfull = sfull + NQ, *odone = pfull + NQ, *ofinal = odone + NQ;
    uint64_t *sfree = ofinal + NQ;                       // P in shared memory: S_t has been read
    uint64_t *mma_done = sfree + (C::PSMEM ? NQ : 0);
    uint64_t *kload = mma_done + 1, *vload = kload + NSK;  // E4M3: the codes of a tile have landed
    uint64_t *qfull = mma_done + 1;                        // bf16: both query tiles have landed
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + C::NBAR);
    // [3][NQ][NSPLIT][128] fp32: max (2 parities), sum; with P in shared
    // memory [2][NQ][NSPLIT][128] bf16 maxima
    float *xch = reinterpret_cast<float *>(smem + C::OFF_X);
    uint16_t *xch16 = reinterpret_cast<uint16_t *>(smem + C::OFF_X);

    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    // CTA -> (chunk c, kv head, query tiles from i0).  CTAs start in the order
    // of their linear index (x fastest); in a causal chunk a later query tile
    // attends more keys, so each chunk's CTAs are taken longest first
    // (query-tile pair descending, kv heads within), which leaves shorter
    // work for the end of the grid.  Shared-prefix mode keeps the grid as is.
    int c = 0, kvh = blockIdx.y, qx = blockIdx.x;
    if (a.shared_len <= 0) {
        const int nx = gridDim.x, lin = blockIdx.x + nx * (blockIdx.y + gridDim.y * blockIdx.z);
        const int rem = lin % (nx * gridDim.y);
        c = lin / (nx * gridDim.y);
        qx = nx - 1 - rem / gridDim.y;
        kvh = rem % gridDim.y;
    }
    const int i0 = qx * (NQ * C::QPOS);
    pdl_trigger();
    pdl_wait();
    if (C::SLACK == 0 && smem != smem_raw) {  // no room to align: the base must be aligned (uniform per launch)
        if (tid == 0) flag_error(a.err, PA_DEVERR_LAYOUT);
        return;
    }
    const uint64_t deadline = wait_deadline();  // shared by every wait of this launch
    // causal chunk: rows are positions pfx + i, keys [0, pfx + i]; shared
    // prefix: rows are sequences, keys [0, shared_len) for every row
    const bool shared = a.shared_len > 0;
    // a shared prefix is split over its keys (grid z): this CTA attends key
    // tiles [jt0, jt1) and writes split-K piece blockIdx.z of its rows
    const int ks = shared ? (int)gridDim.z : 1, kz = shared ? (int)blockIdx.z : 0;
    const int jt0 = shared ? kz * ((a.shared_len + KT - 1) / KT) / ks : 0;
    const int jt1 = shared ? (kz + 1) * ((a.shared_len + KT - 1) / KT) / ks : 0;
    // the loader's first window of 32 block-table entries (lane l: entry
    // jt0 * KT/16 + l), requested together with the chunk's lengths; entries
    // past the sequence's last block are never used
    const int32_t *bt = a.block_tables + (size_t)c * a.max_blocks;
    const int went0 = w == C::W_LOAD ? bt[min(jt0 * (KT / 16) + lane, a.max_blocks - 1)] : 0;
    const int q_start = shared ? 0 : a.cu_q[c];
    const int clen = shared ? a.total_q : a.cu_q[c + 1] - q_start;
    const int pfx = shared ? a.shared_len : a.prefix_lens[c];
    if (i0 >= clen) return;  // this CTA's rows lie past the chunk (uniform per CTA)
    const int L = shared ? pfx : pfx + clen;  // keys of the sequence
    if (clen < 0 || pfx < 0 || L > a.max_blocks * 16 || q_start < 0 || q_start + clen > a.total_q) {
        if (tid == 0) flag_error(a.err, PA_DEVERR_BAD_LEN);
        return;
    }
    const int nalloc = (L + 15) >> 4;  // blocks of the sequence
    if (shared && jt1 <= jt0) {  // more splits than key tiles
        if (tid == 0) flag_error(a.err, PA_DEVERR_BAD_LEN);
        return;
    }
    // K/V tiles each query tile needs (causal: up to its last valid row)
    int ntl[NQ], ntiles = 0;
#pragma unroll
    for (int t = 0; t < NQ; ++t) {
        const int first = i0 + t * C::QPOS;
        const int nv = max(0, min(C::QPOS, clen - first));
        ntl[t] = nv > 0 ? (shared ? jt1 - jt0 : (pfx + first + nv + KT - 1) / KT) : 0;
        ntiles = max(ntiles, ntl[t]);
    }

    if (w == C::W_MMA) tmem_alloc(tmem_slot, C::TMEM_COLS);
    // The first loader thread sets up the barriers, requests the query tiles
    // (bf16) and goes on to the K/V copies without waiting for the other
    // warps (it arrives on the start barrier, they wait there), so the query
    // tiles, the first block-table entries and the first K tile are all in
    // flight at once.
    if (tid == C::W_LOAD * 32) {
        for (int i = 0; i < NSK; ++i) {
            mbar_init(&kfull[i], C::FULL_ARRIVALS);
            mbar_init(&kempty[i], 1);
        }
        for (int i = 0; i < NSV; ++i) {
            mbar_init(&vfull[i], C::FULL_ARRIVALS);
            mbar_init(&vempty[i], 1);
        }
        for (int t = 0; t < NQ; ++t) {
            mbar_init(&sfull[t], 1);
            mbar_init(&pfull[t], 128 * C::NSPLIT);
            mbar_init(&odone[t], 1);
            mbar_init(&ofinal[t], 1);
            if constexpr (C::PSMEM) mbar_init(&sfree[t], 128 * C::NSPLIT);
        }
        mbar_init(mma_done, 1);
        if constexpr (C::FP8)
            for (int i = 0; i < NSK + NSV; ++i) mbar_init(&kload[i], 1);
        else
            mbar_init(qfull, 1);
        fence_mbar_init();
        if constexpr (!C::FP8) {
            // ---- query tiles (bf16): row r of tile t = (position r / G,
            // head r % G) is one 3-D box per 64-column atom (64 columns x G
            // heads x QPOS positions of q, 128-byte swizzle).  Rows past the
            // chunk are read as they stand (zeros past the end of q); they
            // produce rows that are never stored.
            mbar_arrive_expect_tx(qfull, NQ * C::QTILE);
#pragma unroll
            for (int t = 0; t < NQ; ++t)
#pragma unroll
                for (int at = 0; at < C::NATOM; ++at)
                    tma_load_3d(sQ + t * C::QTILE + at * C::QATOM, &tmQ, at * 64, kvh * G, q_start + i0 + t * C::QPOS,
                                qfull);
        }
    }
    // ---- query tiles (E4M3 cache), by the softmax warps: the operands are
    // f16, so each row is scaled by a power of two 2^qexp that puts its
    // largest magnitude in [2^14, 2^15) (exact for every bf16 value in f16's
    // normal range), and 2^-qexp is folded into the row's softmax scale.
    int qexp = 0;
    if (C::FP8 && w < C::NSMW) {
        const int t = w / (4 * C::NSPLIT), half = (w / 4) % C::NSPLIT, r = (w % 4) * 32 + lane;
        const int ip = i0 + t * C::QPOS + r / G;
        const bool valid = ip < clen;
        const __nv_bfloat16 *src =
            static_cast<const __nv_bfloat16 *>(a.q) + ((size_t)(q_start + ip) * a.Hq + (size_t)kvh * G + r % G) * D;
        uint8_t *dst = sQ + t * C::QTILE + r * 128;
        constexpr int NCH = D / 8 / C::NSPLIT;  // 16-byte chunks of the row per thread
        uint4 v[NCH];
#pragma unroll
        for (int k = 0; k < NCH; ++k)
            v[k] = valid ? *reinterpret_cast<const uint4 *>(src + (half + k * C::NSPLIT) * 8) : make_uint4(0, 0, 0, 0);
        if constexpr (C::FP8) {
            float amax = 0.f;
#pragma unroll
            for (int k = 0; k < NCH; ++k) {
                const uint32_t ws[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = bf16x2_to_float2(ws[e]);
                    amax = fmax3(amax, fabsf(f.x), fabsf(f.y));
                }
            }
            float *xq = xch + ((2 * NQ + t) * C::NSPLIT) * 128 + r;  // the sum slots, free until the epilogue
            xq[half * 128] = amax;
            named_bar_sync(1 + t * 4 + (w % 4), 32 * C::NSPLIT);
#pragma unroll
            for (int hh = 0; hh < C::NSPLIT; ++hh) amax = fmaxf(amax, xq[hh * 128]);
            if (amax > 0.f) qexp = min(max(14 - ((int)((__float_as_uint(amax) >> 23) & 0xff) - 127), -60), 60);
            const float qs = __uint_as_float((uint32_t)(127 + qexp) << 23);
#pragma unroll
            for (int k = 0; k < NCH; ++k) {
                const uint32_t ws[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
                uint32_t hw[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = bf16x2_to_float2(ws[e]);
                    const __half2 h = __floats2half2_rn(f.x * qs, f.y * qs);
                    hw[e] = *reinterpret_cast<const uint32_t *>(&h);
                }
                v[k] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
            }
        }
#pragma unroll
        for (int k = 0; k < NCH; ++k) {
            const int ch = half + k * C::NSPLIT, at = ch / 8, cc = ch % 8;
            *reinterpret_cast<uint4 *>(dst + at * C::QATOM + ((cc ^ (r & 7)) * 16)) = v[k];
        }
    }
    uint32_t tmem = 0;
    if (w == C::W_LOAD) {
        __syncwarp();
        named_bar_arrive(kStartBar, C::NT);
    } else {
        fence_proxy_async_smem();
        tc_fence_before();
        named_bar_sync(kStartBar, C::NT);
        tc_fence_after();
        tmem = *tmem_slot;
    }
    // ok turns false at the first wait that runs past the deadline; after
    // that no role issues another wait of the protocol: the loader and the
    // MMA warp stop issuing, the softmax warps only keep their named
    // barriers and arrivals in step (so no thread waits on a partner that has
    // left), and the asynchronous work already issued is drained below.
    // Every lane polls the barrier itself (each lane's accesses are then
    // ordered after its own observation of the phase).  In the loader and
    // MMA warps, whose tensor-core and TMA instructions are issued by single
    // lanes, ok is per lane: a lane past the deadline fails every later wait
    // at once, so all lanes leave their loops within one step of each other.
    // The softmax warps' tcgen05.ld/st are warp-collective, so there ok is
    // made warp-uniform by a vote once per tile (wait_all).  (A vote after
    // every wait of the MMA and loader warps measured 7% of the kernel's
    // time; one polling lane with a broadcast, twice as long.)
    bool ok = true;
    auto wait = [&](uint64_t *bar, uint32_t parity) {
        ok = ok && mbar_wait(bar, parity, deadline);
        return ok;
    };
    auto wait_all = [&](uint64_t *bar, uint32_t parity) {
        ok = ok && mbar_wait(bar, parity, deadline);
        ok = __all_sync(0xffffffffu, ok);
        return ok;
    };

    if (C::FP8 && w >= C::W_LOAD && w < C::W_MMA) {
        // ---- E4M3 cache: the first loader warp gathers each K and V tile's
        // codes (8 paged blocks, 2-D TMA boxes of 16 rows x D bytes, no
        // multicast) into the tile's staging area; both loader warps widen
        // the staged rows exactly to f16 into the 128-byte swizzled operand
        // layout (thread ct: rows ct and ct + 64), zero the rows past the
        // sequence end, fence the stores for the tensor core and arrive on
        // the slot's full barrier.  A slot is refilled once the MMAs reading
        // its previous tile have completed (its empty barrier).
        constexpr int BPT = KT / 16;  // blocks per tile
        constexpr int NS = C::NSK;    // K and V slots (as many of each)
        const int ct = tid - C::W_LOAD * 32;
        const bool issuer = w == C::W_LOAD;
        int win0 = jt0 * BPT, went = went0;
        auto stage = [&](int s, int kv) -> uint8_t * {
            if constexpr (C::STG_IN_PLACE) return (kv ? sV : sK) + s * C::KTILE + C::KATOM;
            return smem + C::OFF_STG + (2 * s + kv) * C::STG_BYTES;
        };
        auto issue = [&](int j, int kv) {  // issuer warp: TMA of tile j's codes of K (kv 0) or V
            const int s = j % NS, jb = (jt0 + j) * BPT;
            if (jb + BPT > win0 + 32) {
                win0 = jb;
                went = bt[min(win0 + lane, nalloc - 1)];
            }
            int phys = __shfl_sync(0xffffffffu, went, (min(jb + lane % BPT, nalloc - 1) - win0) & 31);
            if (lane < BPT && (phys < 0 || phys >= a.num_blocks)) {
                flag_error(a.err, PA_DEVERR_BAD_BLOCK);
                phys = 0;
            }
            uint64_t *ld = kv ? &vload[s] : &kload[s];
            if (lane == 0) mbar_arrive_expect_tx(ld, C::STG_BYTES);
            __syncwarp();
            if (lane < BPT) tma_load_2d(stage(s, kv) + lane * 16 * D, kv ? &tmV : &tmK, 0, (phys * a.Hkv + kvh) * 16, ld);
            __syncwarp();
        };
        auto widen = [&](int j, int kv) {  // both warps: tile j's staged codes -> f16 operand slot
            const int s = j % NS;
            if (!wait(kv ? &vload[s] : &kload[s], (j / NS) & 1)) return false;
            uint8_t *tile = (kv ? sV : sK) + s * C::KTILE;
            const uint8_t *codes = stage(s, kv);
#pragma unroll
            for (int h = 0; h < KT / 64; ++h) {
                const int i = ct + 64 * h;                      // key row of the tile
                const bool live = (jt0 + j) * KT + i < L;
                uint4 src[D / 16];
#pragma unroll
                for (int u = 0; u < D / 16; ++u)
                    src[u] = live ? *reinterpret_cast<const uint4 *>(codes + i * D + 16 * u) : make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int u = 0; u < D / 16; ++u) {
                    const uint32_t ws[4] = {src[u].x, src[u].y, src[u].z, src[u].w};
                    uint32_t hv[8];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        hv[2 * e] = e4m3x2_to_h2(ws[e]);
                        hv[2 * e + 1] = e4m3x2_to_h2(ws[e] >> 16);
                    }
#pragma unroll
                    for (int hc = 0; hc < 2; ++hc) {  // f16 chunk 2u + hc: 8 elements
                        const int ch = 2 * u + hc, at = ch / 8, cc = ch % 8;
                        *reinterpret_cast<uint4 *>(tile + at * C::KATOM + i * 128 + ((cc ^ (i & 7)) * 16)) =
                            make_uint4(hv[4 * hc], hv[4 * hc + 1], hv[4 * hc + 2], hv[4 * hc + 3]);
                    }
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(kv ? &vfull[s] : &kfull[s]);
            return true;
        };
        int kissued = 0, vissued = 0;  // tiles whose codes were requested
        if (issuer)
            for (int j = 0; j < min(NS, ntiles); ++j) {
                issue(j, 0);
                issue(j, 1);
                kissued = vissued = j + 1;
            }
        for (int j = 0; j < ntiles && ok; ++j) {
            if (!widen(j, 0) || !widen(j, 1)) break;
            // refill the slot of tile j-1 with tile j-1+NS once its MMAs are done
            const int jr = j - 1 + NS;
            if (issuer && j >= 1 && jr < ntiles) {
                if (!wait(&kempty[(j - 1) % NS], ((j - 1) / NS) & 1)) break;
                issue(jr, 0);
                kissued = jr + 1;
                if (!wait(&vempty[(j - 1) % NS], ((j - 1) / NS) & 1)) break;
                issue(jr, 1);
                vissued = jr + 1;
            }
        }
        if (!ok && issuer) {
            // each slot has at most one fill of codes in flight: wait for the
            // last one of every slot, with a short fresh budget
            const uint64_t dd = drain_deadline();
            for (int sl = 0; sl < NS; ++sl) {
                if (kissued > sl) mbar_wait(&kload[sl], ((kissued - 1 - sl) / NS) & 1, dd);
                if (vissued > sl) mbar_wait(&vload[sl], ((vissued - 1 - sl) / NS) & 1, dd);
            }
            __syncwarp();
        }
    } else if (!C::FP8 && w == C::W_LOAD) {
        // ---- producer: K tile j+1, then V tile j, into rings of NSK and NSV
        // slots (K_{j+1} is needed by the next scores while tile j's softmax
        // runs, V_j only by tile j's P.V).  The warp keeps a window of 32
        // block-table entries in registers (lane l holds entry win0 + l),
        // refilled every 32/BPT tiles, so a tile's copies are issued without
        // a global round trip; a tile's row is kept from its K copy for its V.
        constexpr int BPT = KT / 16;  // blocks per tile
        int win0 = jt0 * BPT, went = went0;
        auto tile_row = [&](int jj) {  // lanes 0..BPT-1: cache row of block jj*BPT + lane (tiles in order)
            const int jb = (jt0 + jj) * BPT;
            if (jb + BPT > win0 + 32) {
                win0 = jb;
                went = bt[min(win0 + lane, nalloc - 1)];
            }
            // past the end: the last block, masked later
            int phys = __shfl_sync(0xffffffffu, went, (min(jb + lane % BPT, nalloc - 1) - win0) & 31);
            if (lane < BPT && (phys < 0 || phys >= a.num_blocks)) {
                flag_error(a.err, PA_DEVERR_BAD_BLOCK);
                phys = 0;
            }
            return (phys * a.Hkv + kvh) * 16;
        };
        int kissued = 0, vissued = 0;  // tiles whose K / V copies were issued
        auto fill = [&](int jj, int kv, int row) {  // wait for the slot, then copy tile jj of K (kv 0) or V
            const int ns = kv ? NSV : NSK, sl = jj % ns;
            const uint32_t use = jj / ns;  // how many times the slot was filled before
            if (use > 0 && !wait(kv ? &vempty[sl] : &kempty[sl], (use - 1) & 1)) return false;
            (kv ? vissued : kissued) = jj + 1;
            uint64_t *full = kv ? &vfull[sl] : &kfull[sl];
            if (lane == 0) mbar_arrive_expect_tx(full, C::TX_BYTES);
            __syncwarp();
            if (lane < BPT) {
                uint8_t *dst = (kv ? sV : sK) + sl * C::KTILE + lane * 16 * 128;
#pragma unroll
                for (int at = 0; at < C::NATOM; ++at)
                    tma_load_2d(dst + at * C::KATOM, kv ? &tmV : &tmK, at * 64, row, full);
            }
            __syncwarp();
            return true;
        };
        int row_next = ntiles > 0 ? tile_row(0) : 0;
        if (ntiles > 0) fill(0, 0, row_next);
        for (int j = 0; j < ntiles && ok; ++j) {
            const int row = row_next;
            if (j + 1 < ntiles) {
                row_next = tile_row(j + 1);
                if (!fill(j + 1, 0, row_next)) break;
            }
            if (!fill(j, 1, row)) break;
        }
        if (!ok) {
            // each slot has at most one copy in flight (a slot is refilled only
            // after its previous fill was consumed): wait for the last fill of
            // every slot, with a short fresh budget
            const uint64_t dd = drain_deadline();
            for (int sl = 0; sl < NSK; ++sl)
                if (kissued > sl) mbar_wait(&kfull[sl], ((kissued - 1 - sl) / NSK) & 1, dd);
            for (int sl = 0; sl < NSV; ++sl)
                if (vissued > sl) mbar_wait(&vfull[sl], ((vissued - 1 - sl) / NSV) & 1, dd);
            __syncwarp();
        }
        // the query tiles' copy has landed before the CTA may exit (the MMA
        // warp waits for it before the first scores unless it gave up first)
        if (!mbar_wait(qfull, 0, ok ? deadline : drain_deadline())) ok = false;
        __syncwarp();
    } else if (w == C::W_MMA) {
        constexpr uint32_t idS = idesc_f16kind_f32(128, KT, false, !C::FP8);
        constexpr uint32_t idO = idesc_f16kind_f32(128, D, true, !C::FP8);
        auto issue_s = [&](int t, int ks) {  // S_t from the K tile in ring slot ks
            if (lane == 0) {
                tc_fence_after();
                const uint32_t q0 = smem_addr(sQ + t * C::QTILE), k0 = smem_addr(sK + ks * C::KTILE);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    tc_mma_bf16(tmem + t * KT, smem_desc_sw128(q0 + (kk / 4) * C::QATOM + (kk % 4) * 32, 16, 1024),
                                smem_desc_sw128(k0 + (kk / 4) * C::KATOM + (kk % 4) * 32, 16, 1024), idS, kk > 0);
                tc_commit(&sfull[t]);
            }
            __syncwarp();
        };
        auto zero_tail = [&](int j, uint8_t *vt) {  // key rows past the sequence end: zero them before they meet P
            const int kv0 = (jt0 + j) * KT;
            if (!C::FP8 && kv0 + KT > L) {  // (the loader of an E4M3 cache writes those rows as zeros)
                for (int r = max(L - kv0, 0) + lane; r < KT; r += 32)
#pragma unroll
                    for (int at = 0; at < C::NATOM; ++at)
#pragma unroll
                        for (int cc = 0; cc < 8; ++cc)
                            *reinterpret_cast<uint4 *>(vt + at * C::KATOM + r * 128 + cc * 16) = make_uint4(0, 0, 0, 0);
                fence_proxy_async_smem();
                __syncwarp();
            }
        };
        if (ntiles > 0 && (C::FP8 || wait(qfull, 0)) && wait(&kfull[0], 0)) {
#pragma unroll
            for (int t = 0; t < NQ; ++t)
                if (ntl[t] > 0) issue_s(t, 0);
            if (lane == 0) tc_commit(&kempty[0]);
            __syncwarp();
        }
        if constexpr (C::PSMEM) {
            // ---- MMA issue with P in shared memory, per K/V tile j: first the
            // next scores S_t(j+1) = Q_t K_{j+1}^T, each as soon as softmax t has
            // loaded S_t(j) (S free); then O_t += P_t(j) V_j as P_t(j) arrives
            // The tensor core computes tile j+1's scores while tile j's
            // exponentials run.
            for (int j = 0; j < ntiles && ok; ++j) {
                const int jn = j + 1;
                if (jn < ntiles) {
                    const int sn = jn % NSK;
                    if (!wait(&kfull[sn], (jn / NSK) & 1)) break;
#pragma unroll
                    for (int t = 0; t < NQ; ++t)
                        if (jn < ntl[t]) {
                            if (!wait(&sfree[t], j & 1)) break;  // S_t(j) is in softmax t's registers
                            issue_s(t, sn);
                        }
                    if (!ok) break;
                    if (lane == 0) tc_commit(&kempty[sn]);  // after both S(j+1)
                    __syncwarp();
                }
                const int s = j % NSV;
                if (!wait(&vfull[s], (j / NSV) & 1)) break;
                zero_tail(j, sV + s * C::KTILE);
#pragma unroll
                for (int t = 0; t < NQ; ++t)
                    if (j < ntl[t]) {
                        if (!wait(&pfull[t], j & 1)) break;  // P_t(j) is in shared memory
                        if (lane == 0) {
                            tc_fence_after();
                            const uint32_t p0 = smem_addr(sP + t * C::PTILE), v0 = smem_addr(sV + s * C::KTILE);
#pragma unroll
                            for (int kk = 0; kk < KT / 16; ++kk)
                                tc_mma_bf16(tmem + C::COL_O + t * D,
                                            smem_desc_sw128(p0 + (kk / 4) * C::PATOM + (kk % 4) * 32, 16, 1024),
                                            smem_desc_sw128(v0 + kk * 16 * 128, C::KATOM, 1024), idO, j > 0 || kk > 0);
                            tc_commit(&odone[t]);
                            if (j == ntl[t] - 1) tc_commit(&ofinal[t]);
                        }
                        __syncwarp();
                    }
                if (!ok) break;
                if (lane == 0) tc_commit(&vempty[s]);
                __syncwarp();
            }
        } else {
            // ---- MMA issue with P in TMEM (E4M3 cache), software-pipelined
            // per query tile: O_t += P_t(j) V_j as soon as softmax t hands over
            // P_t(j), then S_t(j+1) = Q_t K_{j+1}^T as soon as that P.V has
            // completed (S_t(j+1) overwrites P_t).  Tile 0's next scores never
            // wait for tile 1's softmax, and tile 1 stays half a step behind
            // tile 0, so the two softmaxes use MUFU in turns.
            constexpr int NS = NSK;
            for (int j = 0; j < ntiles && ok; ++j) {
                const int s = j % NS, jn = j + 1, sn = jn % NS;
                if (!wait(&vfull[s], (j / NS) & 1)) break;
                zero_tail(j, sV + s * C::KTILE);
                bool kready = false;  // K tile j+1 has landed
#pragma unroll
                for (int t = 0; t < NQ; ++t) {
                    if (j < ntl[t]) {
                        if (!wait(&pfull[t], j & 1)) break;  // P_t(j) is in TMEM
                        if (lane == 0) {
                            tc_fence_after();
                            const uint32_t v0 = smem_addr(sV + s * C::KTILE);
#pragma unroll
                            for (int kk = 0; kk < KT / 16; ++kk)
                                tc_mma_bf16_tmem_a(tmem + C::COL_O + t * D, tmem + t * KT + kk * 8,
                                                   smem_desc_sw128(v0 + kk * 16 * 128, C::KATOM, 1024), idO,
                                                   j > 0 || kk > 0);
                            tc_commit(&odone[t]);
                            if (j == ntl[t] - 1) tc_commit(&ofinal[t]);
                        }
                        __syncwarp();
                    }
                    if (jn < ntl[t]) {
                        if (!kready) {
                            if (!wait(&kfull[sn], (jn / NS) & 1)) break;
                            kready = true;
                        }
                        if (!wait(&odone[t], j & 1)) break;  // P_t(j) consumed
                        issue_s(t, sn);
                    }
                }
                if (!ok) break;
                if (lane == 0) tc_commit(&vempty[s]);
                __syncwarp();
                if (jn < ntiles) {
                    if (!kready && !wait(&kfull[sn], (jn / NS) & 1)) break;
                    if (lane == 0) tc_commit(&kempty[sn]);  // after every S(j+1) above
                    __syncwarp();
                }
            }
        }
        // every MMA of this CTA has completed before TMEM is released (after
        // a failure: with a short fresh budget)
        if (lane == 0) tc_commit(mma_done);
        __syncwarp();
        const bool done = mbar_wait(mma_done, 0, ok ? deadline : drain_deadline());
        ok = __all_sync(0xffffffffu, ok && done);
    } else {
        // ---- softmax of query tile t: NSPLIT threads per accumulator row,
        // each with SCOL of the row's keys and OCOL of its O columns
        constexpr int NSP = C::NSPLIT, SCOL = C::SCOL, OCOL = C::OCOL;
        const int t = w / (4 * NSP), half = (w / 4) % NSP, r = (w % 4) * 32 + lane;
        const int bar_id = 1 + t * 4 + (w % 4);  // named barrier of the NSP warps sharing these rows
        const int ip = i0 + t * C::QPOS + r / G;
        const bool row_valid = ip < clen;
        const int pos = shared ? pfx - 1 : pfx + ip;  // last key the row attends
        // log2 units; an E4M3 row also undoes its query scale 2^qexp
        const float sl2 = a.scale * kLog2e * (a.k_scale ? a.k_scale[kvh] : 1.f) *
                          __uint_as_float((uint32_t)(127 - qexp) << 23);
        const uint32_t lane_base = tmem + ((uint32_t)((w & 3) * 32) << 16);
        const uint32_t scol = t * KT + half * SCOL;            // this thread's S columns
        const uint32_t pcol = t * KT + half * (SCOL / 2);      // its P words (two bf16 each)
        const uint32_t ocol = C::COL_O + t * D + half * OCOL;  // its O columns
        auto xslot = [&](int k, int hh) { return xch + ((k * NQ + t) * NSP + hh) * 128 + r; };
        float m = -INFINITY, l = 0.f;
        for (int j = 0; j < ntl[t]; ++j) {
            // after a failed wait this thread issues no further wait and
            // touches no TMEM, but still meets its partner warp at every named
            // barrier and arrives on P full, so that no thread is left waiting
            // on it
            float sv[SCOL];
            if (wait_all(&sfull[t], j & 1)) {
                tc_fence_after();
#pragma unroll
                for (int q = 0; q < SCOL / 32; ++q) {
                    float t32[32];
                    tmem_ld32(lane_base + scol + 32 * q, t32);
#pragma unroll
                    for (int e = 0; e < 32; ++e) sv[32 * q + e] = t32[e];
                }
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int e = 0; e < SCOL; ++e) sv[e] = -INFINITY;
            }
            if constexpr (C::PSMEM) {  // S_t(j) is in registers: the next scores may overwrite it
                tc_fence_before();
                mbar_arrive(&sfree[t]);
            }
            // raw scores (the scale is positive, so the max commutes with it);
            // the causal mask only where the tile reaches past this row
            const int kv0 = (jt0 + j) * KT + half * SCOL;
            if (!(row_valid && kv0 + SCOL - 1 <= pos)) {
#pragma unroll
                for (int e = 0; e < SCOL; ++e) sv[e] = (row_valid && kv0 + e <= pos) ? sv[e] : -INFINITY;
            }
            float mraw = -INFINITY;
#pragma unroll
            for (int e = 0; e < SCOL; e += 2) mraw = fmax3(mraw, sv[e], sv[e + 1]);
            // the row's max over its threads; after this barrier every thread
            // of the row has read its S columns, so P may overwrite them
            if constexpr (C::PSMEM) {
                // as bf16 rounded up: every thread of the row takes the max of
                // the same rounded values, and it stays >= the true row max
                uint16_t *x = xch16 + ((j & 1) * NQ + t) * NSP * 128 + r;
                x[half * 128] = __bfloat16_as_ushort(__float2bfloat16_ru(mraw));
                named_bar_sync(bar_id, 32 * NSP);
                mraw = -INFINITY;
#pragma unroll
                for (int hh = 0; hh < NSP; ++hh) mraw = fmaxf(mraw, __uint_as_float((uint32_t)x[hh * 128] << 16));
            } else {
                *xslot(j & 1, half) = mraw;
                named_bar_sync(bar_id, 32 * NSP);
#pragma unroll
                for (int hh = 0; hh < NSP; ++hh) mraw = fmaxf(mraw, *xslot(j & 1, hh));
            }
            if (!ok) {
                mbar_arrive(&pfull[t]);
                continue;
            }
            const float mt = mraw * sl2;
            const bool rescale = mt > m + kRescaleThreshold;
            float alpha = 1.f;
            if (rescale) {
                alpha = (m == -INFINITY) ? 0.f : ex2(m - mt);
                m = mt;
                l *= alpha;
            }
            // p = 2^(s*scale*log2e - m): one packed FMA and one MUFU.EX2 per
            // score; masked scores are -inf and give 2^-inf = 0
            const float mb = (m == -INFINITY) ? 0.f : m;
            const float2 sc2 = make_float2(sl2, sl2), nb2 = make_float2(-mb, -mb);
            float2 sum2 = make_float2(0.f, 0.f);
            bool ready = true;  // P in shared memory: P_t(j-1).V_{j-1} has completed
#pragma unroll
            for (int h = 0; h < SCOL / 64; ++h) {
                uint32_t pk[32];
#pragma unroll
                for (int e = 0; e < 64; e += 2) {
                    const float2 x = ffma2(make_float2(sv[64 * h + e], sv[64 * h + e + 1]), sc2, nb2);
                    const float2 pp = ((e / 2) % 8 < kEmuPairs) ? exp2_fma2(x) : make_float2(ex2(x.x), ex2(x.y));
                    if constexpr (!C::FP8) {
                        const __nv_bfloat162 bb = __floats2bfloat162_rn(pp.x, pp.y);
                        pk[e / 2] = *reinterpret_cast<const uint32_t *>(&bb);
                        // the normaliser sums the fp32 probabilities (summing them
                        // as rounded to bf16 cost 3% of the kernel): each weight
                        // of the P.V product is then off by at most 2^-9
                        // relative, within the tolerance
                        sum2 = fadd2(sum2, pp);
                    } else {
                        // f16 P; the normaliser sums it as rounded too.  An f16
                        // moved up 13 bits is an fp32 of the same significand
                        // and 2^-112 times the value (f16 subnormals and zero
                        // included), so the sum is kept scaled by 2^-112 and
                        // scaled back once, in the epilogue
                        const __half2 hh = __floats2half2_rn(pp.x, pp.y);
                        const uint32_t wh = *reinterpret_cast<const uint32_t *>(&hh);
                        pk[e / 2] = wh;
                        sum2 = fadd2(sum2, make_float2(__uint_as_float((wh & 0xffffu) << 13),
                                                       __uint_as_float((wh >> 16) << 13)));
                    }
                }
                if constexpr (C::PSMEM) {
                    // P_t(j) goes where P_t(j-1) was, once its P.V has read it
                    // (that also makes O_t complete up to tile j-1)
                    if (h == 0 && j > 0) ready = wait_all(&odone[t], (j - 1) & 1);
                    if (ready) {
                        uint8_t *prow = sP + t * C::PTILE + ((half * SCOL) / 64 + h) * C::PATOM + r * 128;
#pragma unroll
                        for (int cc = 0; cc < 8; ++cc)
                            *reinterpret_cast<uint4 *>(prow + ((cc ^ (r & 7)) * 16)) =
                                make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
                    }
                } else {
                    tmem_st32_u(lane_base + pcol + 32 * h, pk);  // P over S columns already read
                }
            }
            l += sum2.x + sum2.y;  // this thread's keys; the row sum is combined at the end
            // O_t holds P.V up to tile j-1, complete (P in shared memory: the
            // wait above; else S_t(j) was issued after it): rescale in TMEM;
            // tcgen05.ld/st are warp-collective, so the warp rescales if any of
            // its rows needs it
            if (C::PSMEM) tc_fence_after();
            if (ready && j > 0 && __any_sync(0xffffffffu, rescale)) {
#pragma unroll
                for (int q = 0; q < OCOL / 32; ++q) {
                    float o[32];
                    tmem_ld32(lane_base + ocol + 32 * q, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] *= alpha;
                    tmem_st32(lane_base + ocol + 32 * q, o);
                }
            }
            if constexpr (C::PSMEM) fence_proxy_async_smem();  // P stores -> the tensor core
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&pfull[t]);
        }
        if (ntl[t] > 0) {
            // ---- epilogue: O / l, as bf16 output rows (or as split-K piece kz).
            // The row sum over its threads: with P in shared memory through
            // Q_t's buffer, which is free once O_t is final
            bool fin;
            if constexpr (C::PSMEM) {
                fin = wait_all(&ofinal[t], 0);
                float *xs = reinterpret_cast<float *>(sQ + t * C::QTILE) + r;
                xs[half * 128] = l;
                named_bar_sync(bar_id, 32 * NSP);
                l = 0.f;
#pragma unroll
                for (int hh = 0; hh < NSP; ++hh) l += xs[hh * 128];
            } else {
                *xslot(2, half) = l;
                named_bar_sync(bar_id, 32 * NSP);
                l = 0.f;
#pragma unroll
                for (int hh = 0; hh < NSP; ++hh) l += *xslot(2, hh);
                if constexpr (C::FP8) l *= 0x1p112f;  // the f16 sum was kept scaled by 2^-112
                fin = wait_all(&ofinal[t], 0);
            }
            if (fin) {
                tc_fence_after();
                const size_t grow = (size_t)(q_start + ip) * a.Hq + (size_t)kvh * G + r % G;  // q / out row
                __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(a.out) + grow * D + half * OCOL;
                const float inv = (l > 0.f) ? 1.f / l : 0.f;
                const float vs = a.v_scale ? a.v_scale[kvh] : 1.f;  // E4M3 V scale (1 for bf16)
                if (shared) {
                    // split-K piece kz of the row: normalised fp32 output and log2-sum-exp
                    float *wo = a.ws_o + (grow * a.max_parts + kz) * D + half * OCOL;
#pragma unroll
                    for (int q = 0; q < OCOL / 32; ++q) {
                        float o[32];
                        tmem_ld32(lane_base + ocol + 32 * q, o);
                        tmem_wait_ld();
                        if (row_valid) {
#pragma unroll
                            for (int e = 0; e < 32; e += 4)
                                *reinterpret_cast<float4 *>(wo + 32 * q + e) =
                                    make_float4(o[e] * inv * vs, o[e + 1] * inv * vs, o[e + 2] * inv * vs,
                                                o[e + 3] * inv * vs);
                        }
                    }
                    if (row_valid && half == 0) a.ws_lse[grow * a.max_parts + kz] = (l > 0.f) ? m + lg2(l) : -INFINITY;
                } else {
#pragma unroll
                    for (int q = 0; q < OCOL / 32; ++q) {
                        float o[32];
                        tmem_ld32(lane_base + ocol + 32 * q, o);
                        tmem_wait_ld();
                        if (row_valid) {
#pragma unroll
                            for (int e = 0; e < 32; e += 8) {
                                uint32_t wds[4];
#pragma unroll
                                for (int u = 0; u < 4; ++u) {
                                    const __nv_bfloat162 bb =
                                        __floats2bfloat162_rn(o[e + 2 * u] * inv * vs, o[e + 2 * u + 1] * inv * vs);
                                    wds[u] = *reinterpret_cast<const uint32_t *>(&bb);
                                }
                                *reinterpret_cast<uint4 *>(dst + 32 * q + e) =
                                    make_uint4(wds[0], wds[1], wds[2], wds[3]);
                            }
                        }
                    }
                }
            }  // O final
        }
    }
    if (!ok && lane == 0) flag_error(a.err, PA_DEVERR_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (w == C::W_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// ---- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// The cache seen as a 2-D bf16 tensor [num_blocks*Hkv*16 rows][D]; a box is
// 16 rows (one block of one kv head) x 64 columns, 128-byte swizzled.
bool cache_map(CUtensorMap *map, const void *base, int64_t rows, int D) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64, 16};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// An E4M3 cache seen as a 2-D byte tensor [num_blocks*Hkv*16 rows][D]; a box
// is 16 rows (one block of one kv head) x D bytes, unswizzled (rows land
// row-major in the staging area).
bool code_map(CUtensorMap *map, const void *base, int64_t rows, int D) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)D};
    const cuuint32_t box[2] = {(cuuint32_t)D, 16};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// q [total_q][Hq][D] bf16 seen as a 3-D tensor (D, Hq, total_q); a box is
// 64 columns x G heads x 128/G positions = the 128 rows of one atom column
// of a query tile (row = position * G + head), 128-byte swizzled.
bool query_map(CUtensorMap *map, const void *base, int total_q, int Hq, int D, int G) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hq, (cuuint64_t)total_q};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hq * D * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)G, (cuuint32_t)(128 / G)};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <class C>
cudaError_t run_prefill(const PrefillArgs &a, cudaStream_t st) {
    static std::mutex mu;
    static bool ready[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!ready[dev]) {
            e = cudaFuncSetAttribute(prefill_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
            if (e != cudaSuccess) return e;
            ready[dev] = true;
        }
    }
    CUtensorMap tk, tv, tq = {};
    const int64_t rows = a.num_blocks * a.Hkv * 16;
    auto map = C::FP8 ? code_map : cache_map;
    if (!map(&tk, a.k_cache, rows, C::D) || !map(&tv, a.v_cache, rows, C::D)) return cudaErrorInvalidValue;
    // (an E4M3 cache takes the query rows through registers, to scale them)
    if (!C::FP8 && !query_map(&tq, a.q, a.total_q, a.Hq, C::D, C::G)) return cudaErrorInvalidValue;
    dim3 grid((a.max_q_len + C::NQ * C::QPOS - 1) / (C::NQ * C::QPOS), a.Hkv,
              a.shared_len > 0 ? std::max(a.key_splits, 1) : a.n_chunks);
    return launch_pdl(prefill_kernel<C>, grid, dim3(C::NT), C::SMEM, st, a, tk, tv, tq);
}

template <int D, bool FP8>
cudaError_t prefill_by_group(const PrefillArgs &a, cudaStream_t st) {
    switch (a.Hq / a.Hkv) {
        case 1: return run_prefill<PCfg<D, 1, FP8>>(a, st);
        case 2: return run_prefill<PCfg<D, 2, FP8>>(a, st);
        case 4: return run_prefill<PCfg<D, 4, FP8>>(a, st);
        case 8: return run_prefill<PCfg<D, 8, FP8>>(a, st);
        default: return cudaErrorNotSupported;
    }
}

}  // namespace

cudaError_t launch_prefill(const PrefillArgs &a, cudaStream_t st) {
    if (a.fp8 && (!a.k_scale || !a.v_scale)) return cudaErrorInvalidValue;
    if (a.D == 128) return a.fp8 ? prefill_by_group<128, true>(a, st) : prefill_by_group<128, false>(a, st);
    if (a.D == 64) return a.fp8 ? prefill_by_group<64, true>(a, st) : prefill_by_group<64, false>(a, st);
    return cudaErrorNotSupported;
}

}  // namespace pa
