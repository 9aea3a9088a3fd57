// ripe_persist_sm100.cu -- the all-depths verify of one layer (k draft tokens of
// each listed sequence at every loop depth 1..R) as one persistent sm_100a kernel.
//
// What is computed (RIPE abstract, sentence introducing RIPE): row (token j,
// depth r) of sequence b attends to positions [0, A) at the deepest plane R, to
// the window positions [A, T) at plane r, and to draft tokens 0..j at plane r,
// with A = min(ws_b, T).  The deep region [0, A) is the same for all k*R rows of a
// sequence, so it is one stacked-query contraction on the tensor cores; each
// (depth, 8-token) slice of rows has its own window and block keys.
//
// Work items, spread over one wave of CTAs (one CTA per SM):
//   deep item (sequence g, head h, chunk c): keys [c*chunk, (c+1)*chunk) of the
//     deep region for all k*R rows (the last chunk runs to the region's end).
//     S = Q K^T (tcgen05.mma, fp32 in TMEM), online
//     softmax on CUDA cores, O += P V (tcgen05.mma, P read from TMEM); K, V by TMA
//     through ST shared-memory stages.  Warps 0-3 own TMEM lanes (one row each),
//     warp 4 lane 0 issues TMA, warp 5 allocates TMEM and its lane 0 issues MMAs.
//     The first `pd` CTAs take deep items pd apart.
//   window unit (g, h, r, 8-token slice q): the window keys at plane r (ring
//     slots, or deep-plane rows for r = R) and the slice's draft-block keys, then
//     S^T = K Q^T and O^T = V^T P^T on warp-level MMA tiles (m16n8k16: keys and
//     channels on the 16-row side, the <= 8 query rows on the 8-column side).
//     Every CTA takes a contiguous range of units: n_lo per deep CTA, n_hi per
//     other CTA (the host balances the work).  Two forms:
//     * stage ring (every unit one chunk of KC keys, no sliding window): producer
//       warps load units in order into a ring of shared-memory stages (the whole
//       ring plane by one Wcap-row tensor box per column chunk, the draft tokens by
//       16-byte copies); consumer warps (the deep warps too, once their items are
//       done) take tickets, compute, free the stage and publish.  A consumer loads
//       the queries of its next unit into registers while it computes this one.
//     * per-warp stages (otherwise): each warp runs its units one chunk at a time
//       through its own stage (8-row boxes where eight window keys sit together in
//       memory, copies for the rest).
//
// No merging here: every deep item and window unit writes its partial result (m
// in log2 units, l, unnormalised o) to scratch -- segment c of its rows for deep
// chunk c, segment nsplit for the window -- and the merge kernel launched after
// this one (programmatic dependent launch) combines each row's segments in fixed
// order: M = max m, L = sum l 2^(m-M), O = sum o 2^(m-M) / L, and the LSE.  No CTA
// ever waits for another; global round trips under full memory load cost
// microseconds, so the kernel makes none on its critical paths.
#include <cuda.h>

#include <cstring>

#include "ripe_launch.h"
#include "ripe_verify.cuh"
#include "sm100_ptx.cuh"

namespace {

constexpr int kN = 64;           // deep keys per tile
constexpr int kDeepWarps = 6;    // warps 0-3 softmax, 4 TMA, 5 MMA
constexpr int kWR = 8;           // rows per window unit (the N of an m16n8k16 tile)
constexpr int kMaxItems = 32;    // deep items per CTA

// Tensor maps: deep K, V in 64-row boxes (deep region); ring K, V and deep K, V in
// 8-row boxes (window chunks); Q of this call as [rows][H][d] in 128-row boxes of
// one head.  All 32 columns wide with the 64-byte swizzle.
struct PMaps {
    CUtensorMap dk, dv, wk, wv, rk, rv, q;
    CUtensorMap wkf, wvf, rkf, rvf;  // ring / deep planes in boxes of Wcap rows (a whole ring plane)
};

struct DeepItem {
    int g, h, c, seq, kb, ke, E, ntiles, fb, fp;  // fb, fp: fork parent and position
};

// Scalars of a launch beyond the common verify arguments.
struct PArgs {
    int pd;            // CTAs that take deep items
    int n_lo, n_hi;    // window units per deep CTA / per other CTA
    int ndeep;         // G * H * nsplit deep items
    int nunits;        // G * H * R * ceil(k / 8) window units
    // Test hook: when nonzero, the softmax warps of every deep CTA first wait, this
    // many clock cycles at most, on a barrier nothing signals, so that the bounded
    // wait runs out (RIPE_DEVERR_TIMEOUT) and the abort path runs.
    long long probe_cycles;
    // Per-query sliding window (RIPE abstract, fifth sentence, read per query):
    // draft token j at position T + j reads positions T+j-W+1 .. T+j at its own
    // depth, older ones at plane R; 0 = the store's window for every row.
    int sliding;
    int full_box;  // the Wcap-row maps are valid (Wcap <= 256)
};

template <int D, int MT, int ST, int NWW, int KC>
struct PLayout {
    static constexpr int NCH = D / 32;
    static constexpr bool QT = MT == 1;  // Q of the deep region in TMEM (one M tile) or shared memory
    static constexpr int Q_BYTES = QT ? 0 : MT * NCH * 8192;
    static constexpr int KV_STAGE = NCH * 4096;  // 64 keys x 64 B per column chunk
    static constexpr int KCB = KC * 64;          // one column chunk of a window chunk
    static constexpr int WSTAGE = 2 * NCH * KCB;  // K chunks, then V chunks
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + Q_BYTES;
    static constexpr int OFF_V = OFF_K + ST * KV_STAGE;
    static constexpr int OFF_W = OFF_V + ST * KV_STAGE;
    static constexpr int THREADS = 32 * (kDeepWarps + NWW);
    static constexpr int NWARPS = THREADS / 32;
    static constexpr int OST_BYTES = 4 * 8 * (32 * 4 + 16);
    // q_full, k_full[ST], v_full[ST], kv_empty[ST], s_full[2], p_full[2], pv_done[2], drain, epi_done, probe
    static constexpr int NBAR = 1 + 3 * ST + 9;
    static constexpr int DESC_BYTES = 96;
    static constexpr int ITEM_BYTES = (kMaxItems * (int)sizeof(DeepItem) + 15) / 16 * 16;
    // What follows the stage region: softmax staging, barriers, flags, tables.
    static constexpr int TAIL = OST_BYTES + NBAR * 8 + 2 * NWARPS * 8 + 64 + ITEM_BYTES + NWARPS * DESC_BYTES +
                                NWARPS * 4 + NWARPS + 64;
    static constexpr int SMEM_CAP = 232448;  // 227 KB per CTA
    // The stage region takes the rest of the budget: the deep stages, then window
    // stages of a deep CTA; a CTA without deep items puts window stages everywhere.
    static constexpr int OFF_WEND = (SMEM_CAP - 1024 - TAIL) / 1024 * 1024;
    static constexpr int NS_DEEP_RAW = (OFF_WEND - OFF_W) / WSTAGE;
    static constexpr int NS_DEEP = NS_DEEP_RAW < NWARPS ? NS_DEEP_RAW : NWARPS;  // window stages of a deep CTA
    static constexpr int NW_FULL = (OFF_WEND / WSTAGE) < NWARPS ? (OFF_WEND / WSTAGE) : NWARPS;
    static constexpr int OFF_OST = OFF_WEND;  // epilogue staging of the softmax warps
    static constexpr int OFF_BAR = OFF_OST + OST_BYTES;
    // Window stage barriers: one per warp (full), then one per warp (empty, stage ring).
    static constexpr int OFF_WBAR = OFF_BAR + NBAR * 8;
    static constexpr int OFF_MISC = OFF_WBAR + 2 * NWARPS * 8;
    static constexpr int OFF_ITEMS = OFF_MISC + 64;
    // Stage ring: the unit held by each stage.
    static constexpr int OFF_DESC = OFF_ITEMS + ITEM_BYTES;
    // Stage ring: the ticket last issued into each stage.
    static constexpr int OFF_ISS = OFF_DESC + NWARPS * DESC_BYTES;
    // Stage ring: whether a stage's last use wrote window rows by 16-byte copies.
    static constexpr int OFF_DIRTY = OFF_ISS + NWARPS * 4;
    static constexpr int BYTES = OFF_DIRTY + NWARPS;
    static constexpr int SMEM = BYTES + 1024;
    static_assert(NS_DEEP >= 1, "a deep CTA needs a window stage");
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t S_COL(int mt, int sb) { return (uint32_t)((mt * 2 + sb) * kN); }
    static constexpr uint32_t O_COL(int mt) { return (uint32_t)(MT * 2 * kN + mt * 128); }
    static constexpr uint32_t Q_COL = 2 * kN + 128;
    static_assert(WSTAGE % 1024 == 0 && KV_STAGE % 1024 == 0 && Q_BYTES % 1024 == 0, "stage alignment");
    static_assert(KC % 16 == 0 && KC <= 80, "window chunk");
};

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int32_t* err) {
    const bool ok = sm100::mbar_wait(bar, parity, abort, err);
    return __all_sync(0xffffffffu, ok);
}

// Named barrier over the four softmax warps (ids 0 is __syncthreads).
__device__ __forceinline__ void softmax_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Context of sequence slot g of an all-depths call: its id, committed length T,
// deep-region length A and the number E of partial segments of each of its rows
// (deep chunks with keys, plus the window); ok is false for an id outside the
// store (reported once).
struct GroupCtx {
    int seq, T, A, E, fb, fp;  // fb, fp: deep positions below fp are read from sequence fb
    bool ok;
};

__device__ __forceinline__ GroupCtx group_ctx(const VerifyArgs& a, int g, bool report) {
    GroupCtx c;
    c.seq = a.ba.seq_ids[g];
    c.ok = c.seq >= 0 && c.seq < a.s.Bmax;
    if (!c.ok) {
        if (report) set_device_error(a.s.err, RIPE_DEVERR_SEQ_RANGE);
        c.T = c.A = 0;
        c.E = 1;
        c.fb = c.fp = 0;
        return c;
    }
    c.T = context_length(a.s.len, a.ctx, a.s.err, c.seq, report);
    c.A = min(a.s.ws[c.seq], c.T);
    c.E = deep_splits_used(c.A, a.chunk, a.nsplit) + 1;
    c.fp = a.s.fpos[c.seq];
    c.fb = c.fp > 0 ? a.s.fbase[c.seq] : c.seq;
    return c;
}

// Visibility to row (token) j, under the sliding window, of a window unit's key
// that follows its window keys: e counts from the first such key; nblk draft
// tokens at plane r, then ndw window positions A + e at plane R, then nbr draft
// tokens at plane R.  sbase = T - W + 1 - A is row 0's first plane-r position,
// minus A.
__device__ __forceinline__ bool slide_visible(int e, int j, int nblk, int ndw, int nbr, int sbase, int W) {
    if (e < nblk) return e <= j && e >= j - W + 1;        // draft token e at plane r
    e -= nblk;
    if (e < ndw) return e < sbase + j;                    // window position A + e at plane R
    e -= ndw;
    if (e < nbr) return e < j - W + 1;                    // draft token e at plane R
    return false;
}

template <int D, int MT, int ST, int NWW, int KC, bool RING>
__global__ void __launch_bounds__(PLayout<D, MT, ST, NWW, KC>::THREADS, 1)
persist_kernel(const __grid_constant__ PMaps tm, VerifyArgs a, PArgs pa) {
    using Lay = PLayout<D, MT, ST, NWW, KC>;
    using namespace sm100;
    constexpr int NCH = Lay::NCH;
    constexpr uint32_t IDESC_QK = idesc_bf16(128, kN, 0);
    constexpr uint32_t IDESC_PV = idesc_bf16(128, D, 1);

    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = sm + Lay::OFF_Q;
    uint8_t* sK = sm + Lay::OFF_K;
    uint8_t* sV = sm + Lay::OFF_V;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Lay::OFF_BAR);
    uint64_t* q_full = bars;
    uint64_t* k_full = bars + 1;
    uint64_t* v_full = bars + 1 + ST;
    uint64_t* kv_empty = bars + 1 + 2 * ST;
    uint64_t* s_full = bars + 1 + 3 * ST;
    uint64_t* p_full = s_full + 2;
    uint64_t* pv_done = s_full + 4;
    uint64_t* drain = s_full + 6;
    uint64_t* epi_done = s_full + 7;
    uint64_t* probe = s_full + 8;  // never signalled (test hook)
    uint64_t* wbar = reinterpret_cast<uint64_t*>(sm + Lay::OFF_WBAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Lay::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + Lay::OFF_MISC + 4);
    int* n_items_s = reinterpret_cast<int*>(sm + Lay::OFF_MISC + 8);
    // Snapshots of the abort flag for the softmax warps: written by thread 0 before
    // a named barrier, read by all four after it, so that they decide alike even if
    // another role sets the flag in between.
    volatile int* stop_snap = reinterpret_cast<volatile int*>(sm + Lay::OFF_MISC + 12);
    // Next window unit of this CTA's range to hand to a warp that asks for one.
    int* unit_next = reinterpret_cast<int*>(sm + Lay::OFF_MISC + 16);
    DeepItem* items = reinterpret_cast<DeepItem*>(sm + Lay::OFF_ITEMS);

    const StoreView& s = a.s;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int cta = blockIdx.x;
    const bool deep_cta = cta < pa.pd;
    const int R = s.R, H = s.H, k = a.ba.k;
    const int QS = (k + kWR - 1) / kWR;  // 8-token slices per depth
    const int kR = k * R;

    if (threadIdx.x == 0) {
        if (deep_cta) {
            mbar_init(q_full, 128);
            for (int i = 0; i < ST; ++i) {
                mbar_init(k_full + i, 1);
                mbar_init(v_full + i, 1);
                mbar_init(kv_empty + i, 1);
            }
            for (int i = 0; i < 2; ++i) {
                mbar_init(s_full + i, 1);
                mbar_init(p_full + i, 128);
                mbar_init(pv_done + i, 1);
            }
            mbar_init(drain, 1);
            mbar_init(epi_done, 4);
            mbar_init(probe, 1);
        }
        // Window stages: 32 cp.async arrivals (one per lane) + lane 0's expect_tx;
        // the ring's empty barriers: one consumer's arrival.
        for (int i = 0; i < Lay::NWARPS; ++i) {
            mbar_init(wbar + i, 33);
            mbar_init(wbar + Lay::NWARPS + i, 1);
        }
        *reinterpret_cast<int*>(sm + Lay::OFF_MISC + 20) = 0;  // the ring's next ticket
        for (int i = 0; i < Lay::NWARPS; ++i) {
            reinterpret_cast<int*>(sm + Lay::OFF_ISS)[i] = -1;
            sm[Lay::OFF_DIRTY + i] = 0;
        }
        *abort_flag = 0;
        const int64_t ub = cta < pa.pd ? (int64_t)cta * pa.n_lo
                                       : (int64_t)pa.pd * pa.n_lo + (int64_t)(cta - pa.pd) * pa.n_hi;
        *unit_next = (int)(ub < pa.nunits ? ub : pa.nunits);
        fence_barrier_init();
    }
    if (deep_cta && warp == 5) {
        tmem_alloc(tmem_slot, Lay::TMEM_COLS);
        tmem_relinquish();
    }
    if (lane == 0 && warp == 4) {
        prefetch_tmap(&tm.dk);
        prefetch_tmap(&tm.dv);
        prefetch_tmap(&tm.wk);
        prefetch_tmap(&tm.wv);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = deep_cta ? *tmem_slot : 0u;

    // Inputs, metadata and scratch may belong to the previous kernel in the stream.
    grid_dependency_wait();
    grid_launch_dependents();

    // ---- this CTA's deep items: item i = cta + pd * t, decoded as (g, h, c)
    if (deep_cta && warp == 0) {
        const int i = cta + pa.pd * lane;
        DeepItem it{};
        const bool have = lane < kMaxItems && i < pa.ndeep;
        if (have) {
            it.c = i % a.nsplit;
            it.h = (i / a.nsplit) % H;
            it.g = i / (a.nsplit * H);
            const GroupCtx gc = group_ctx(a, it.g, it.h == 0 && it.c == 0);
            it.seq = gc.seq;
            it.E = gc.E;
            it.fb = gc.fb;
            it.fp = gc.fp;
            // The last chunk takes every key past the others, so any deep length is
            // covered whatever the length the host planned for.
            it.kb = it.c * a.chunk;
            it.ke = !gc.ok ? 0 : it.c == a.nsplit - 1 ? gc.A : min(gc.A, it.kb + a.chunk);
            it.ntiles = it.ke > it.kb ? (it.ke - it.kb + kN - 1) / kN : 0;
        }
        // Compact the items that hold keys (empty chunks neither compute nor arrive).
        const unsigned m = __ballot_sync(0xffffffffu, have && it.ntiles > 0);
        if (have && it.ntiles > 0) items[__popc(m & ((1u << lane) - 1))] = it;
        if (lane == 0) *n_items_s = __popc(m);
    }
    __syncthreads();
    const int n_items = deep_cta ? *n_items_s : 0;

    // ======================================================== deep pipeline
    if (deep_cta && warp < kDeepWarps) {
        if (warp == 4) {
            // -------------------------------------------- TMA producer
            if (lane == 0) {
                int it = 0;
                bool ok = true;
                for (int n = 0; n < n_items && ok; ++n) {
                    const DeepItem& di = items[n];
                    // A fork's tiles below its fork position (a multiple of the tile) come
                    // from its parent's deep plane.
                    const int own_base = ((a.layer * s.Bmax + di.seq) * H + di.h) * s.Tmax + di.kb;
                    const int par_base = ((a.layer * s.Bmax + di.fb) * H + di.h) * s.Tmax + di.kb;
                    for (int i = 0; i < di.ntiles; ++i, ++it) {
                        const int st = it % ST;
                        if (it >= ST && !mbar_wait(kv_empty + st, ((it / ST) - 1) & 1, abort_flag, s.err)) {
                            ok = false;
                            break;
                        }
                        const int y = (di.kb + i * kN < di.fp ? par_base : own_base) + i * kN;
                        mbar_expect_tx(k_full + st, Lay::KV_STAGE);
#pragma unroll
                        for (int c = 0; c < NCH; ++c)
                            tma_load_2d(sK + st * Lay::KV_STAGE + c * 4096, &tm.dk, 32 * c, y, k_full + st);
                        mbar_expect_tx(v_full + st, Lay::KV_STAGE);
#pragma unroll
                        for (int c = 0; c < NCH; ++c)
                            tma_load_2d(sV + st * Lay::KV_STAGE + c * 4096, &tm.dv, 32 * c, y, v_full + st);
                    }
                }
                if (*abort_flag) {
                    // Let the copies already issued land before the shared memory goes away.
                    volatile int no_abort = 0;
                    for (int t = it > ST ? it - ST : 0; t < it; ++t) {
                        mbar_wait(k_full + t % ST, (t / ST) & 1, &no_abort, s.err);
                        mbar_wait(v_full + t % ST, (t / ST) & 1, &no_abort, s.err);
                    }
                }
            }
        } else if (warp == 5) {
            // -------------------------------------------- MMA issuer
            if (lane == 0 && n_items > 0) {
                const uint32_t q0 = smem_u32(sQ), k0 = smem_u32(sK), v0 = smem_u32(sV);
                // P V of global tile t (tile ti of its item): P from the S buffer t & 1.
                auto issue_pv = [&](int t, int ti) -> bool {
                    const int st = t % ST, pb = t & 1;
                    if (!mbar_wait(p_full + pb, (t >> 1) & 1, abort_flag, s.err)) return false;
                    if (!mbar_wait(v_full + st, (t / ST) & 1, abort_flag, s.err)) return false;
                    tc_fence_after();
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
                        for (int ks = 0; ks < kN / 16; ++ks) {
                            const uint64_t bd =
                                smem_desc(v0 + st * Lay::KV_STAGE + ks * 1024, kN * 64, 512, kLayoutSwizzle64B);
                            mma_bf16_ts(tmem + Lay::O_COL(mt), tmem + Lay::S_COL(mt, pb) + ks * 8, bd, IDESC_PV,
                                        (ti > 0 || ks > 0) ? 1u : 0u);
                        }
                    }
                    mma_commit(kv_empty + st);
                    mma_commit(pv_done + pb);
                    return true;
                };
                bool ok = true;
                int it = 0;
                for (int n = 0; n < n_items && ok; ++n) {
                    const int ntiles = items[n].ntiles;
                    // Q of this item is in place (the previous item's epilogue is done with O).
                    if (!mbar_wait(q_full, n & 1, abort_flag, s.err)) {
                        ok = false;
                        break;
                    }
                    for (int i = 0; i < ntiles; ++i, ++it) {
                        const int st = it % ST, sb = it & 1;
                        if (!mbar_wait(k_full + st, (it / ST) & 1, abort_flag, s.err)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
#pragma unroll
                        for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
                            for (int ks = 0; ks < D / 16; ++ks) {
                                const uint32_t off = (ks & 1) * 32;
                                const uint64_t bd = smem_desc(k0 + st * Lay::KV_STAGE + (ks >> 1) * 4096 + off, 16,
                                                              512, kLayoutSwizzle64B);
                                if constexpr (Lay::QT) {
                                    mma_bf16_ts(tmem + Lay::S_COL(mt, sb), tmem + Lay::Q_COL + ks * 8, bd, IDESC_QK,
                                                ks > 0 ? 1u : 0u);
                                } else {
                                    const uint64_t ad = smem_desc(q0 + mt * NCH * 8192 + (ks >> 1) * 8192 + off, 16,
                                                                  512, kLayoutSwizzle64B);
                                    mma_bf16(tmem + Lay::S_COL(mt, sb), ad, bd, IDESC_QK, ks > 0 ? 1u : 0u);
                                }
                            }
                        }
                        mma_commit(s_full + sb);
                        if (i > 0 && !(ok = issue_pv(it - 1, i - 1))) break;
                    }
                    if (ok) ok = issue_pv(it - 1, ntiles - 1);
                }
                volatile int no_abort = 0;
                mma_commit(drain);
                mbar_wait(drain, 0, &no_abort, s.err);
            }
        } else {
            // -------------------------------------------- softmax + epilogue (warps 0-3)
            const int t = threadIdx.x;  // TMEM lane = M row within a tile
            const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
            const float c2 = a.scale_log2;
            float m[MT], l[MT];
            bool ok = true;
            int it = 0;
            // A failed wait (timeout or abort) skips the remaining work, but every
            // softmax warp still passes the epilogue's named barriers of this item;
            // the abort flag, set before any of them, ends the loop for all alike.
            for (int n = 0; n < n_items; ++n) {
                const DeepItem di = items[n];
                const int grow0 = di.g * kR;  // first row of the group
                // ---- Q of this item (the previous item's MMAs are done: its epilogue waited for them)
                if constexpr (Lay::QT) {
                    const bool vq = t < kR;
                    const uint4* src = reinterpret_cast<const uint4*>(a.Q + ((int64_t)(grow0 + (vq ? t : 0)) * H + di.h) * D * 2);
#pragma unroll
                    for (int c0 = 0; c0 < D / 2; c0 += 16) {
                        uint32_t w[16];
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            const uint4 x = vq ? __ldg(src + c0 / 4 + v) : make_uint4(0, 0, 0, 0);
                            w[4 * v] = x.x;
                            w[4 * v + 1] = x.y;
                            w[4 * v + 2] = x.z;
                            w[4 * v + 3] = x.w;
                        }
                        tmem_st16(lane_addr + Lay::Q_COL + c0, w);
                    }
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(q_full);
                } else {
                    if (t == 0) {
                        const bool go = n == 0 || mbar_wait(epi_done, (n - 1) & 1, abort_flag, s.err);
                        if (go) {
                            mbar_expect_tx(q_full, MT * NCH * 8192);
#pragma unroll
                            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                                for (int c = 0; c < NCH; ++c)
                                    tma_load_3d(sQ + mt * NCH * 8192 + c * 8192, &tm.q, 32 * c, di.h,
                                                grow0 + mt * 128, q_full);
                        }
                    } else {
                        mbar_arrive(q_full);
                    }
                }
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    m[mt] = -INFINITY;
                    l[mt] = 0.f;
                }
                if (pa.probe_cycles > 0 && n == 0) {
                    const bool got = mbar_wait_slow(probe, 0, abort_flag, s.err, pa.probe_cycles);
                    ok = __all_sync(0xffffffffu, got) && ok;
                }
                for (int i = 0; i < di.ntiles && ok; ++i, ++it) {
                    const int sb = it & 1;
                    if (!warp_wait(s_full + sb, (it >> 1) & 1, abort_flag, s.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int nvalid = min(kN, di.ke - (di.kb + i * kN));
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) {
                        float sc[kN];
                        tmem_ld32(lane_addr + Lay::S_COL(mt, sb), sc);
                        tmem_ld32(lane_addr + Lay::S_COL(mt, sb) + 32, sc + 32);
                        tmem_wait_ld();
                        if (nvalid < kN) {
#pragma unroll
                            for (int c = 0; c < kN; ++c)
                                if (c >= nvalid) sc[c] = -INFINITY;
                        }
                        float m4[4] = {sc[0], sc[1], sc[2], sc[3]};
#pragma unroll
                        for (int c = 4; c < kN; c += 4) {
                            m4[0] = fmaxf(m4[0], sc[c]);
                            m4[1] = fmaxf(m4[1], sc[c + 1]);
                            m4[2] = fmaxf(m4[2], sc[c + 2]);
                            m4[3] = fmaxf(m4[3], sc[c + 3]);
                        }
                        const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * c2;
                        // The running max moves only when it grows by more than 2^8.
                        float alpha = 1.f;
                        const bool grow = mx > m[mt] + 8.f;
                        if (grow) {
                            const float mn = fmaxf(mx, m[mt]);
                            alpha = ex2(m[mt] - mn);
                            m[mt] = mn;
                        }
                        const float nm = -m[mt];
                        float s4[4] = {0.f, 0.f, 0.f, 0.f};
                        float pw[kN / 2];
#pragma unroll
                        for (int c = 0; c < kN / 2; ++c) {
                            const float x0 = ex2(fmaf(sc[2 * c], c2, nm));
                            const float x1 = ex2(fmaf(sc[2 * c + 1], c2, nm));
                            s4[c & 3] += x0 + x1;
                            pw[c] = __uint_as_float(pack_bf16(x0, x1));
                        }
                        tmem_st32(lane_addr + Lay::S_COL(mt, sb), pw);
                        l[mt] = l[mt] * alpha + ((s4[0] + s4[1]) + (s4[2] + s4[3]));
                        if (i > 0 && __any_sync(0xffffffffu, grow)) {
                            if (!warp_wait(pv_done + ((it - 1) & 1), ((it - 1) >> 1) & 1, abort_flag, s.err)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
#pragma unroll 1
                            for (int c0 = 0; c0 < D; c0 += 32) {
                                float o[32];
                                tmem_ld32(lane_addr + Lay::O_COL(mt) + c0, o);
                                tmem_wait_ld();
#pragma unroll
                                for (int c = 0; c < 32; ++c) o[c] *= alpha;
                                tmem_st32(lane_addr + Lay::O_COL(mt) + c0, o);
                            }
                            tmem_wait_st();
                        }
                    }
                    if (!ok) break;
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(p_full + sb);
                }
                // ---- epilogue of the item: publish every row's partial (segment c);
                // the merge kernel that follows combines the segments.
                if (ok) ok = warp_wait(pv_done + ((it - 1) & 1), ((it - 1) >> 1) & 1, abort_flag, s.err);
                tc_fence_after();
                softmax_bar();
                // 8 rows x 32 columns at a time staged in shared memory, 128-byte pieces.
                {
                    constexpr int OSTR = 32 * 4 + 16;
                    uint8_t* ostage = sm + Lay::OFF_OST + warp * 8 * OSTR;
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) {
                        const int rl = mt * 128 + t;
                        const bool pub = ok && rl < kR;
                        const int64_t pi = pub ? ((int64_t)(grow0 + rl) * H + di.h) * a.nseg + di.c : -1;
                        if (pub) a.part_ml[pi] = make_float2(m[mt], l[mt]);
                        if (!__any_sync(0xffffffffu, pub)) continue;
#pragma unroll 1
                        for (int c0 = 0; c0 < D; c0 += 32) {
                            float o[32];
                            tmem_ld32(lane_addr + Lay::O_COL(mt) + c0, o);
                            tmem_wait_ld();
#pragma unroll
                            for (int part = 0; part < 4; ++part) {
                                if ((lane >> 3) == part) {
                                    float4* d4 = reinterpret_cast<float4*>(ostage + (lane & 7) * OSTR);
#pragma unroll
                                    for (int c = 0; c < 8; ++c)
                                        d4[c] = make_float4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
                                }
                                __syncwarp();
#pragma unroll
                                for (int e0 = 0; e0 < 8 * 8; e0 += 32) {
                                    const int e = e0 + lane, kr = e >> 3, c4 = e & 7;
                                    const int64_t pk = __shfl_sync(0xffffffffu, pi, part * 8 + kr);
                                    if (pk >= 0)
                                        reinterpret_cast<float4*>(a.part_o + pk * D + c0)[c4] =
                                            *reinterpret_cast<const float4*>(ostage + kr * OSTR + c4 * 16);
                                }
                                __syncwarp();
                            }
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                // The epilogue is done with O and (MT = 2) with the Q buffer's staging.
                fence_proxy_async_smem();
                if (lane == 0) mbar_arrive(epi_done);
                if (t == 0) *stop_snap = *abort_flag;
                softmax_bar();  // the flags are rewritten by the next item
                if (*stop_snap) break;
            }
        }
    }

    // ======================================================== window units
    // Two forms (a template parameter).
    // Per-warp stages: deep CTA: warps 6.. start at once with the stages after the
    // deep ones; once the deep items are done (every deep warp at the named barrier
    // below, so no copy or tensor-core read of the deep stages is in flight) the
    // first deep warps join, with stages in the deep region.  Other CTAs: every warp
    // with a stage anywhere in the stage region.  Warps take the CTA's units one at
    // a time from a shared counter.  Each runs a unit one chunk of keys at a time
    // through its own stage; when a unit's last chunk has been read out of the
    // stage, the warp issues the next unit's first chunk and its Q loads, then
    // publishes the unit's partial.
    // Stage ring (every unit one chunk): producer warps (the first window warps)
    // walk the CTA's units in order and load each into the next free stage of a
    // ring; every other warp (the deep warps too, once their items are done) is a
    // consumer that takes the next ticket, waits for that stage, computes, frees the
    // stage at once and only then publishes.
    constexpr int NX = Lay::OFF_W / Lay::WSTAGE < kDeepWarps ? Lay::OFF_W / Lay::WSTAGE : kDeepWarps;
    if (deep_cta && warp < kDeepWarps) asm volatile("bar.sync 2, %0;" ::"n"(32 * kDeepWarps) : "memory");
    const int wfirst = deep_cta ? kDeepWarps : 0;  // the ring's first producer
    const bool win_role = RING ? true : deep_cta ? (warp >= kDeepWarps || warp < NX) : warp < Lay::NW_FULL;
    if (win_role) {
        uint8_t* stage = sm + (deep_cta && warp >= kDeepWarps ? Lay::OFF_W + (warp - kDeepWarps) * Lay::WSTAGE
                                                              : warp * Lay::WSTAGE);
        uint64_t* bar = wbar + warp;
        const uint32_t stage_a = smem_u32(stage);
        const int64_t ub64 = cta < pa.pd ? (int64_t)cta * pa.n_lo
                                         : (int64_t)pa.pd * pa.n_lo + (int64_t)(cta - pa.pd) * pa.n_hi;
        const int64_t ue64 = ub64 + (cta < pa.pd ? pa.n_lo : pa.n_hi);
        const int uend = (int)(ue64 < pa.nunits ? ue64 : pa.nunits);
        constexpr int NKS = D / 16, NMT = D / 16, NT = KC / 16, VPR = NCH * 4;
        const float c2 = a.scale_log2;
        const int q4 = lane & 3, r8 = lane >> 2;
        const int ra = 2 * q4, rb = ra + 1;
        // ldmatrix row addresses in the swizzled layout (K: A operand, rows = keys;
        // V: A operand of O^T by .trans).
        const int rk = (lane & 7) + 8 * ((lane >> 3) & 1), rv = (lane & 7) + 8 * (lane >> 4);
        const uint32_t k_sw0 = (((lane >> 4) + 0) ^ ((rk >> 1) & 3)) << 4;
        const uint32_t k_sw1 = (((lane >> 4) + 2) ^ ((rk >> 1) & 3)) << 4;
        const uint32_t v_sw0 = ((((lane >> 3) & 1) + 0) ^ ((rv >> 1) & 3)) << 4;
        const uint32_t v_sw1 = ((((lane >> 3) & 1) + 2) ^ ((rv >> 1) & 3)) << 4;
        int cached_g = -1;
        GroupCtx gc{};

        // A unit (group g, head h, depth r, slice j0..j0+nr-1) and its keys: nw window
        // positions A.. at plane r (ring) or R (deep rows), nblk draft tokens at plane
        // r, and under the sliding window ndw window positions and nbr draft tokens at
        // plane R.
        // Whole-window units (fast): when the ring plane (Wcap slots) and the unit's
        // other keys fit one chunk, the window keys are the Wcap ring slots in slot
        // order (or Wcap deep rows from A at depth R), loaded by one Wcap-row TMA box
        // per column chunk; koff = Wcap keys then precede the draft tokens.
        // Otherwise koff = nw window keys in position order, 8-row boxes.
        struct Unit {
            int g, h, r, j0, nr, nw, nblk, ndw, nbr, nk, koff, slot0, sbase, E, A, seq, fb, fp;
            bool ring, slide, ok, fast;
        };
        // The rows a unit's partial belongs to.
        struct Slice {
            int g, h, r, j0, nr, E;
        };
        auto describe_at = [&](int g, int h, int r, int q) {
            Unit w;
            w.r = r;
            w.h = h;
            w.g = g;
            if (w.g != cached_g) {
                gc = group_ctx(a, w.g, false);
                cached_g = w.g;
            }
            // The group's segment count for the merge kernel, from its first unit.
            if (h == 0 && r == 1 && q == 0 && lane == 0) a.gE[g] = gc.ok ? gc.E : 0;
            w.ok = gc.ok;
            w.E = gc.E;
            w.A = gc.A;
            w.seq = gc.seq;
            w.j0 = q * kWR;
            w.nr = min(kWR, k - w.j0);
            w.nw = gc.T - gc.A;
            w.nblk = w.j0 + w.nr;
            w.ring = w.r < R;
            // Sliding window (depth r < R only; at depth R both readings agree): row j
            // reads window position p at plane r iff p >= T + j - W + 1, else at plane
            // R, and draft token j' at plane r iff j' >= j - W + 1, else its depth-R row.
            w.slide = pa.sliding && w.ring;
            w.sbase = gc.T - s.W + 1 - gc.A;  // (T + j - W + 1) - A at j = 0
            w.ndw = w.slide ? max(0, min(w.nw, w.sbase + w.j0 + w.nr - 1)) : 0;
            w.nbr = w.slide ? max(0, w.j0 + w.nr - s.W) : 0;
            w.slot0 = gc.A % s.Wcap;
            w.fp = gc.fp;
            w.fb = gc.fb;
            // one Wcap-row box holds the window unless a fork position cuts deep rows
            w.fast = pa.full_box && w.nw <= s.Wcap && s.Wcap + w.nblk + w.ndw + w.nbr <= KC &&
                     (w.ring || !(gc.A < gc.fp && gc.A + s.Wcap > gc.fp));
            w.koff = w.fast ? s.Wcap : w.nw;
            w.nk = w.koff + w.nblk + w.ndw + w.nbr;
            return w;
        };
        auto describe = [&](int u) {
            return describe_at(u / (QS * R * H), (u / (QS * R)) % H, (u / QS) % R + 1, u % QS);
        };
        // The CTA's next unit whose group is valid (warp-uniform).
        auto next_valid = [&](Unit& w) {
            while (true) {
                int u = 0;
                if (lane == 0) u = atomicAdd(unit_next, 1);
                u = __shfl_sync(0xffffffffu, u, 0);
                if (u >= uend) return false;
                w = describe(u);
                if (w.ok) return true;
            }
        };
        // Q^T fragments (B operand): Q[j0 + lane/4][16 ks + 2 q4 ..] and 8 channels on.
        auto load_q = [&](const Unit& w, uint32_t (&b)[NKS][2]) {
            const bool okq = r8 < w.nr;
            const uint32_t* qp = reinterpret_cast<const uint32_t*>(
                a.Q + (okq ? (((int64_t)w.g * kR + (int64_t)(w.j0 + r8) * R + w.r - 1) * H + w.h) * (2 * D) : 0));
#pragma unroll
            for (int ks = 0; ks < NKS; ++ks) {
                b[ks][0] = okq ? __ldg(qp + 8 * ks + q4) : 0u;
                b[ks][1] = okq ? __ldg(qp + 8 * ks + 4 + q4) : 0u;
            }
        };
        // Keys [k0, k0 + 16 nt) of unit w into the stage: 8-key groups of window keys
        // contiguous in memory by TMA (lane 0), the rest (a group that wraps the ring,
        // a partial group, draft tokens, plane-R keys of the sliding window, zero fill)
        // by 16-byte copies.  The stage's earlier reads are done (caller's __syncwarp).
        auto issue = [&](const Unit& w, int k0, uint8_t* stage, uint64_t* bar) {
            const int nt = (min(KC, w.nk - k0) + 15) / 16;
            const int64_t grow0 = (int64_t)w.g * kR;
            // Rows of ring plane r (slot 0) and of the deep plane (position 0; deep_yp:
            // the fork parent's) in the tensor maps' 2-D views.
            const int64_t ring_y = ((((int64_t)a.layer * s.Bmax + w.seq) * H + w.h) * (R - 1) + (w.r - 1)) * s.Wcap;
            const int64_t deep_y = (((int64_t)a.layer * s.Bmax + w.seq) * H + w.h) * s.Tmax;
            const int64_t deep_yp = (((int64_t)a.layer * s.Bmax + w.fb) * H + w.h) * s.Tmax;
            fence_proxy_async_smem();
            // Source of key kk's 16-byte vector v, for the keys that go by copy.
            auto key_src = [&](int kk, int v, const char*& ks_, const char*& vs_) -> bool {
                int64_t off = v * 16;
                if (kk < w.koff) {  // window key (position order: the chunked form)
                    const int pos = w.A + kk;
                    off += (w.ring ? ring_y + (w.slot0 + kk) % s.Wcap : (pos < w.fp ? deep_yp : deep_y) + pos) *
                           (2 * D);
                    ks_ = (w.ring ? s.kwin : s.kdeep) + off;
                    vs_ = (w.ring ? s.vwin : s.vdeep) + off;
                    return true;
                }
                int e = kk - w.koff;
                if (e < w.nblk) {  // draft token e at plane r
                    off += ((grow0 + (int64_t)e * R + w.r - 1) * H + w.h) * (2 * D);
                    ks_ = a.Kb + off;
                    vs_ = a.Vb + off;
                    return true;
                }
                e -= w.nblk;
                if (e < w.ndw) {  // sliding: window position at plane R
                    const int pos = w.A + e;
                    off += ((pos < w.fp ? deep_yp : deep_y) + pos) * (2 * D);
                    ks_ = s.kdeep + off;
                    vs_ = s.vdeep + off;
                    return true;
                }
                e -= w.ndw;
                if (e < w.nbr) {  // sliding: draft token e at plane R (its depth-R row)
                    off += ((grow0 + (int64_t)e * R + R - 1) * H + w.h) * (2 * D);
                    ks_ = a.Kb + off;
                    vs_ = a.Vb + off;
                    return true;
                }
                return false;  // past the unit's keys: zero fill
            };
            auto copy_key = [&](int kl, int v) {
                const char* ks_ = a.Q;
                const char* vs_ = a.Q;
                const bool valid = key_src(k0 + kl, v, ks_, vs_);
                const int c = v >> 2, v4 = v & 3;
                uint8_t* dk = stage + c * Lay::KCB + kl * 64 + ((v4 ^ ((kl >> 1) & 3)) << 4);
                cp_async16_zfill(dk, ks_, valid);
                cp_async16_zfill(dk + NCH * Lay::KCB, vs_, valid);
            };
            if (w.fast) {
                // The whole window in one box per column chunk (k0 = 0), then the
                // chunk's other keys and zero fill by copies.
                if (lane == 0) {
                    mbar_expect_tx(bar, (uint32_t)(s.Wcap * 64 * NCH * 2));
                    const int y = w.ring ? (int)ring_y : (int)((w.A < w.fp ? deep_yp : deep_y) + w.A);
                    const CUtensorMap* mk = w.ring ? &tm.wkf : &tm.rkf;
                    const CUtensorMap* mv = w.ring ? &tm.wvf : &tm.rvf;
#pragma unroll
                    for (int c = 0; c < NCH; ++c) {
                        tma_load_2d(stage + c * Lay::KCB, mk, 32 * c, y, bar);
                        tma_load_2d(stage + (NCH + c) * Lay::KCB, mv, 32 * c, y, bar);
                    }
                }
                const int nrest = 16 * nt - s.Wcap;
                for (int e = lane; e < nrest * VPR; e += 32) copy_key(s.Wcap + e / VPR, e % VPR);
                cp_async_mbar_arrive(bar);
                return;
            }
            uint32_t tma_groups = 0;
#pragma unroll
            for (int gm = 0; gm < 2 * NT; ++gm) {
                const int kk = k0 + 8 * gm;
                if (gm < 2 * nt && kk + 8 <= w.nw) {
                    // contiguous in one ring plane, or deep rows on one side of a fork position
                    const bool contig = w.ring ? ((w.slot0 + kk) % s.Wcap) + 8 <= s.Wcap
                                               : (w.A + kk < w.fp) == (w.A + kk + 7 < w.fp);
                    if (contig) tma_groups |= 1u << gm;
                }
            }
            if (lane == 0) {
                mbar_expect_tx(bar, (uint32_t)__popc(tma_groups) * 8 * 64 * NCH * 2);
                uint32_t gmask = tma_groups;
                while (gmask) {
                    const int gm = __ffs(gmask) - 1;
                    gmask &= gmask - 1;
                    const int kk = k0 + 8 * gm;
                    const int y = w.ring ? (int)(ring_y + (w.slot0 + kk) % s.Wcap)
                                         : (int)((w.A + kk < w.fp ? deep_yp : deep_y) + w.A + kk);
                    const CUtensorMap* mk = w.ring ? &tm.wk : &tm.rk;
                    const CUtensorMap* mv = w.ring ? &tm.wv : &tm.rv;
#pragma unroll
                    for (int c = 0; c < NCH; ++c) {
                        tma_load_2d(stage + c * Lay::KCB + gm * 512, mk, 32 * c, y, bar);
                        tma_load_2d(stage + (NCH + c) * Lay::KCB + gm * 512, mv, 32 * c, y, bar);
                    }
                }
            }
            uint32_t other = ((1u << (2 * nt)) - 1) & ~tma_groups;
            while (other) {  // warp-uniform
                const int gm = __ffs(other) - 1;
                other &= other - 1;
                for (int e = lane; e < 8 * VPR; e += 32) copy_key(8 * gm + e / VPR, e % VPR);
            }
            cp_async_mbar_arrive(bar);
        };

        // A whole-window unit into a ring stage: the ring plane (or Wcap deep rows) by
        // one tensor box per column chunk (a lane each), the draft tokens after it by
        // 16-byte copies, the V rows of the rest of the unit's 16-key tiles zeroed.  Tensor copies write rows below Wcap and the other writes rows from
        // Wcap on, so a stage needs a proxy fence only after a use that wrote window
        // rows by copies (a unit of the general form; `dirty`).
        auto ring_issue = [&](const Unit& w, uint8_t* stage, uint64_t* bar, uint8_t* dirty) {
            if (*dirty) {
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) *dirty = 0;
            }
            if (lane == 0) mbar_expect_tx(bar, (uint32_t)(s.Wcap * 64 * NCH * 2));
            __syncwarp();
            if (lane < 2 * NCH) {  // one box per lane: K column chunks, then V
                const int64_t y = w.ring ? ((((int64_t)a.layer * s.Bmax + w.seq) * H + w.h) * (R - 1) + (w.r - 1)) * s.Wcap
                                         : (((int64_t)a.layer * s.Bmax + (w.A < w.fp ? w.fb : w.seq)) * H + w.h) * s.Tmax + w.A;
                const bool isv = lane >= NCH;
                const int c = isv ? lane - NCH : lane;
                const CUtensorMap* m = w.ring ? (isv ? &tm.wvf : &tm.wkf) : (isv ? &tm.rvf : &tm.rkf);
                tma_load_2d(stage + lane * Lay::KCB, m, 32 * c, (int)y, bar);
            }
            const int64_t grow0 = (int64_t)w.g * kR;
            // draft tokens e < nblk (K and V rows)
            const int ncopy = 2 * w.nblk * VPR;
            for (int e = lane; e < ncopy; e += 32) {
                const int v = e % VPR, rr = e / VPR, c = v >> 2, v4 = v & 3;
                const int tok = rr >> 1, part = rr & 1, kl = w.koff + tok;
                const char* src =
                    (part ? a.Vb : a.Kb) + ((grow0 + (int64_t)tok * R + w.r - 1) * H + w.h) * (2 * D) + v * 16;
                cp_async16(stage + (part * NCH + c) * Lay::KCB + kl * 64 + ((v4 ^ ((kl >> 1) & 3)) << 4), src);
            }
            // zeros in the V rows past the unit's keys up to its last 16-key tile (their
            // probabilities are 0, and 0 x finite is 0; K rows there are masked whatever
            // they hold)
            const int z0 = w.koff + w.nblk, z1 = (w.nk + 15) / 16 * 16;
            const int nz = (z1 - z0) * VPR;
            for (int e = lane; e < nz; e += 32) {
                const int v = e % VPR, kl = z0 + e / VPR, c = v >> 2, v4 = v & 3;
                *reinterpret_cast<uint4*>(stage + (NCH + c) * Lay::KCB + kl * 64 + ((v4 ^ ((kl >> 1) & 3)) << 4)) =
                    make_uint4(0u, 0u, 0u, 0u);
            }
            cp_async_mbar_arrive(bar);
        };

        // One chunk of keys [k0, k0 + KC) of unit w from the stage at sb_in into the
        // running (o, m, l) of rows ra, rb.
        auto compute = [&](const Unit& w, int k0, uint32_t sb_in, const uint32_t (&bq)[NKS][2], float (&o)[NMT][4],
                           float& m_a, float& m_b, float& l_a, float& l_b) {
            const int nt = (min(KC, w.nk - k0) + 15) / 16;
            const uint32_t sb = smem_ready(sb_in);
            // Two 16-key tiles per pass of a loop that is not unrolled (the body is
            // what every window warp runs, so it stays in the instruction cache),
            // with the running maxima and sums rescaled once per pass.
#pragma unroll 1
            for (int t0 = 0; t0 < nt; t0 += 2) {
                const bool two = t0 + 1 < nt;
                // ---- S^T = K Q^T for the pass's tiles (independent chains)
                float sc[2][4];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    sc[u][0] = sc[u][1] = sc[u][2] = sc[u][3] = 0.f;
                    if (u == 0 || two) {
#pragma unroll
                        for (int ks = 0; ks < NKS; ++ks) {
                            uint32_t a0, a1, a2, a3;
                            ldsm_x4_r(sb + (ks >> 1) * Lay::KCB + (16 * (t0 + u) + rk) * 64 + ((ks & 1) ? k_sw1 : k_sw0),
                                      a0, a1, a2, a3);
                            mma_16816(sc[u], a0, a1, a2, a3, bq[ks][0], bq[ks][1]);
                        }
                    }
                }
                // ---- visibility and the pass's row maxima.  Key kk is visible to row j
                // if it is a window key, or block token kk - koff <= j (sliding: per row).
                float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
                for (int u = 0; u < 2; ++u) {
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        const int kk = k0 + 16 * (t0 + u) + r8 + 8 * hf;
                        bool va, vb;
                        if (u == 1 && !two) {
                            va = vb = false;
                        } else if (kk < w.koff) {
                            // window key: offset i from A (whole-window ring: slot kk)
                            int i = kk;
                            if (w.fast && w.ring) {
                                i = kk + s.Wcap - w.slot0;
                                if (i >= s.Wcap) i -= s.Wcap;
                            }
                            va = vb = i < w.nw;
                            if (w.slide) {
                                va = va && i >= w.sbase + w.j0 + ra;
                                vb = vb && i >= w.sbase + w.j0 + rb;
                            }
                        } else if (!w.slide) {
                            const int e = kk - w.koff;
                            va = e < w.nblk && e <= w.j0 + ra;
                            vb = e < w.nblk && e <= w.j0 + rb;
                        } else {
                            const int e = kk - w.koff;
                            va = slide_visible(e, w.j0 + ra, w.nblk, w.ndw, w.nbr, w.sbase, s.W);
                            vb = slide_visible(e, w.j0 + rb, w.nblk, w.ndw, w.nbr, w.sbase, s.W);
                        }
                        float& xa = sc[u][2 * hf];
                        float& xb = sc[u][2 * hf + 1];
                        xa = va ? xa * c2 : -INFINITY;
                        xb = vb ? xb * c2 : -INFINITY;
                        mx_a = fmaxf(mx_a, xa);
                        mx_b = fmaxf(mx_b, xb);
                    }
                }
#pragma unroll
                for (int o2 = 4; o2 < 32; o2 <<= 1) {
                    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, o2));
                    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, o2));
                }
                const float mn_a = fmaxf(m_a, mx_a), mn_b = fmaxf(m_b, mx_b);
                const float al_a = mn_a == -INFINITY ? 1.f : ex2(m_a - mn_a);
                const float al_b = mn_b == -INFINITY ? 1.f : ex2(m_b - mn_b);
                m_a = mn_a;
                m_b = mn_b;
                l_a *= al_a;
                l_b *= al_b;
#pragma unroll
                for (int mt = 0; mt < NMT; ++mt) {
                    o[mt][0] *= al_a;
                    o[mt][2] *= al_a;
                    o[mt][1] *= al_b;
                    o[mt][3] *= al_b;
                }
                // ---- probabilities, P^T fragments (8x8 transposes of the S^T fragments)
                // and O^T += V^T P^T
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    if (u == 0 || two) {
                        const float p0 = mn_a == -INFINITY ? 0.f : ex2(sc[u][0] - mn_a);
                        const float p1 = mn_b == -INFINITY ? 0.f : ex2(sc[u][1] - mn_b);
                        const float p2 = mn_a == -INFINITY ? 0.f : ex2(sc[u][2] - mn_a);
                        const float p3 = mn_b == -INFINITY ? 0.f : ex2(sc[u][3] - mn_b);
                        l_a += p0 + p2;
                        l_b += p1 + p3;
                        const uint32_t pb0 = movmatrix_t(pack_bf16(p0, p1));
                        const uint32_t pb1 = movmatrix_t(pack_bf16(p2, p3));
#pragma unroll
                        for (int mt = 0; mt < NMT; ++mt) {
                            uint32_t a0, a1, a2, a3;
                            ldsm_x4_t_r(sb + NCH * Lay::KCB + (mt >> 1) * Lay::KCB + (16 * (t0 + u) + rv) * 64 +
                                            ((mt & 1) ? v_sw1 : v_sw0),
                                        a0, a1, a2, a3);
                            mma_16816(o[mt], a0, a1, a2, a3, pb0, pb1);
                        }
                    }
                }
            }
            __syncwarp();  // every lane is done reading the stage
        };

        // A whole unit (every key in the stage, no sliding window) in one pass: S^T of
        // all its 16-key tiles (independent accumulation chains), the visibility mask,
        // one row max, the probabilities and O^T = V^T P^T.  The unit's keys fit in
        // registers, so no running rescale is needed; the chain from the stage's
        // arrival to its release is a few hundred cycles.
        auto compute_whole = [&](const Unit& w, uint32_t sb_in, const uint32_t (&bq)[NKS][2], float (&o)[NMT][4],
                                 float& m_a, float& m_b, float& l_a, float& l_b) {
            const int nt = (w.nk + 15) / 16;  // <= NT (the producer checked nk <= KC)
            const uint32_t sb = smem_ready(sb_in);
            float sc[NT][4];
#pragma unroll
            for (int u = 0; u < NT; ++u) {
                sc[u][0] = sc[u][1] = sc[u][2] = sc[u][3] = 0.f;
                if (u < nt) {
#pragma unroll
                    for (int ks = 0; ks < NKS; ++ks) {
                        uint32_t a0, a1, a2, a3;
                        ldsm_x4_r(sb + (ks >> 1) * Lay::KCB + (16 * u + rk) * 64 + ((ks & 1) ? k_sw1 : k_sw0), a0, a1,
                                  a2, a3);
                        mma_16816(sc[u], a0, a1, a2, a3, bq[ks][0], bq[ks][1]);
                    }
                }
            }
            // Key kk is visible to row j if it is a live window slot (whole-window ring
            // units: slot kk holds position A + ((kk - A) mod Wcap)), or draft token
            // kk - koff <= j.  Keys past the unit's are draft indices >= nblk.
            const bool wrap = w.fast && w.ring;
            float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
            for (int u = 0; u < NT; ++u) {
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const int kk = 16 * u + r8 + 8 * hf;
                    bool va, vb;
                    if (kk < w.koff) {
                        int i = kk;
                        if (wrap) {
                            i += s.Wcap - w.slot0;
                            if (i >= s.Wcap) i -= s.Wcap;
                        }
                        va = vb = i < w.nw;
                    } else {
                        const int e = kk - w.koff;
                        va = e < w.nblk && e <= w.j0 + ra;
                        vb = e < w.nblk && e <= w.j0 + rb;
                    }
                    float& xa = sc[u][2 * hf];
                    float& xb = sc[u][2 * hf + 1];
                    xa = va ? xa * c2 : -INFINITY;
                    xb = vb ? xb * c2 : -INFINITY;
                    mx_a = fmaxf(mx_a, xa);
                    mx_b = fmaxf(mx_b, xb);
                }
            }
#pragma unroll
            for (int o2 = 4; o2 < 32; o2 <<= 1) {
                mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, o2));
                mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, o2));
            }
            m_a = mx_a;
            m_b = mx_b;
            float la = 0.f, lb = 0.f;
#pragma unroll
            for (int u = 0; u < NT; ++u) {
                if (u < nt) {
                    const float p0 = mx_a == -INFINITY ? 0.f : ex2(sc[u][0] - mx_a);
                    const float p1 = mx_b == -INFINITY ? 0.f : ex2(sc[u][1] - mx_b);
                    const float p2 = mx_a == -INFINITY ? 0.f : ex2(sc[u][2] - mx_a);
                    const float p3 = mx_b == -INFINITY ? 0.f : ex2(sc[u][3] - mx_b);
                    la += p0 + p2;
                    lb += p1 + p3;
                    const uint32_t pb0 = movmatrix_t(pack_bf16(p0, p1));
                    const uint32_t pb1 = movmatrix_t(pack_bf16(p2, p3));
#pragma unroll
                    for (int mt = 0; mt < NMT; ++mt) {
                        uint32_t a0, a1, a2, a3;
                        ldsm_x4_t_r(sb + NCH * Lay::KCB + (mt >> 1) * Lay::KCB + (16 * u + rv) * 64 +
                                        ((mt & 1) ? v_sw1 : v_sw0),
                                    a0, a1, a2, a3);
                        mma_16816(o[mt], a0, a1, a2, a3, pb0, pb1);
                    }
                }
            }
            l_a = la;
            l_b = lb;
            __syncwarp();  // every lane is done reading the stage
        };

        // Publish a unit's partial (segment nsplit of its rows).
        auto publish = [&](const Slice& w, const float (&o)[NMT][4], float m_a, float m_b, float l_a, float l_b) {
#pragma unroll
            for (int o2 = 4; o2 < 32; o2 <<= 1) {
                l_a += __shfl_xor_sync(0xffffffffu, l_a, o2);
                l_b += __shfl_xor_sync(0xffffffffu, l_b, o2);
            }
            {
                const bool va = ra < w.nr, vb = rb < w.nr;
                const int64_t grow0 = (int64_t)w.g * kR;
                const int64_t pa_ = ((grow0 + (int64_t)(w.j0 + ra) * R + w.r - 1) * H + w.h) * a.nseg + a.nsplit;
                const int64_t pb_ = ((grow0 + (int64_t)(w.j0 + rb) * R + w.r - 1) * H + w.h) * a.nseg + a.nsplit;
#pragma unroll
                for (int mt = 0; mt < NMT; ++mt) {
                    const int ch = 16 * mt + r8;
                    if (va) {
                        a.part_o[pa_ * D + ch] = o[mt][0];
                        a.part_o[pa_ * D + ch + 8] = o[mt][2];
                    }
                    if (vb) {
                        a.part_o[pb_ * D + ch] = o[mt][1];
                        a.part_o[pb_ * D + ch + 8] = o[mt][3];
                    }
                }
                if (r8 == 0) {
                    if (va) a.part_ml[pa_] = make_float2(m_a, l_a);
                    if (vb) a.part_ml[pb_] = make_float2(m_b, l_b);
                }
            }
        };

        if constexpr (RING) {
            // ---- stage ring: full[st] (33 arrivals: 32 lanes' copies + the expect_tx),
            // empty[st] (the consumer that read it), the unit in desc[st].
            static_assert(sizeof(Unit) <= Lay::DESC_BYTES, "unit descriptor");
            const int NS = deep_cta ? Lay::NS_DEEP : Lay::NW_FULL;
            uint8_t* sring = sm + (deep_cta ? Lay::OFF_W : 0);
            uint64_t* full = wbar;
            uint64_t* empty = wbar + Lay::NWARPS;
            Unit* desc = reinterpret_cast<Unit*>(sm + Lay::OFF_DESC);
            int* ticket = reinterpret_cast<int*>(sm + Lay::OFF_MISC + 20);
            // A consumer waits for its ticket to be issued into its stage before it
            // looks at the stage's barrier: a ticket a full ring ahead would otherwise
            // see the parity of the stage's previous use and pass at once.  (Shared
            // memory is one coherent store for the CTA: once the ticket shows, the
            // barrier's earlier phases show too.)
            volatile int* issued = reinterpret_cast<volatile int*>(sm + Lay::OFF_ISS);
            // Producer warps take tickets in turn: four in a CTA without deep items
            // (when it has eight warps or more), two or one in a deep CTA.
            const int nwin = deep_cta ? Lay::NWARPS - kDeepWarps : Lay::NWARPS;
            const int NP = nwin >= 8 ? 4 : nwin >= 4 ? 2 : 1;
            const int ub = (int)(ub64 < pa.nunits ? ub64 : pa.nunits);
            const int ntk = uend > ub ? uend - ub : 0;
            if (warp >= wfirst && warp < wfirst + NP) {
                // ---------------------------------------- producers
                // (g, h, r, q) of the warp's next unit, stepped without divisions
                const int u0 = ub + (warp - wfirst);
                int cg = u0 / (QS * R * H), ch = (u0 / (QS * R)) % H, cr = (u0 / QS) % R + 1, cq = u0 % QS;
                auto step = [&]() {
                    if (++cq == QS) {
                        cq = 0;
                        if (++cr > R) {
                            cr = 1;
                            if (++ch == H) {
                                ch = 0;
                                ++cg;
                            }
                        }
                    }
                };
                for (int idx = warp - wfirst; idx < ntk; idx += NP) {
                    const int st = idx % NS;
                    if (idx >= NS) {
                        // The stage's previous ticket (another producer's) must be issued
                        // before its empty barrier is looked at, for the same reason.
                        int okc = 1;
                        if (lane == 0) okc = count_wait(issued + st, idx - NS - 1, abort_flag, s.err);
                        if (!__shfl_sync(0xffffffffu, okc, 0)) break;
                        if (!warp_wait(empty + st, ((idx / NS) - 1) & 1, abort_flag, s.err)) break;
                    }
                    Unit w = describe_at(cg, ch, cr, cq);
                    for (int i = 0; i < NP; ++i) step();
                    // every unit here is one chunk, without the sliding window
                    if (w.ok && (w.nk > KC || w.slide)) {
                        if (lane == 0) set_device_error(s.err, RIPE_DEVERR_BRANCH);
                        w.ok = false;
                    }
                    if (lane == 0) desc[st] = w;  // published by lane 0's arrival below
                    if (w.ok && w.fast) {
                        ring_issue(w, sring + st * Lay::WSTAGE, full + st, sm + Lay::OFF_DIRTY + st);
                    } else if (w.ok) {
                        issue(w, 0, sring + st * Lay::WSTAGE, full + st);
                        if (lane == 0) sm[Lay::OFF_DIRTY + st] = 1;
                    } else {
                        if (lane == 0) mbar_arrive(full + st);
                        cp_async_mbar_arrive(full + st);
                    }
                    if (lane == 0) issued[st] = idx;
                }
                // This warp's copies land before it leaves (the tensor copies of a ring
                // that gave up are waited for at the end of the kernel).
                cp_async_wait_all();
            } else {
                // ---------------------------------------- consumers
                // A consumer claims its next ticket as it starts a unit and loads that
                // unit's queries into registers meanwhile (the ticket names the unit).
                auto claim = [&](uint32_t (&b)[NKS][2]) {
                    int t = 0;
                    if (lane == 0) t = atomicAdd(ticket, 1);
                    t = __shfl_sync(0xffffffffu, t, 0);
                    if (t < ntk) {
                        const int u = ub + t;
                        Unit q;
                        q.g = u / (QS * R * H);
                        q.h = (u / (QS * R)) % H;
                        q.r = (u / QS) % R + 1;
                        q.j0 = (u % QS) * kWR;
                        q.nr = min(kWR, k - q.j0);
                        load_q(q, b);
                    }
                    return t;
                };
                uint32_t bqn[NKS][2];
                int tn = claim(bqn);
                while (tn < ntk) {
                    const int t = tn;
                    uint32_t bq[NKS][2];
#pragma unroll
                    for (int ks = 0; ks < NKS; ++ks) {
                        bq[ks][0] = bqn[ks][0];
                        bq[ks][1] = bqn[ks][1];
                    }
                    tn = claim(bqn);
                    const int st = t % NS;
                    int okc = 1;
                    if (lane == 0) okc = count_wait(issued + st, t - 1, abort_flag, s.err);
                    if (!__shfl_sync(0xffffffffu, okc, 0)) break;
                    if (!warp_wait(full + st, (t / NS) & 1, abort_flag, s.err)) break;
                    const Unit w = desc[st];
                    const uint32_t sa = smem_u32(sring + st * Lay::WSTAGE);
                    float o[NMT][4];
                    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
                    if (w.ok) {
#pragma unroll
                        for (int mt = 0; mt < NMT; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
                        compute_whole(w, sa, bq, o, m_a, m_b, l_a, l_b);
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(empty + st);  // the stage is free again
                    if (w.ok) publish(Slice{w.g, w.h, w.r, w.j0, w.nr, w.E}, o, m_a, m_b, l_a, l_b);
                }
            }
        } else {
            uint32_t phase = 0;
            bool wok = true;
            // One site per step (next unit, issue, publish) keeps the loop's code small.
            // Each pass: pick the next load (the current unit's next chunk, or a new
            // unit), issue it, publish a unit that just ended, then wait for the load
            // and compute on it.
            Unit cur{};
            int k0 = 0;
            bool started = false;
            uint32_t bq[NKS][2];
            float o[NMT][4];
            float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
            while (true) {
                const Slice cs{cur.g, cur.h, cur.r, cur.j0, cur.nr, cur.E};
                Unit nxt;
                int nk0 = 0;
                bool have;
                if (started && k0 + KC < cur.nk) {
                    nxt = cur;
                    nk0 = k0 + KC;
                    have = true;
                } else {
                    have = next_valid(nxt);
                }
                const bool ended = started && nk0 == 0;
                if (have) {
                    issue(nxt, nk0, stage, bar);
                    if (nk0 == 0) load_q(nxt, bq);  // the current unit's compute is done with bq
                }
                if (ended) publish(cs, o, m_a, m_b, l_a, l_b);  // segment nsplit of its rows
                if (!have) break;
                cur = nxt;
                k0 = nk0;
                started = true;
                if (k0 == 0) {
#pragma unroll
                    for (int mt = 0; mt < NMT; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
                    m_a = m_b = -INFINITY;
                    l_a = l_b = 0.f;
                }
                if (!warp_wait(bar, phase & 1, abort_flag, s.err)) {
                    wok = false;
                    break;
                }
                ++phase;
                compute(cur, k0, stage_a, bq, o, m_a, m_b, l_a, l_b);
            }
            if (!wok) {
                // Let this warp's copies land before the CTA's shared memory goes away.
                volatile int no_abort = 0;
                cp_async_wait_all();
                mbar_wait(bar, phase & 1, &no_abort, s.err);
            }
        }
    }


    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (RING && threadIdx.x == 0 && *abort_flag) {
        // A ring that gave up may still have tensor copies in flight: wait for the
        // last phase issued into each stage before the shared memory goes away.
        const int NS = deep_cta ? Lay::NS_DEEP : Lay::NW_FULL;
        const int* iss = reinterpret_cast<const int*>(sm + Lay::OFF_ISS);
        volatile int no_abort = 0;
        for (int st = 0; st < NS; ++st)
            if (iss[st] >= 0) mbar_wait(wbar + st, (iss[st] / NS) & 1, &no_abort, s.err);
    }
    if (deep_cta && warp == 5) tmem_dealloc(tmem, Lay::TMEM_COLS);
}

// The merge of the persistent kernel's partials: one warp per (row, head), small
// enough that every warp of the grid is resident at once.  A row of group g has
// E = gE[g] segments (0: the group was skipped): deep chunks 0..E-2 in order, then
// the window (segment nsplit).  M = max m_s, L = sum l_s 2^(m_s-M),
// O = sum 2^(m_s-M) o_s / L, lse = (M + log2 L) ln 2, segments in that order.
// E and the first segments load together (the deep ones speculatively).
template <int D>
__global__ void __launch_bounds__(128, 12) persist_merge_kernel(VerifyArgs a, int nrows) {
    sm100::grid_dependency_wait();  // the persistent kernel's partials
    const int H = a.s.H, kR = a.ba.k * a.s.R;
    const int lane = threadIdx.x % 32;
    const int64_t item = (int64_t)blockIdx.x * 4 + threadIdx.x / 32;
    if (item >= (int64_t)nrows * H) return;
    const int row = (int)(item / H), h = (int)(item % H);
    const int E = __ldcg(a.gE + row / kR);
    const int64_t base = ((int64_t)row * H + h) * a.nseg;
    constexpr int NC = D / 32, NS0 = 3;  // deep segments loaded with E
    const int nd0 = a.nsplit < NS0 ? a.nsplit : NS0;
    float2 mw = __ldcg(a.part_ml + base + a.nsplit);
    float xw[NC];
    {
        const float* po = a.part_o + (base + a.nsplit) * D + lane;
#pragma unroll
        for (int i = 0; i < NC; ++i) xw[i] = __ldcg(po + 32 * i);
    }
    float2 md[NS0];
    float xd[NS0][NC];
#pragma unroll
    for (int j = 0; j < NS0; ++j) {
        md[j] = make_float2(-INFINITY, 0.f);
#pragma unroll
        for (int i = 0; i < NC; ++i) xd[j][i] = 0.f;
        if (j < nd0) {
            md[j] = __ldcg(a.part_ml + base + j);
            const float* po = a.part_o + (base + j) * D + lane;
#pragma unroll
            for (int i = 0; i < NC; ++i) xd[j][i] = __ldcg(po + 32 * i);
        }
    }
    if (E <= 0) return;
    const int nd = E - 1;  // deep segments with keys
    float M = mw.x;
    for (int j = 0; j < nd; ++j) {
        float2 mj = md[0];
#pragma unroll
        for (int q = 1; q < NS0; ++q) mj = j == q ? md[q] : mj;
        if (j >= NS0) mj = __ldcg(a.part_ml + base + j);
        M = fmaxf(M, mj.x);
    }
    float L = 0.f;
    float acc[NC];
#pragma unroll
    for (int i = 0; i < NC; ++i) acc[i] = 0.f;
#pragma unroll
    for (int j = 0; j < NS0; ++j) {
        if (j < nd) {
            const float f = sm100::ex2(md[j].x - M);
            L = fmaf(md[j].y, f, L);
#pragma unroll
            for (int i = 0; i < NC; ++i) acc[i] = fmaf(xd[j][i], f, acc[i]);
        }
    }
    for (int j = NS0; j < nd; ++j) {  // more than NS0 deep segments (rare)
        const float2 mj = __ldcg(a.part_ml + base + j);
        const float* po = a.part_o + (base + j) * D + lane;
        const float f = sm100::ex2(mj.x - M);
        L = fmaf(mj.y, f, L);
#pragma unroll
        for (int i = 0; i < NC; ++i) acc[i] = fmaf(__ldcg(po + 32 * i), f, acc[i]);
    }
    {
        const float f = sm100::ex2(mw.x - M);
        L = fmaf(mw.y, f, L);
#pragma unroll
        for (int i = 0; i < NC; ++i) acc[i] = fmaf(xw[i], f, acc[i]);
    }
    const float inv = 1.f / L;
    __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.O) + ((int64_t)row * H + h) * D + lane;
#pragma unroll
    for (int i = 0; i < NC; ++i) orow[32 * i] = __float2bfloat16_rn(acc[i] * inv);
    if (lane == 0 && a.lse) a.lse[(int64_t)row * H + h] = (M + log2f(L)) * 0.69314718055994531f;
}

template <int D>
cudaError_t launch_merge(const VerifyArgs& a, int nrows, cudaStream_t st) {
    const int64_t blocks = ((int64_t)nrows * a.s.H + 3) / 4;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(128);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, persist_merge_kernel<D>, a, nrows);
    ripe_count_launch();
    return e;
}

template <int D, int MT, int ST, int NWW, int KC, bool RING>
cudaError_t launch_p(const PMaps& tm, const VerifyArgs& a, const PArgs& pa, int grid, cudaStream_t st) {
    using Lay = PLayout<D, MT, ST, NWW, KC>;
    static_assert(Lay::SMEM <= 232448, "shared memory budget");
    // Per-warp stages: every window warp of a deep CTA owns a stage.
    static_assert(RING || Lay::NS_DEEP >= NWW, "window stages of a deep CTA");
    static PerDeviceOnce configured;
    cudaError_t ce = per_device_once(configured, [] {
        cudaError_t e = cudaFuncSetAttribute(persist_kernel<D, MT, ST, NWW, KC, RING>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::SMEM);
        if (e != cudaSuccess) return e;
        return cudaFuncSetAttribute(persist_kernel<D, MT, ST, NWW, KC, RING>,
                                    cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    });
    if (ce != cudaSuccess) return ce;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(Lay::THREADS);
    cfg.dynamicSmemBytes = Lay::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, persist_kernel<D, MT, ST, NWW, KC, RING>, tm, a, pa);
    ripe_count_launch();
    return e;
}

}  // namespace

// Keys per window chunk of the instantiation for (d, mt).
static int persist_kc(int d, int mt) { return d == 128 && mt == 2 ? 48 : 80; }

// Whether the window units run through the stage ring: every unit one chunk (the
// whole window, the draft tokens), no sliding window (whose units read more keys).
bool persist_ring_ok(int d, int mt, int Wcap, int k, int sliding, int full_box) {
    return !sliding && full_box && Wcap + k <= persist_kc(d, mt);
}

// Window warps a CTA of each role runs, for the planner's cost model.
void persist_shape(int d, int mt, int* nww_deep, int* nww_other) {
#define RIPE_SHAPE(D_, MT_, ST_, NWW_, KC_)                      \
    if (d == D_ && mt == MT_) {                                  \
        *nww_deep = NWW_;                                        \
        *nww_other = PLayout<D_, MT_, ST_, NWW_, KC_>::NW_FULL;  \
        return;                                                  \
    }
    RIPE_SHAPE(64, 1, 4, 6, 80)
    RIPE_SHAPE(96, 1, 4, 4, 80)
    RIPE_SHAPE(128, 1, 3, 3, 80)
    RIPE_SHAPE(64, 2, 4, 5, 80)
    RIPE_SHAPE(96, 2, 3, 3, 80)
    RIPE_SHAPE(128, 2, 3, 2, 48)
#undef RIPE_SHAPE
    *nww_deep = *nww_other = 0;
}

cudaError_t launch_persist(const void* tmaps, const VerifyArgs& args, int pd, int n_lo, int n_hi,
                           int ndeep, int nunits, int grid, int mt, long long probe_cycles, int sliding,
                           int full_box, cudaStream_t st) {
    // Cache maps: 0 deep K, 1 deep V (64-row boxes); 6 ring K, 7 ring V, 8 deep K,
    // 9 deep V (8-row boxes); 10-13 the same four in Wcap-row boxes; plus one of
    // this call's Q.
    PMaps tm;
    const CUtensorMap* cm = reinterpret_cast<const CUtensorMap*>(tmaps);
    tm.dk = cm[0];
    tm.dv = cm[1];
    tm.wk = cm[6];
    tm.wv = cm[7];
    tm.rk = cm[8];
    tm.rv = cm[9];
    tm.wkf = cm[10];
    tm.wvf = cm[11];
    tm.rkf = cm[12];
    tm.rvf = cm[13];
    VerifyArgs a = args;
    if (!make_q_map(&tm.q, a)) return cudaErrorInvalidValue;
    PArgs pa{pd, n_lo, n_hi, ndeep, nunits, probe_cycles, sliding, full_box};
    const int d = a.s.d;
    // The stage ring when every unit is one chunk with room for its queries.
    const bool ring = persist_ring_ok(d, mt, a.s.Wcap, a.ba.k, sliding, full_box);
    // The kernel publishes every partial; the merge kernel (its dependent launch)
    // combines them.
    // Deep stages: ST_ with per-warp window stages; STR_ with the ring, whose deep
    // CTAs need only a stage or two for their few window units (the deep pipeline is
    // bound by its bytes in flight).
#define RIPE_LAUNCH(D_, MT_, ST_, STR_, NWW_, KC_)                                            \
    if (d == D_ && mt == MT_) {                                                            \
        cudaError_t e = ring ? launch_p<D_, MT_, STR_, NWW_, KC_, true>(tm, a, pa, grid, st)  \
                             : launch_p<D_, MT_, ST_, NWW_, KC_, false>(tm, a, pa, grid, st);  \
        if (e != cudaSuccess) return e;                                                    \
        return launch_merge<D_>(a, a.ba.nrows, st);                                        \
    }
    RIPE_LAUNCH(64, 1, 4, 8, 6, 80)
    RIPE_LAUNCH(96, 1, 4, 6, 4, 80)
    RIPE_LAUNCH(128, 1, 3, 4, 3, 80)
    RIPE_LAUNCH(64, 2, 4, 4, 5, 80)
    RIPE_LAUNCH(96, 2, 3, 3, 3, 80)
    RIPE_LAUNCH(128, 2, 3, 3, 2, 48)
#undef RIPE_LAUNCH
    return cudaErrorInvalidValue;
}
