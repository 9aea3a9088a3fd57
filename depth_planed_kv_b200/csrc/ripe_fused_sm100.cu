// ripe_fused_sm100.cu -- RIPE verify-attention of one layer in one sm_100a kernel.
//
// Every query row of a sequence -- all draft tokens at all loop depths, and every
// LoopSpec branch -- reads the same deepest plane R outside the window, while a
// row at depth r reads plane r of the positions still inside the window and the
// draft-block tokens of its own branch (RIPE abstract, sentence introducing RIPE;
// LoopSpec article on mixed-depth branches in one batched call).
//
// One CTA serves one (sequence group, head, split of the deep region):
//
//   deep region (warps 0-5): the group's rows are stacked into 128-row tiles and
//     S = Q K^T (tcgen05.mma, fp32 in TMEM) -> online softmax on CUDA cores ->
//     O += P V (tcgen05.mma, fp32 in TMEM)
//   runs over this split's chunk of plane R, K and V streamed by TMA through a
//   ring of shared-memory stages.  Warps 0-3 own TMEM lanes 0-127 (one row each)
//   and do Q staging, softmax and the epilogue; warp 4 lane 0 issues TMA; warp 5
//   allocates TMEM and its lane 0 issues the MMAs.
//
//   window planes and draft block (warps 6..6+NW-1): the keys differ from depth
//   to depth, so nothing stacks across depths; a unit is one branch's chunk of
//   <= 8 rows.  Each window warp streams its units' keys 16 at a time through its
//   own ring of cp.async stages and runs both products on warp-level MMA tiles
//   (m16n8k16) in the transposed form S^T = K Q^T, O^T = V^T P^T: keys and
//   channels fill the 16-row side and the <= 8 query rows the 8-column side, and
//   P^T reaches the B operand by an 8x8 transpose (movmatrix).
//
// The splits of one (group, head) form a thread-block cluster.  Each CTA writes
// its partial results (m in log2 units, l, unnormalised o) to scratch; after a
// cluster barrier every CTA merges a share of the rows -- deep splits in order,
// then the window partial: M = max m, L = sum l 2^(m-M), O = sum o 2^(m-M) / L --
// and writes O and the LSE.  One merger per row, fixed order: bit-reproducible.
//
// Shared-memory operand layouts of the deep part (64-byte swizzle, 8-row /
// 512-byte atoms): Q, K K-major in 32-element column chunks of [rows][64 B];
// V MN-major (the same chunks read with head-dim as N); P K-major [128][32 keys]
// chunks written by the softmax threads.  Window stages hold the K and V rows of
// 16 keys in the same 64-byte-swizzled 32-column boxes (conflict-free ldmatrix).
#include <cuda.h>

#include <cstring>

#include "ripe_launch.h"
#include "ripe_verify.cuh"
#include "sm100_ptx.cuh"

namespace {

constexpr int kN = 64;             // deep keys per tile
constexpr int kDeepThreads = 192;  // warps 0-3 softmax, 4 TMA, 5 MMA
constexpr int kMaxGroupBranches = 64;
constexpr int kWinRows = 8;   // rows per window unit (the N of an m16n8k16 tile)
constexpr int kWinKeys = 16;  // keys per window tile (the M of an m16n8k16 tile)
constexpr int kRowTable = 512;  // group rows whose Q/O row index is tabulated in shared memory

// Tensor maps of one launch: deep K, V in 64-row boxes; ring K, V and deep K, V
// in 16-row boxes; Q of this call as [rows][H][d] in 128-row boxes of one head (all
// 32 columns wide, 64-byte swizzle).  The first six belong to the cache.
struct TMaps {
    CUtensorMap dk, dv, wk, wv, rk, rv, q;
};

// One branch of the group: its rows, its offset among the group's rows, its
// depth and the index of its first window unit.
struct BranchEnt {
    int row0, stride, ntok, off, depth, uoff;
};

struct GroupInfo {
    int first, nb, seq, nrows, T, A, key_begin, key_end, units;
    int fb, fp;  // deep positions below fp are read from sequence fb (a fork's parent)
};

template <int D, int MT, int ST, int NW, int NS>
struct FusedLayout {
    static constexpr int NCH = D / 32;               // 64-byte column chunks of the head dim
    // With one M tile, Q lives in tensor memory (A operand of QK^T from TMEM); with two,
    // TMEM is full and Q stays in shared memory (128 rows x 64 B per chunk).
    static constexpr bool QT = MT == 1;
    static constexpr int Q_BYTES = QT ? 0 : MT * NCH * 8192;
    static constexpr int KV_STAGE = NCH * 4096;      // 64 keys x 64 B per chunk
    static constexpr int WBOX = kWinKeys * 64;       // one 16-row x 64-byte window box
    static constexpr int WKV = NCH * WBOX;           // K (or V) of one window tile
    static constexpr int WSTAGE = 2 * WKV;           // K boxes, then V boxes
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + Q_BYTES;
    static constexpr int OFF_V = OFF_K + ST * KV_STAGE;
    static constexpr int OFF_W = OFF_V + ST * KV_STAGE;
    static constexpr int OFF_OST = OFF_W + NW * NS * WSTAGE;  // epilogue staging (Q in TMEM)
    static constexpr int OST_BYTES = QT ? 4 * 8 * (32 * 4 + 16) : 0;
    static constexpr int OFF_BAR = OFF_OST + OST_BYTES;
    // barriers: q_full, k_full[ST], v_full[ST], kv_empty[ST], s_full[2], p_full[2], pv_done[2], drain,
    // epi_done
    static constexpr int NBAR = 1 + 3 * ST + 8;
    static constexpr int OFF_WBAR = OFF_BAR + NBAR * 8;  // one per window stage
    static constexpr int OFF_MISC = OFF_WBAR + NW * NS * 8;
    static constexpr int OFF_BT = OFF_MISC + 64;
    static constexpr int OFF_RT = OFF_BT + kMaxGroupBranches * (int)sizeof(BranchEnt);
    static constexpr int BYTES = OFF_RT + kRowTable * 4;
    static constexpr int SMEM = BYTES + 1024;  // alignment slack
    static constexpr int THREADS = kDeepThreads + 32 * NW;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t S_COL(int mt, int sb) { return (uint32_t)((mt * 2 + sb) * kN); }
    static constexpr uint32_t O_COL(int mt) { return (uint32_t)(MT * 2 * kN + mt * 128); }
    static constexpr uint32_t Q_COL = 2 * kN + 128;  // Q in TMEM (QT): D/2 columns
};

// Warp-uniform bounded wait: every lane waits, and all lanes agree on the outcome
// (the tcgen05.ld/st that follow are warp-collective).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int32_t* err) {
    const bool ok = sm100::mbar_wait(bar, parity, abort, err);
    return __all_sync(0xffffffffu, ok);
}

// Row (of Q/O) of the group's rl-th query, branches in table order; -1 past the end.
__device__ int group_row_scan(const BranchEnt* bt, int nb, int rl) {
    for (int i = 0; i < nb; ++i)
        if (rl < bt[i].off + bt[i].ntok) return bt[i].row0 + (rl - bt[i].off) * bt[i].stride;
    return -1;
}
// The same from the shared-memory row table for the first kRowTable rows.
__device__ __forceinline__ int group_row(const int* rowtab, const BranchEnt* bt, int nb, int nrows, int rl) {
    if (rl >= nrows) return -1;
    return rl < kRowTable ? rowtab[rl] : group_row_scan(bt, nb, rl);
}

// Start of the g-th run of equal sequence ids in the branch table (warp-wide).
__device__ int group_start(const ripe_branch_t* tb, int nbranch, int g, int lane) {
    int count = 0;
    for (int base = 0; base < nbranch; base += 32) {
        const int i = base + lane;
        const bool st = i < nbranch && (i == 0 || tb[i].seq != tb[i - 1].seq);
        unsigned m = __ballot_sync(0xffffffffu, st);
        const int c = __popc(m);
        if (count + c > g) {
            for (int k = g - count; k > 0; --k) m &= m - 1;
            return base + __ffs(m) - 1;
        }
        count += c;
    }
    return nbranch;
}

// Window keys of a group: the positions [A, T) still inside the window.  At depth
// r < R they sit in ring plane r at slots (A .. T-1) mod Wcap; the unit reads the
// ring in slot order, slots lo .. lo+wk-1 (one contiguous run; slots outside the
// window are masked and zero-filled, which costs no traffic).  At depth R they
// are rows A .. T-1 of the deep plane.
struct WinKeys {
    int nwin, slot0, lo_ring, wk_ring;
};

__device__ __forceinline__ WinKeys win_keys(int A, int T, int Wcap) {
    WinKeys k;
    k.nwin = T - A;
    k.slot0 = A % Wcap;
    if (k.nwin == 0) {
        k.lo_ring = 0;
        k.wk_ring = 0;
    } else if (k.slot0 + k.nwin <= Wcap) {
        k.lo_ring = k.slot0 & ~15;
        k.wk_ring = k.slot0 + k.nwin - k.lo_ring;
    } else {
        k.lo_ring = 0;
        k.wk_ring = Wcap;
    }
    return k;
}

// A window unit: rows j0..j0+nr-1 of one branch against nk keys -- wk window keys
// (ring slots lo.. or deep rows A..), then block tokens 0..j0+nr-1 -- in ntiles
// tiles of 16 keys.
struct WinUnit {
    int row0, stride, depth, j0, nr, wk, lo, nk, ntiles;
};

// Unit u of the group (warp-collective): its branch is the last one whose first
// unit is <= u (branches without units share the next branch's first unit).
__device__ __forceinline__ WinUnit win_unit(const BranchEnt* bt, int nb, int u, const WinKeys& wkeys, int R,
                                           int lane) {
    const bool p0 = lane < nb && bt[lane].uoff <= u;
    const bool p1 = lane + 32 < nb && bt[lane + 32].uoff <= u;
    const int i = __popc(__ballot_sync(0xffffffffu, p0)) + __popc(__ballot_sync(0xffffffffu, p1)) - 1;
    const BranchEnt e = bt[i];
    WinUnit w;
    w.row0 = e.row0;
    w.stride = e.stride;
    w.depth = e.depth;
    w.j0 = (u - e.uoff) * kWinRows;
    w.nr = min(kWinRows, e.ntok - w.j0);
    const bool ring = e.depth < R;
    w.wk = ring ? wkeys.wk_ring : wkeys.nwin;
    w.lo = ring ? wkeys.lo_ring : 0;
    w.nk = w.wk + w.j0 + w.nr;
    w.ntiles = (w.nk + kWinKeys - 1) / kWinKeys;
    return w;
}

// Window key `key` (< wk) of a unit holds a position inside the window.
__device__ __forceinline__ bool win_valid(const WinUnit& w, const WinKeys& k, int R, int Wcap, int key) {
    if (w.depth >= R) return true;
    int d = w.lo + key - k.slot0;
    if (d < 0) d += Wcap;
    return d < k.nwin;
}

// The merge of NR rows (ro: row * H + head; ok: row exists): deep splits 0..np-1
// in order, then the window partial (segment nsplit): M = max m,
// L = sum l 2^(m-M), O = sum o 2^(m-M) / L.  Eight lanes per row (lane sl holds
// channels 4*sl + 32*c); every load of the NR rows is issued before the
// arithmetic (one round trip).  NU >= np + 1 bounds the segments.
template <int D, int NU, int NR>
__device__ __forceinline__ void merge_rows(const VerifyArgs& a, const int64_t* ro, const bool* ok, int np, int sl) {
    using sm100::ex2;
    using sm100::pack_bf16;
    constexpr int CH = D / 32;
    float2 ml[NR][NU];
    float4 x[NR][NU][CH];
#pragma unroll
    for (int r = 0; r < NR; ++r) {
#pragma unroll
        for (int sg = 0; sg < NU; ++sg) {
            if (ok[r] && sg <= np) {
                const int64_t seg = ro[r] * a.nseg + (sg < np ? sg : a.nsplit);
                ml[r][sg] = __ldcg(a.part_ml + seg);
#pragma unroll
                for (int c = 0; c < CH; ++c)
                    x[r][sg][c] = __ldcg(reinterpret_cast<const float4*>(a.part_o + seg * D + 4 * sl + 32 * c));
            }
        }
    }
#pragma unroll
    for (int r = 0; r < NR; ++r) {
        if (!ok[r]) continue;
        float M = -INFINITY;
#pragma unroll
        for (int sg = 0; sg < NU; ++sg)
            if (sg <= np) M = fmaxf(M, ml[r][sg].x);
        float f[NU], L = 0.f;
#pragma unroll
        for (int sg = 0; sg < NU; ++sg) {
            if (sg <= np) {
                f[sg] = ex2(ml[r][sg].x - M);
                L = fmaf(ml[r][sg].y, f[sg], L);
            }
        }
        __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.O) + ro[r] * D;
        const float inv = 1.f / L;
#pragma unroll
        for (int c = 0; c < CH; ++c) {
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int sg = 0; sg < NU; ++sg) {
                if (sg <= np) {
                    acc[0] = fmaf(x[r][sg][c].x, f[sg], acc[0]);
                    acc[1] = fmaf(x[r][sg][c].y, f[sg], acc[1]);
                    acc[2] = fmaf(x[r][sg][c].z, f[sg], acc[2]);
                    acc[3] = fmaf(x[r][sg][c].w, f[sg], acc[3]);
                }
            }
            *reinterpret_cast<uint2*>(orow + 4 * sl + 32 * c) =
                make_uint2(pack_bf16(acc[0] * inv, acc[1] * inv), pack_bf16(acc[2] * inv, acc[3] * inv));
        }
        if (sl == 0 && a.lse) a.lse[ro[r]] = (M + log2f(L)) * 0.69314718055994531f;
    }
}

// The same merge for any number of deep splits, one segment at a time (the same
// operation order, so the same result).
template <int D>
__device__ __noinline__ void merge_row_any(const float2* part_ml, const float* part_o, char* O_, float* lse,
                                           int nseg, int nsplit, int64_t ro, int np, int sl) {
    using sm100::ex2;
    using sm100::pack_bf16;
    constexpr int CH = D / 32;
    const int64_t base = ro * nseg;
    float M = -INFINITY;
    for (int sg = 0; sg <= np; ++sg) M = fmaxf(M, __ldcg(part_ml + base + (sg < np ? sg : nsplit)).x);
    float L = 0.f, acc[CH][4];
#pragma unroll
    for (int c = 0; c < CH; ++c) acc[c][0] = acc[c][1] = acc[c][2] = acc[c][3] = 0.f;
    for (int sg = 0; sg <= np; ++sg) {
        const int64_t seg = base + (sg < np ? sg : nsplit);
        const float2 ml = __ldcg(part_ml + seg);
        const float f = ex2(ml.x - M);
        L = fmaf(ml.y, f, L);
#pragma unroll
        for (int c = 0; c < CH; ++c) {
            const float4 x = __ldcg(reinterpret_cast<const float4*>(part_o + seg * D + 4 * sl + 32 * c));
            acc[c][0] = fmaf(x.x, f, acc[c][0]);
            acc[c][1] = fmaf(x.y, f, acc[c][1]);
            acc[c][2] = fmaf(x.z, f, acc[c][2]);
            acc[c][3] = fmaf(x.w, f, acc[c][3]);
        }
    }
    __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(O_) + ro * D;
    const float inv = 1.f / L;
#pragma unroll
    for (int c = 0; c < CH; ++c)
        *reinterpret_cast<uint2*>(orow + 4 * sl + 32 * c) =
            make_uint2(pack_bf16(acc[c][0] * inv, acc[c][1] * inv), pack_bf16(acc[c][2] * inv, acc[c][3] * inv));
    if (sl == 0 && lse) lse[ro] = (M + log2f(L)) * 0.69314718055994531f;
}

// One CTA per SM.  Registers come from the four SM sub-partitions (16384 each),
// which hold ceil(warps / 4) warps apiece: 168 per thread for 9-12 warps.
template <int D, int MT, int ST, int NW, int NS>
__global__ void __launch_bounds__(FusedLayout<D, MT, ST, NW, NS>::THREADS, 1)
verify_kernel(const __grid_constant__ TMaps tm, VerifyArgs a) {
    using Lay = FusedLayout<D, MT, ST, NW, NS>;
    using namespace sm100;
    constexpr int NCH = Lay::NCH;
    constexpr int RT = 128 * MT;
    constexpr uint32_t IDESC_QK = idesc_bf16(128, kN, 0);
    constexpr uint32_t IDESC_PV = idesc_bf16(128, D, 1);
    constexpr int NWARPS = Lay::THREADS / 32;

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
    uint64_t* epi_done = s_full + 7;  // the softmax warps' epilogue staging is finished
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Lay::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + Lay::OFF_MISC + 4);
    GroupInfo* gi = reinterpret_cast<GroupInfo*>(sm + Lay::OFF_MISC + 16);
    BranchEnt* bt = reinterpret_cast<BranchEnt*>(sm + Lay::OFF_BT);
    int* rowtab = reinterpret_cast<int*>(sm + Lay::OFF_RT);

    const StoreView& s = a.s;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int g = blockIdx.x, h = blockIdx.y, split = blockIdx.z;

    if (threadIdx.x == 0) {
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
        for (int i = 0; i < NW * NS; ++i) mbar_init(reinterpret_cast<uint64_t*>(sm + Lay::OFF_WBAR) + i, 32);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 5) {
        tmem_alloc(tmem_slot, Lay::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 4 && lane == 0) {
        prefetch_tmap(&tm.dk);
        prefetch_tmap(&tm.dv);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // Inputs and scratch may belong to the previous kernel in the stream.
    grid_dependency_wait();
    grid_launch_dependents();

    // ---- the group of branches this CTA serves (one sequence), its key range and units
    if (warp == 0) {
        int first, end;
        if (a.ba.table) {
            first = group_start(a.ba.table, a.ba.nbranch, g, lane);
            end = first < a.ba.nbranch ? group_start(a.ba.table, a.ba.nbranch, g + 1, lane) : first;
        } else {
            first = min(g * s.R, a.ba.nbranch);
            end = min(first + s.R, a.ba.nbranch);
        }
        int nb = end - first;
        if (nb > kMaxGroupBranches) {
            if (lane == 0) set_device_error(s.err, RIPE_DEVERR_BRANCH);
            nb = 0;
        }
        // Branch entries loaded in parallel; row and unit offsets by warp prefix sums.
        int seq = -1, base = 0, ubase = 0;
        for (int c0 = 0; c0 < nb; c0 += 32) {
            const int i = c0 + lane;
            Branch br;
            br.ok = false;
            if (i < nb) br = load_branch(a.ba, s.R, s.Bmax, first + i);
            if (i < nb && !br.ok && split == 0 && h == 0) set_device_error(s.err, RIPE_DEVERR_BRANCH);
            const int n = (i < nb && br.ok) ? br.ntok : 0;
            const int nu = (n + kWinRows - 1) / kWinRows;
            int incl = n, uincl = nu;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                const int uy = __shfl_up_sync(0xffffffffu, uincl, o);
                if (lane >= o) {
                    incl += y;
                    uincl += uy;
                }
            }
            if (i < nb) {
                bt[i] = BranchEnt{br.row0, br.stride, n, base + incl - n, br.depth, ubase + uincl - nu};
                for (int j = 0, rl = base + incl - n; j < n && rl < kRowTable; ++j, ++rl)
                    rowtab[rl] = br.row0 + j * br.stride;
            }
            const unsigned okm = __ballot_sync(0xffffffffu, i < nb && br.ok);
            if (seq < 0 && okm) seq = __shfl_sync(0xffffffffu, br.seq, __ffs(okm) - 1);
            base += __shfl_sync(0xffffffffu, incl, 31);
            ubase += __shfl_sync(0xffffffffu, uincl, 31);
        }
        if (lane == 0) {
            GroupInfo info{first, nb, seq, base, 0, 0, 0, 0, ubase, seq, 0};
            if (seq >= 0 && base > 0) {
                info.T = context_length(s.len, a.ctx, s.err, seq, split == 0 && h == 0);
                info.A = min(s.ws[seq], info.T);
                info.fp = s.fpos[seq];
                info.fb = info.fp > 0 ? s.fbase[seq] : seq;
                info.key_begin = split * a.chunk;
                info.key_end = min(info.A, info.key_begin + a.chunk);
            } else {
                info.nrows = 0;
                info.units = 0;
            }
            if (g == gridDim.x - 1 && a.ba.table && end < a.ba.nbranch)
                set_device_error(s.err, RIPE_DEVERR_BRANCH);  // more runs of sequences than CTAs
            *gi = info;
        }
    }
    __syncthreads();
    const GroupInfo G = *gi;
    const int ntiles = G.key_end > G.key_begin ? (G.key_end - G.key_begin + kN - 1) / kN : 0;
    const int nrt = (G.nrows + RT - 1) / RT;
    const int total_it = ntiles * nrt;
    // All-depths groups (k tokens x R depths of one sequence) are one block of Q rows.
    const int q_block =
        (a.q_tma && !a.ba.table && G.nrows == a.ba.k * s.R) ? g * a.ba.k * s.R : -1;

    if (warp < 6) {
        if (total_it > 0) {
            if (warp == 4) {
                // ------------------------------------------------ TMA producer
                if (lane == 0) {
                    // A fork's tiles below its fork position (a multiple of the tile) come from
                    // its parent's deep plane.
                    const int own_base = ((a.layer * s.Bmax + G.seq) * s.H + h) * s.Tmax + G.key_begin;
                    const int par_base = ((a.layer * s.Bmax + G.fb) * s.H + h) * s.Tmax + G.key_begin;
                    int issued = 0;
                    for (int it = 0; it < total_it; ++it) {
                        const int i = it % ntiles, st = it % ST;
                        if (it >= ST && !mbar_wait(kv_empty + st, ((it / ST) - 1) & 1, abort_flag, s.err)) break;
                        issued = it + 1;
                        const int y = (G.key_begin + i * kN < G.fp ? par_base : own_base) + i * kN;
                        mbar_expect_tx(k_full + st, Lay::KV_STAGE);
#pragma unroll
                        for (int c = 0; c < NCH; ++c)
                            tma_load_2d(sK + st * Lay::KV_STAGE + c * 4096, &tm.dk, 32 * c, y, k_full + st);
                        mbar_expect_tx(v_full + st, Lay::KV_STAGE);
#pragma unroll
                        for (int c = 0; c < NCH; ++c)
                            tma_load_2d(sV + st * Lay::KV_STAGE + c * 4096, &tm.dv, 32 * c, y, v_full + st);
                    }
                    if (*abort_flag) {
                        // Let the copies already issued land before the CTA's shared memory goes away.
                        volatile int no_abort = 0;
                        for (int it = issued > ST ? issued - ST : 0; it < issued; ++it) {
                            mbar_wait(k_full + it % ST, (it / ST) & 1, &no_abort, s.err);
                            mbar_wait(v_full + it % ST, (it / ST) & 1, &no_abort, s.err);
                        }
                    }
                }
            } else if (warp == 5) {
                // ------------------------------------------------ MMA issuer
                if (lane == 0) {
                    const uint32_t q0 = smem_u32(sQ), k0 = smem_u32(sK), v0 = smem_u32(sV);
                    auto issue_pv = [&](int t) -> bool {
                        const int st = t % ST, pb = t & 1, it_in_rt = t % ntiles;  // P of tile t in S buffer pb
                        if (!mbar_wait(p_full + pb, (t >> 1) & 1, abort_flag, s.err)) return false;
                        if (!mbar_wait(v_full + st, (t / ST) & 1, abort_flag, s.err)) return false;
                        tc_fence_after();
#pragma unroll
                        for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
                            for (int ks = 0; ks < kN / 16; ++ks) {
                                const uint64_t bd = smem_desc(v0 + st * Lay::KV_STAGE + ks * 1024, kN * 64, 512,
                                                              kLayoutSwizzle64B);
                                mma_bf16_ts(tmem + Lay::O_COL(mt), tmem + Lay::S_COL(mt, pb) + ks * 8, bd, IDESC_PV,
                                            (it_in_rt > 0 || ks > 0) ? 1u : 0u);
                            }
                        }
                        mma_commit(kv_empty + st);
                        mma_commit(pv_done + pb);
                        return true;
                    };
                    bool ok = true;
                    for (int it = 0; it < total_it && ok; ++it) {
                        const int i = it % ntiles, st = it % ST, sb = it & 1;
                        if (i == 0) {
                            // A new row tile: finish the previous one before waiting for its Q.
                            if (it > 0 && !(ok = issue_pv(it - 1))) break;
                            if (!mbar_wait(q_full, (it / ntiles) & 1, abort_flag, s.err)) {
                                ok = false;
                                break;
                            }
                        }
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
                        if (i > 0) ok = issue_pv(it - 1);
                    }
                    if (ok) issue_pv(total_it - 1);
                    // Every MMA issued so far has completed before TMEM is released.
                    volatile int no_abort = 0;
                    mma_commit(drain);
                    mbar_wait(drain, 0, &no_abort, s.err);
                }
            } else {
                // ------------------------------------------------ softmax + epilogue (warps 0-3)
                const int t = threadIdx.x;  // TMEM lane / row within an M tile
                const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
                const float c2 = a.scale_log2;
                float m[MT], l[MT];
                int rows[MT];
                bool ok = true;
                for (int it = 0; it < total_it && ok; ++it) {
                    const int i = it % ntiles, rt = it / ntiles, sb = it & 1;
                    if (i == 0 && Lay::QT) {
                        // Q into tensor memory: each thread its own row (TMEM lane t), loaded
                        // as 16-byte vectors and stored as D/2 columns of bf16 pairs.  The
                        // previous row tile's QK^T are done (its epilogue waited for them).
                        const int rl = rt * RT + t;
                        const int row = q_block >= 0 ? (rl < G.nrows ? q_block + rl : -1)
                                                     : group_row(rowtab, bt, G.nb, G.nrows, rl);
                        rows[0] = row;
                        m[0] = -INFINITY;
                        l[0] = 0.f;
                        const uint4* src = reinterpret_cast<const uint4*>(a.Q + ((int64_t)(row >= 0 ? row : 0) * s.H + h) * D * 2);
#pragma unroll
                        for (int c0 = 0; c0 < D / 2; c0 += 16) {
                            uint32_t w[16];
#pragma unroll
                            for (int v = 0; v < 4; ++v) {
                                const uint4 x = row >= 0 ? __ldg(src + c0 / 4 + v) : make_uint4(0, 0, 0, 0);
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
                    } else if (i == 0 && q_block >= 0) {
                        // The group's rows are one block of Q (all-depths form): M row t is
                        // Q row q_block + t; one thread loads the row tile by TMA, once the
                        // previous row tile's epilogue has left the Q buffer.
#pragma unroll
                        for (int mt = 0; mt < MT; ++mt) {
                            const int rl = rt * RT + mt * 128 + t;
                            rows[mt] = rl < G.nrows ? q_block + rl : -1;
                            m[mt] = -INFINITY;
                            l[mt] = 0.f;
                        }
                        if (t == 0) {
                            bool go = rt == 0 || mbar_wait(epi_done, (rt - 1) & 1, abort_flag, s.err);
                            if (go) {
                                mbar_expect_tx(q_full, MT * NCH * 8192);
#pragma unroll
                                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                                    for (int c = 0; c < NCH; ++c)
                                        tma_load_3d(sQ + mt * NCH * 8192 + c * 8192, &tm.q, 32 * c, h,
                                                    q_block + rt * RT + mt * 128, q_full);
                            }
                        } else {
                            mbar_arrive(q_full);
                        }
                    } else if (i == 0) {
                        // Rows of this row tile (each thread finds its own); the warp copies
                        // its 32 rows' Q, 16 bytes per lane in row order (coalesced), into
                        // the swizzled K-major layout.
#pragma unroll
                        for (int mt = 0; mt < MT; ++mt) {
                            const int row = group_row(rowtab, bt, G.nb, G.nrows, rt * RT + mt * 128 + t);
                            rows[mt] = row;
                            constexpr int QV = 2 * D / 16;  // 16-byte vectors per row
#pragma unroll 1
                            for (int e0 = 0; e0 < 32 * QV; e0 += 32) {
                                const int e = e0 + lane, r = e / QV, v = e - r * QV;
                                const int rrow = __shfl_sync(0xffffffffu, row, r);
                                const int tr = warp * 32 + r;  // TMEM lane / row within the M tile
                                uint8_t* dst = sQ + mt * NCH * 8192 + (v >> 2) * 8192 + tr * 64 +
                                               (((v & 3) ^ ((tr >> 1) & 3)) << 4);
                                const char* src =
                                    rrow >= 0 ? a.Q + ((int64_t)rrow * s.H + h) * D * 2 + v * 16 : a.Q;
                                cp_async16_zfill(dst, src, rrow >= 0);
                            }
                            m[mt] = -INFINITY;
                            l[mt] = 0.f;
                        }
                        cp_async_commit();
                        cp_async_wait_all();
                        fence_proxy_async_smem();
                        mbar_arrive(q_full);
                    }
                    if (!warp_wait(s_full + sb, (it >> 1) & 1, abort_flag, s.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int key0 = G.key_begin + i * kN;
                    const int nvalid = min(kN, G.key_end - key0);
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
                        // Row max of the raw scores (scale > 0 commutes with max), four chains.
                        float m4[4] = {sc[0], sc[1], sc[2], sc[3]};
#pragma unroll
                        for (int c = 4; c < kN; c += 4) {
                            m4[0] = fmaxf(m4[0], sc[c]);
                            m4[1] = fmaxf(m4[1], sc[c + 1]);
                            m4[2] = fmaxf(m4[2], sc[c + 2]);
                            m4[3] = fmaxf(m4[3], sc[c + 3]);
                        }
                        const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * c2;
                        // The running max moves only when it grows by more than 2^8 (probabilities
                        // then stay below 256); the O rescale is warp-collective.
                        float alpha = 1.f;
                        const bool grow = mx > m[mt] + 8.f;
                        if (grow) {
                            const float mn = fmaxf(mx, m[mt]);
                            alpha = ex2(m[mt] - mn);
                            m[mt] = mn;
                        }
                        // p = 2^(s*scale*log2e - m): one FMA and one ex2 per score.  P (bf16
                        // pairs) goes back into the first 32 columns of this tile's S buffer,
                        // the A operand of P V (the next write of the buffer, QK of tile
                        // it+2, follows P V of this tile in the MMA order).
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
                            // O holds this row tile's earlier tiles: rescale it once PV(it-1) is done
                            // (after P, so the scores no longer occupy registers).
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
                    if (i == ntiles - 1) {
                        // Row-tile epilogue: the partial (m, l, o) of every real row.
                        if (!warp_wait(pv_done + sb, (it >> 1) & 1, abort_flag, s.err)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        // Every MMA of the row tile is done, so this warp's own Q rows are
                        // free (other warps may already stage their next Q rows): the warp
                        // passes its rows through the first 2 KB of them, 8 rows x 32
                        // columns at a time, and stores 128-byte row pieces (coalesced).
                        constexpr int OSTR = 32 * 4 + 16;
                        static_assert(8 * OSTR <= 2048, "epilogue staging");
                        uint8_t* ostage = Lay::QT ? sm + Lay::OFF_OST + warp * 8 * OSTR : sQ + warp * 2048;
#pragma unroll
                        for (int mt = 0; mt < MT; ++mt) {
                            const int row = rows[mt];
                            const int64_t pi = row >= 0 ? ((int64_t)row * s.H + h) * a.nseg + split : -1;
                            if (row >= 0) a.part_ml[pi] = make_float2(m[mt], l[mt]);
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
                        // The staging stores come before any later TMA write of the Q buffer.
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(epi_done);
                        tc_fence_before();
                    }
                }
            }
        }
    } else if (G.units > 0) {
        // ------------------------------------------------ window warps
        constexpr int NKS = D / 16;  // k-steps of S^T = K Q^T
        constexpr int NMT = D / 16;  // 16-channel tiles of O^T
        const int ww = warp - 6;
        uint8_t* wbuf = sm + Lay::OFF_W + ww * NS * Lay::WSTAGE;
        uint64_t* wbar = reinterpret_cast<uint64_t*>(sm + Lay::OFF_WBAR) + ww * NS;
        const uint32_t wbuf_a = smem_u32(wbuf);
        const WinKeys wkeys = win_keys(G.A, G.T, s.Wcap);
        const int ustep = a.nsplit * NW;
        const int nunits = G.units;
        const float c2 = a.scale_log2;
        // Row indices, in the 2-D tensor-map views, of ring plane 1 slot 0 and of the
        // first window row of plane R.
        const int ring_y0 = ((a.layer * s.Bmax + G.seq) * s.H + h) * (s.R - 1) * s.Wcap;
        const int deep_y0 = ((a.layer * s.Bmax + G.seq) * s.H + h) * s.Tmax + G.A;
        const int deep_yp0 = ((a.layer * s.Bmax + G.fb) * s.H + h) * s.Tmax + G.A;  // fork parent
        const int q4 = lane & 3, r8 = lane >> 2;
        if (lane == 0) {
            prefetch_tmap(&tm.wk);
            prefetch_tmap(&tm.wv);
        }
        int iu = split + a.nsplit * ww;  // this warp's units: iu, iu + ustep, ...
        if (iu < nunits) {
            // Q^T fragments (B operand) of unit w straight from global memory:
            // b0 = Q[j0 + lane/4][16 ks + 2 q4 ..], b1 the same 8 channels on; rows past nr are 0.
            auto load_q = [&](const WinUnit& w, uint32_t (&b)[NKS][2]) {
                const bool okq = r8 < w.nr;
                const uint32_t* qp = reinterpret_cast<const uint32_t*>(
                    a.Q + (okq ? (((int64_t)w.row0 + (int64_t)(w.j0 + r8) * w.stride) * s.H + h) * (2 * D) : 0));
#pragma unroll
                for (int ks = 0; ks < NKS; ++ks) {
                    b[ks][0] = okq ? __ldg(qp + 8 * ks + q4) : 0u;
                    b[ks][1] = okq ? __ldg(qp + 8 * ks + 4 + q4) : 0u;
                }
            };
            // Tile t of unit w into stage `stage`, in the 64-byte-swizzled box layout
            // (row r, 16-byte chunk c of column block b at b*WBOX + r*64 + ((c ^ (r>>1 & 3)) << 4)).
            // Tiles of window keys only: one lane issues the TMA boxes.  Tiles that hold
            // draft-block keys: lane quads copy rows (zero-filling keys outside the
            // window or past the unit); each lane's arrival waits for its copies.
            auto issue = [&](const WinUnit& w, int t, int stage) {
                uint8_t* sb = wbuf + stage * Lay::WSTAGE;
                uint64_t* bar = wbar + stage;
                const bool ring = w.depth < s.R;
                const int k0t = t * kWinKeys;
                // deep rows of a tile on one side of a fork position come from one plane
                const bool one_owner = ring || ((G.A + k0t < G.fp) == (G.A + k0t + kWinKeys - 1 < G.fp));
                if (k0t + kWinKeys <= w.wk && one_owner) {
                    if (lane == 0) {
                        const int y = (ring ? ring_y0 + (w.depth - 1) * s.Wcap + w.lo
                                            : (G.A + k0t < G.fp ? deep_yp0 : deep_y0)) + k0t;
                        const CUtensorMap* mk = ring ? &tm.wk : &tm.rk;
                        const CUtensorMap* mv = ring ? &tm.wv : &tm.rv;
                        fence_proxy_async_smem();  // earlier reads of this stage come first
                        mbar_expect_tx(bar, Lay::WSTAGE);
#pragma unroll
                        for (int c = 0; c < NCH; ++c) {
                            tma_load_2d(sb + c * Lay::WBOX, mk, 32 * c, y, bar);
                            tma_load_2d(sb + Lay::WKV + c * Lay::WBOX, mv, 32 * c, y, bar);
                        }
                    } else {
                        mbar_arrive(bar);
                    }
                    return;
                }
                const int64_t wbase = ring ? ring_row(s, a.layer, G.seq, h, w.depth, w.lo)
                                           : deep_row(s, a.layer, G.seq, h, G.A);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int kr = half * 8 + r8;
                    const int key = k0t + kr;
                    const char* kp = a.Q;
                    const char* vp = a.Q;
                    bool ok;
                    if (key < w.wk) {
                        ok = win_valid(w, wkeys, s.R, s.Wcap, key);
                        const int64_t off = (!ring && G.A + key < G.fp ? deep_row(s, a.layer, G.fb, h, G.A) : wbase) +
                                            (int64_t)key * 2 * D + q4 * 16;
                        if (ok) {
                            kp = (ring ? s.kwin : s.kdeep) + off;
                            vp = (ring ? s.vwin : s.vdeep) + off;
                        }
                    } else {
                        ok = key < w.nk;
                        if (ok) {
                            const int64_t off =
                                (((int64_t)w.row0 + (int64_t)(key - w.wk) * w.stride) * s.H + h) * 2 * D + q4 * 16;
                            kp = a.Kb + off;
                            vp = a.Vb + off;
                        }
                    }
                    uint8_t* dk = sb + kr * 64 + ((q4 ^ ((kr >> 1) & 3)) << 4);
#pragma unroll
                    for (int j = 0; j < NCH; ++j) {
                        cp_async16_zfill(dk + j * Lay::WBOX, kp + (ok ? 64 * j : 0), ok);
                        cp_async16_zfill(dk + Lay::WKV + j * Lay::WBOX, vp + (ok ? 64 * j : 0), ok);
                    }
                }
                cp_async_mbar_arrive(bar);
            };

            WinUnit wi = win_unit(bt, G.nb, iu, wkeys, s.R, lane);
            WinUnit wc = wi;
            int cu = iu, it_ = 0, ct = 0;
            bool ihas = true;
            int issued = 0;  // tiles issued (stage q % NS holds tile q)
            auto advance_issue = [&]() {
                if (++it_ == wi.ntiles) {
                    iu += ustep;
                    it_ = 0;
                    if (iu < nunits)
                        wi = win_unit(bt, G.nb, iu, wkeys, s.R, lane);
                    else
                        ihas = false;
                }
            };

            uint32_t bq[NKS][2], bq_next[NKS][2];
            load_q(wc, bq_next);
            float o[NMT][4];
            float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
            const int ra = 2 * q4, rb = ra + 1;  // fragment columns (rows) of this lane
            // ldmatrix row addresses in the swizzled layout: K (A operand, rows = keys)
            // and V (A operand of O^T by .trans, rows = keys).
            const int rk = (lane & 7) + 8 * ((lane >> 3) & 1), rv = (lane & 7) + 8 * (lane >> 4);
            const uint32_t k_row = rk * 64, v_row = Lay::WKV + rv * 64;
            const uint32_t k_sw0 = (((lane >> 4) + 0) ^ ((rk >> 1) & 3)) << 4;
            const uint32_t k_sw1 = (((lane >> 4) + 2) ^ ((rk >> 1) & 3)) << 4;
            const uint32_t v_sw0 = ((((lane >> 3) & 1) + 0) ^ ((rv >> 1) & 3)) << 4;
            const uint32_t v_sw1 = ((((lane >> 3) & 1) + 2) ^ ((rv >> 1) & 3)) << 4;
            bool wok = true;
            // Iterations q < 0 only fill the first NS-1 stages (tile q+NS-1 into its stage).
            for (int q = 1 - NS;; ++q) {
                if (ihas) {
                    issue(wi, it_, (q + NS - 1) % NS);
                    ++issued;
                    advance_issue();
                }
                if (q < 0) continue;
                if (ct == 0) {
                    // A new unit: its Q^T fragments (loaded one unit ahead), the next unit's
                    // fragments in flight, a fresh accumulator.
#pragma unroll
                    for (int ks = 0; ks < NKS; ++ks) {
                        bq[ks][0] = bq_next[ks][0];
                        bq[ks][1] = bq_next[ks][1];
                    }
                    if (cu + ustep < nunits) load_q(win_unit(bt, G.nb, cu + ustep, wkeys, s.R, lane), bq_next);
#pragma unroll
                    for (int mt = 0; mt < NMT; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
                    m_a = m_b = -INFINITY;
                    l_a = l_b = 0.f;
                }
                if (!warp_wait(wbar + q % NS, (q / NS) & 1, abort_flag, s.err)) {
                    wok = false;
                    break;
                }
                const uint32_t sb = smem_ready(wbuf_a + (q % NS) * Lay::WSTAGE);
                // ---- S^T = K Q^T for 16 keys x 8 rows (two accumulation chains)
                float c[4] = {0.f, 0.f, 0.f, 0.f}, c_odd[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int ks = 0; ks < NKS; ++ks) {
                    uint32_t a0, a1, a2, a3;
                    ldsm_x4_r(sb + (ks >> 1) * Lay::WBOX + k_row + ((ks & 1) ? k_sw1 : k_sw0), a0, a1, a2, a3);
                    mma_16816((ks & 1) ? c_odd : c, a0, a1, a2, a3, bq[ks][0], bq[ks][1]);
                }
                float s0 = (c[0] + c_odd[0]) * c2, s1 = (c[1] + c_odd[1]) * c2;
                float s2 = (c[2] + c_odd[2]) * c2, s3 = (c[3] + c_odd[3]) * c2;
                // ---- visibility: window slots inside the window for every row, block
                // token j' for rows j >= j'.  Rows past nr are never written: unmasked.
                const int k0 = ct * kWinKeys + (lane >> 2), k1 = k0 + 8;
                const bool w0 = k0 < wc.wk && win_valid(wc, wkeys, s.R, s.Wcap, k0);
                const bool w1 = k1 < wc.wk && win_valid(wc, wkeys, s.R, s.Wcap, k1);
                if (!__all_sync(0xffffffffu, w0 && w1)) {
                    const int jr_a = wc.j0 + ra + wc.wk, jr_b = jr_a + 1;  // last visible key of rows ra, rb
                    const bool v0 = k0 < wc.wk ? w0 : k0 < wc.nk;
                    const bool v1 = k1 < wc.wk ? w1 : k1 < wc.nk;
                    if (!(v0 && (k0 < wc.wk || k0 <= jr_a))) s0 = -INFINITY;
                    if (!(v0 && (k0 < wc.wk || k0 <= jr_b))) s1 = -INFINITY;
                    if (!(v1 && (k1 < wc.wk || k1 <= jr_a))) s2 = -INFINITY;
                    if (!(v1 && (k1 < wc.wk || k1 <= jr_b))) s3 = -INFINITY;
                }
                // The running max m of a row moves only when a score exceeds it by more
                // than 2^8 (probabilities then stay below 256).  Only then is the tile's
                // row max reduced across the lanes; lanes of a row decide alike.
                const bool over = fmaxf(s0, s2) > m_a + 8.f || fmaxf(s1, s3) > m_b + 8.f;
                if (__any_sync(0xffffffffu, over)) {
                    float mx_a = fmaxf(s0, s2), mx_b = fmaxf(s1, s3);
#pragma unroll
                    for (int o2 = 4; o2 < 32; o2 <<= 1) {
                        mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, o2));
                        mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, o2));
                    }
                    if (mx_a > m_a + 8.f) {
                        const float al = ex2(m_a - mx_a);
                        m_a = mx_a;
                        l_a *= al;
#pragma unroll
                        for (int mt = 0; mt < NMT; ++mt) {
                            o[mt][0] *= al;
                            o[mt][2] *= al;
                        }
                    }
                    if (mx_b > m_b + 8.f) {
                        const float al = ex2(m_b - mx_b);
                        m_b = mx_b;
                        l_b *= al;
#pragma unroll
                        for (int mt = 0; mt < NMT; ++mt) {
                            o[mt][1] *= al;
                            o[mt][3] *= al;
                        }
                    }
                }
                const float p0 = m_a == -INFINITY ? 0.f : ex2(s0 - m_a);
                const float p1 = m_b == -INFINITY ? 0.f : ex2(s1 - m_b);
                const float p2 = m_a == -INFINITY ? 0.f : ex2(s2 - m_a);
                const float p3 = m_b == -INFINITY ? 0.f : ex2(s3 - m_b);
                l_a += p0 + p2;
                l_b += p1 + p3;
                // ---- O^T += V^T P^T: P^T by an 8x8 transpose of the S^T fragments
                const uint32_t b0 = movmatrix_t(pack_bf16(p0, p1));
                const uint32_t b1 = movmatrix_t(pack_bf16(p2, p3));
#pragma unroll
                for (int mt = 0; mt < NMT; ++mt) {
                    uint32_t a0, a1, a2, a3;
                    ldsm_x4_t_r(sb + (mt >> 1) * Lay::WBOX + v_row + ((mt & 1) ? v_sw1 : v_sw0), a0, a1, a2, a3);
                    mma_16816(o[mt], a0, a1, a2, a3, b0, b1);
                }
                if (ct == wc.ntiles - 1) {
                    // ---- the unit's partial: rows ra and rb of this lane's columns
#pragma unroll
                    for (int o2 = 4; o2 < 32; o2 <<= 1) {
                        l_a += __shfl_xor_sync(0xffffffffu, l_a, o2);
                        l_b += __shfl_xor_sync(0xffffffffu, l_b, o2);
                    }
                    const bool va = ra < wc.nr, vb = rb < wc.nr;
                    const int64_t pa =
                        (((int64_t)wc.row0 + (int64_t)(wc.j0 + ra) * wc.stride) * s.H + h) * a.nseg + a.nsplit;
                    const int64_t pb =
                        (((int64_t)wc.row0 + (int64_t)(wc.j0 + rb) * wc.stride) * s.H + h) * a.nseg + a.nsplit;
#pragma unroll
                    for (int mt = 0; mt < NMT; ++mt) {
                        const int ch = 16 * mt + (lane >> 2);
                        if (va) {
                            a.part_o[pa * D + ch] = o[mt][0];
                            a.part_o[pa * D + ch + 8] = o[mt][2];
                        }
                        if (vb) {
                            a.part_o[pb * D + ch] = o[mt][1];
                            a.part_o[pb * D + ch + 8] = o[mt][3];
                        }
                    }
                    if (lane < 4) {
                        if (va) a.part_ml[pa] = make_float2(m_a, l_a);
                        if (vb) a.part_ml[pb] = make_float2(m_b, l_b);
                    }
                }
                __syncwarp();
                if (++ct == wc.ntiles) {
                    cu += ustep;
                    if (cu >= nunits) break;
                    wc = win_unit(bt, G.nb, cu, wkeys, s.R, lane);
                    ct = 0;
                }
            }
            if (!wok) {
                // Let every issued tile land before the CTA's shared memory goes away.
                volatile int no_abort = 0;
                for (int qq = issued > NS ? issued - NS : 0; qq < issued; ++qq)
                    mbar_wait(wbar + qq % NS, (qq / NS) & 1, &no_abort, s.err);
            }
            cp_async_wait_all();
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5) tmem_dealloc(tmem, Lay::TMEM_COLS);

    // ---- merge: every partial of the cluster is written; this CTA merges rows
    // split, split + nsplit, ... (8 lanes per row, four rows per warp at a time).
    if (a.nsplit > 1) cluster_sync_all();
    if (G.nrows > 0 && !*abort_flag) {
        const int np = deep_splits_used(G.A, a.chunk, a.nsplit);
        const int sub = lane >> 3, sl = lane & 7;
        for (int k = warp * 4; split + a.nsplit * k < G.nrows; k += NWARPS * 4) {
            const int rl = split + a.nsplit * (k + sub);
            const int row = group_row(rowtab, bt, G.nb, G.nrows, rl);
            const bool ok = row >= 0;
            const int64_t ro = ok ? (int64_t)row * s.H + h : 0;
            if (np < 3)
                merge_rows<D, 3, 1>(a, &ro, &ok, np, sl);
            else if (ok)
                merge_row_any<D>(a.part_ml, a.part_o, a.O, a.lse, a.nseg, a.nsplit, ro, np, sl);
        }
    }
}

template <int D, int MT, int ST, int NW, int NS>
cudaError_t launch_t(const TMaps& tm, const VerifyArgs& a, int gslots, bool pdl, cudaStream_t st) {
    using Lay = FusedLayout<D, MT, ST, NW, NS>;
    static_assert(Lay::SMEM <= 232448, "shared memory budget");
    static PerDeviceOnce configured;
    cudaError_t ce = per_device_once(configured, [] {
        cudaError_t e = cudaFuncSetAttribute(verify_kernel<D, MT, ST, NW, NS>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::SMEM);
        if (e != cudaSuccess) return e;
        return cudaFuncSetAttribute(verify_kernel<D, MT, ST, NW, NS>,
                                    cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    });
    if (ce != cudaSuccess) return ce;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(gslots, a.s.H, a.nsplit);
    cfg.blockDim = dim3(Lay::THREADS);
    cfg.dynamicSmemBytes = Lay::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int n = 0;
    if (a.nsplit > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = 1;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = a.nsplit;
        ++n;
    }
    if (pdl) {
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    cudaError_t e = cudaLaunchKernelEx(&cfg, verify_kernel<D, MT, ST, NW, NS>, tm, a);
    ripe_count_launch();
    return e;
}

}  // namespace

typedef CUresult (*EncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                             const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                             CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled from the driver (looked up once), or NULL.
static EncodeFn encode_fn() {
    static EncodeFn encode = nullptr;
    if (!encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess && fn)
            encode = reinterpret_cast<EncodeFn>(fn);
    }
    return encode;
}

bool fused_supported(int dtype, int d) { return dtype == RIPE_BF16 && (d == 64 || d == 96 || d == 128); }

// This call's Q viewed as [rows][H][d]: boxes of 128 rows x 32 columns of one head
// (the stacked-query tile of the deep region).
bool make_q_map(void* tmap, const VerifyArgs& a) {
    const EncodeFn encode = encode_fn();
    if (!encode) return false;
    const int d = a.s.d;
    const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)a.s.H, (cuuint64_t)a.ba.nrows};
    const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)a.s.H * d * 2};
    const cuuint32_t box[3] = {32, 1, 128};
    const cuuint32_t estr[3] = {1, 1, 1};
    return encode(reinterpret_cast<CUtensorMap*>(tmap), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<char*>(a.Q),
                  dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_fused(const void* tmaps, const VerifyArgs& args, int gslots, int mt, bool pdl, cudaStream_t st) {
    // The cache's first six maps plus one of this call's Q.
    TMaps tm;
    memcpy(&tm, tmaps, 6 * sizeof(CUtensorMap));
    VerifyArgs a = args;
    a.q_tma = make_q_map(&tm.q, a) ? 1 : 0;
    const int d = a.s.d;
    // <D, M tiles, deep stages, window warps, window stages>, each within 227 KB of shared memory.
    if (mt == 1) {
        if (d == 64) return launch_t<64, 1, 4, 8, 3>(tm, a, gslots, pdl, st);
        if (d == 96) return launch_t<96, 1, 3, 8, 3>(tm, a, gslots, pdl, st);
        if (d == 128) return launch_t<128, 1, 3, 5, 2>(tm, a, gslots, pdl, st);
    } else {
        if (d == 64) return launch_t<64, 2, 4, 8, 2>(tm, a, gslots, pdl, st);
        if (d == 96) return launch_t<96, 2, 3, 6, 2>(tm, a, gslots, pdl, st);
        if (d == 128) return launch_t<128, 2, 2, 4, 2>(tm, a, gslots, pdl, st);
    }
    return cudaErrorInvalidValue;
}

// Tensor maps: 2-D [rows][d] bf16 views, 32-column boxes with the 64-byte swizzle
// the kernels' shared-memory layouts expect.  Deep planes (rows = L*Bmax*H*Tmax)
// in 64-row boxes (deep region) and 16-row boxes (window tiles at depth R); ring
// planes (rows = L*Bmax*H*(R-1)*Wcap) in 16-row boxes; ring and deep planes again
// in 8-row boxes and in Wcap-row boxes for the persistent kernel.  Rows past the
// end of a view read as zeros.
int make_tensor_maps(ripe_cache_s* c) {
    const EncodeFn encode = encode_fn();
    if (!encode) return -1;
    static_assert(sizeof(c->tmaps) == 14 * sizeof(CUtensorMap), "tensor map bundle");
    const cuuint64_t deep_rows = (cuuint64_t)c->L * c->Bmax * c->H * c->Tmax;
    const cuuint64_t ring_rows = (cuuint64_t)c->L * c->Bmax * c->H * (c->R - 1) * c->Wcap;
    if (deep_rows >= (1ull << 31) || ring_rows >= (1ull << 31)) return -2;
    const cuuint64_t strides[1] = {(cuuint64_t)c->d * 2};
    const cuuint32_t estr[2] = {1, 1};
    struct Spec {
        void* base;
        cuuint64_t rows;
        cuuint32_t box_rows;
    };
    // With no ring planes (R = 1) the ring maps are never used; they alias the deep planes.
    const bool ring = ring_rows > 0;
    // A whole ring plane (Wcap rows) per box when that fits a box (<= 256 rows).
    c->full_box = c->Wcap <= 256;
    const cuuint32_t full_rows = (cuuint32_t)(c->full_box ? c->Wcap : 256);
    const Spec spec[14] = {{c->kdeep, deep_rows, (cuuint32_t)kN},
                           {c->vdeep, deep_rows, (cuuint32_t)kN},
                           {ring ? c->kwin : c->kdeep, ring ? ring_rows : deep_rows, (cuuint32_t)kWinKeys},
                           {ring ? c->vwin : c->vdeep, ring ? ring_rows : deep_rows, (cuuint32_t)kWinKeys},
                           {c->kdeep, deep_rows, (cuuint32_t)kWinKeys},
                           {c->vdeep, deep_rows, (cuuint32_t)kWinKeys},
                           {ring ? c->kwin : c->kdeep, ring ? ring_rows : deep_rows, 8u},
                           {ring ? c->vwin : c->vdeep, ring ? ring_rows : deep_rows, 8u},
                           {c->kdeep, deep_rows, 8u},
                           {c->vdeep, deep_rows, 8u},
                           {ring ? c->kwin : c->kdeep, ring ? ring_rows : deep_rows, full_rows},
                           {ring ? c->vwin : c->vdeep, ring ? ring_rows : deep_rows, full_rows},
                           {c->kdeep, deep_rows, full_rows},
                           {c->vdeep, deep_rows, full_rows}};
    for (int i = 0; i < 14; ++i) {
        const cuuint64_t dims[2] = {(cuuint64_t)c->d, spec[i].rows};
        const cuuint32_t box[2] = {32, spec[i].box_rows};
        CUresult r = encode(reinterpret_cast<CUtensorMap*>(c->tmaps[i]), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                            spec[i].base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return -3;
    }
    return 0;
}
