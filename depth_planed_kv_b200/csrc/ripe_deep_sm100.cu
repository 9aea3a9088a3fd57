// ripe_deep_sm100.cu -- the deep region of RIPE verify-attention on the sm_100a
// tensor cores.
//
// Outside the window every query row of a sequence -- all draft tokens at all
// loop depths, and every LoopSpec branch -- reads the same deepest plane R
// (RIPE abstract, sentence introducing RIPE; LoopSpec article on mixed-depth
// branches in one batched call).  Stacking those rows turns the read into a dense
// contraction: one CTA takes up to 128 (or 2 x 128) rows of one sequence and
// head against a chunk of the deep plane and runs
//     S = Q K^T (tcgen05.mma, fp32 in TMEM) -> online softmax on CUDA cores ->
//     O += P V (tcgen05.mma, fp32 in TMEM)
// with K and V streamed by TMA through a ring of shared-memory stages.  The
// result is one partial (max m in log2 units, sum l, unnormalised o) per row,
// merged later with the window/block partial.
//
// Roles (192 threads): warps 0-3 own TMEM lanes 0-127 (one query row each; with
// two M tiles, rows i and 128+i) and do Q staging, softmax and the epilogue;
// warp 4 lane 0 issues TMA; warp 5 allocates TMEM and lane 0 issues the MMAs.
//
// Shared-memory operand layouts (all 64-byte swizzle, 8-row / 512-byte atoms):
//   Q, K: K-major, 32-element column chunks of [rows][64 B];
//   V:    MN-major: the same [keys][64 B] chunks read with head-dim as N;
//   P:    K-major [128 rows][32 keys] chunks written by the softmax threads.
#include <cuda.h>

#include "ripe_launch.h"
#include "ripe_verify.cuh"
#include "sm100_ptx.cuh"

namespace {

constexpr int kN = 64;  // keys per tile
constexpr int kThreads = 192;
constexpr int kMaxGroupBranches = 64;  // branches of one sequence in one call
constexpr int kWinRows = 16;           // rows per CTA of the window kernel (its row chunks)

template <int D, int MT, int ST>
struct DeepLayout {
    static constexpr int NCH = D / 32;               // 64-byte column chunks of the head dim
    static constexpr int Q_BYTES = MT * NCH * 8192;  // 128 rows x 64 B per chunk
    static constexpr int KV_STAGE = NCH * 4096;      // 64 keys x 64 B per chunk
    static constexpr int P_BUF = 2 * 8192;           // one M tile: 2 chunks of 32 keys
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + Q_BYTES;
    static constexpr int OFF_V = OFF_K + ST * KV_STAGE;
    static constexpr int OFF_P = OFF_V + ST * KV_STAGE;
    static constexpr int OFF_BAR = OFF_P + 2 * MT * P_BUF;
    // barriers: q_full, k_full[ST], v_full[ST], kv_empty[ST], s_full[2], p_full[2], pv_done[2], drain
    static constexpr int NBAR = 1 + 3 * ST + 7;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int OFF_BT = OFF_MISC + 64;           // branch table of the group
    static constexpr int BYTES = OFF_BT + kMaxGroupBranches * 20;
    static constexpr int SMEM = BYTES + 1024;  // alignment slack
    static constexpr uint32_t TMEM_COLS = MT == 1 ? 256 : 512;
    static constexpr uint32_t S_COL(int mt, int sb) { return (uint32_t)((mt * 2 + sb) * kN); }
    static constexpr uint32_t O_COL(int mt) { return (uint32_t)(MT * 2 * kN + mt * 128); }
};

struct GroupInfo {
    int first, nb, seq, nrows, T, A, key_begin, key_end;
};

// One branch of the group: its rows, its offset among the group's rows, and the
// mask of its window-kernel row chunks whose merge falls to this CTA.
struct BranchEnt {
    int row0, stride, ntok, off, last_mask;
};

// Warp-uniform bounded wait: every lane waits, and all lanes agree on the outcome
// (the tcgen05.ld/st that follow are warp-collective).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int32_t* err) {
    const bool ok = sm100::mbar_wait(bar, parity, abort, err);
    return __all_sync(0xffffffffu, ok);
}

// Row (of Q/O) of the group's rl-th query, branches in table order; -1 past the end.
__device__ int group_row(const BranchEnt* bt, int nb, int rl, int* bidx = nullptr, int* jout = nullptr) {
    for (int i = 0; i < nb; ++i) {
        if (rl < bt[i].off + bt[i].ntok) {
            const int j = rl - bt[i].off;
            if (bidx) *bidx = i;
            if (jout) *jout = j;
            return bt[i].row0 + j * bt[i].stride;
        }
    }
    return -1;
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

template <int D, int MT, int ST>
__global__ void __launch_bounds__(kThreads, 1)
deep_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, VerifyArgs a) {
    using Lay = DeepLayout<D, MT, ST>;
    using namespace sm100;
    constexpr int NCH = Lay::NCH;
    constexpr int RT = 128 * MT;
    constexpr uint32_t IDESC_QK = idesc_bf16(128, kN, 0);
    constexpr uint32_t IDESC_PV = idesc_bf16(128, D, 1);

    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = sm + Lay::OFF_Q;
    uint8_t* sK = sm + Lay::OFF_K;
    uint8_t* sV = sm + Lay::OFF_V;
    uint8_t* sP = sm + Lay::OFF_P;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Lay::OFF_BAR);
    uint64_t* q_full = bars;
    uint64_t* k_full = bars + 1;
    uint64_t* v_full = bars + 1 + ST;
    uint64_t* kv_empty = bars + 1 + 2 * ST;
    uint64_t* s_full = bars + 1 + 3 * ST;
    uint64_t* p_full = s_full + 2;
    uint64_t* pv_done = s_full + 4;
    uint64_t* drain = s_full + 6;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Lay::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + Lay::OFF_MISC + 4);
    GroupInfo* gi = reinterpret_cast<GroupInfo*>(sm + Lay::OFF_MISC + 16);
    BranchEnt* bt = reinterpret_cast<BranchEnt*>(sm + Lay::OFF_BT);

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
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 5) {
        tmem_alloc(tmem_slot, Lay::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 4 && lane == 0) {
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    grid_dependency_wait();
    grid_launch_dependents();

    // ---- the group of branches this CTA serves (one sequence) and its key range
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
        // Branch entries loaded in parallel, row offsets by a warp prefix sum.
        int seq = -1, base = 0;
        for (int c0 = 0; c0 < nb; c0 += 32) {
            const int i = c0 + lane;
            Branch br;
            br.ok = false;
            if (i < nb) br = load_branch(a.ba, s.R, s.Bmax, first + i);
            const int n = (i < nb && br.ok) ? br.ntok : 0;
            int incl = n;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            if (i < nb) bt[i] = BranchEnt{br.row0, br.stride, n, base + incl - n, 0};
            const unsigned okm = __ballot_sync(0xffffffffu, i < nb && br.ok);
            if (seq < 0 && okm) seq = __shfl_sync(0xffffffffu, br.seq, __ffs(okm) - 1);
            base += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) {
            GroupInfo info{first, nb, seq, base, 0, 0, 0, 0};
            if (seq >= 0 && base > 0) {
                info.T = context_length(s.len, a.ctx, s.err, seq, false);
                info.A = min(s.ws[seq], info.T);
                info.key_begin = split * a.chunk;
                info.key_end = min(info.A, info.key_begin + a.chunk);
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
    const int total_it = G.seq >= 0 ? ntiles * nrt : 0;

    if (total_it > 0) {
        if (warp == 4) {
            // ------------------------------------------------ TMA producer
            if (lane == 0) {
                const int row_base = ((a.layer * s.Bmax + G.seq) * s.H + h) * s.Tmax + G.key_begin;
                int issued = 0;
                for (int it = 0; it < total_it; ++it) {
                    const int i = it % ntiles, st = it % ST;
                    if (it >= ST && !mbar_wait(kv_empty + st, ((it / ST) - 1) & 1, abort_flag, s.err)) break;
                    issued = it + 1;
                    const int y = row_base + i * kN;
                    mbar_expect_tx(k_full + st, Lay::KV_STAGE);
#pragma unroll
                    for (int c = 0; c < NCH; ++c)
                        tma_load_2d(sK + st * Lay::KV_STAGE + c * 4096, &tmK, 32 * c, y, k_full + st);
                    mbar_expect_tx(v_full + st, Lay::KV_STAGE);
#pragma unroll
                    for (int c = 0; c < NCH; ++c)
                        tma_load_2d(sV + st * Lay::KV_STAGE + c * 4096, &tmV, 32 * c, y, v_full + st);
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
                const uint32_t q0 = smem_u32(sQ), k0 = smem_u32(sK), v0 = smem_u32(sV), p0 = smem_u32(sP);
                auto issue_pv = [&](int t) -> bool {
                    const int st = t % ST, pb = t & 1, it_in_rt = t % ntiles;
                    if (!mbar_wait(p_full + pb, (t >> 1) & 1, abort_flag, s.err)) return false;
                    if (!mbar_wait(v_full + st, (t / ST) & 1, abort_flag, s.err)) return false;
                    tc_fence_after();
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
                        for (int ks = 0; ks < kN / 16; ++ks) {
                            const uint64_t ad = smem_desc(p0 + (pb * MT + mt) * Lay::P_BUF + (ks >> 1) * 8192 +
                                                              (ks & 1) * 32, 16, 512, kLayoutSwizzle64B);
                            const uint64_t bd = smem_desc(v0 + st * Lay::KV_STAGE + ks * 1024, kN * 64, 512,
                                                          kLayoutSwizzle64B);
                            mma_bf16(tmem + Lay::O_COL(mt), ad, bd, IDESC_PV, (it_in_rt > 0 || ks > 0) ? 1u : 0u);
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
                        if (!mbar_wait(q_full, (it / ntiles) & 1, abort_flag, s.err)) { ok = false; break; }
                    }
                    if (!mbar_wait(k_full + st, (it / ST) & 1, abort_flag, s.err)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
                        for (int ks = 0; ks < D / 16; ++ks) {
                            const uint32_t off = (ks & 1) * 32;
                            const uint64_t ad = smem_desc(q0 + mt * NCH * 8192 + (ks >> 1) * 8192 + off, 16, 512,
                                                          kLayoutSwizzle64B);
                            const uint64_t bd = smem_desc(k0 + st * Lay::KV_STAGE + (ks >> 1) * 4096 + off, 16, 512,
                                                          kLayoutSwizzle64B);
                            mma_bf16(tmem + Lay::S_COL(mt, sb), ad, bd, IDESC_QK, ks > 0 ? 1u : 0u);
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
                if (i == 0) {
                    // Rows of this row tile (each thread finds its own), then their Q into
                    // the swizzled K-major layout.
                    for (int mt = 0; mt < MT; ++mt) {
                        const int row = group_row(bt, G.nb, rt * RT + mt * 128 + t);
                        rows[mt] = row;
                        uint8_t* dst = sQ + mt * NCH * 8192 + t * 64;
                        const uint4* src = row >= 0
                            ? reinterpret_cast<const uint4*>(a.Q + ((int64_t)row * s.H + h) * D * 2) : nullptr;
#pragma unroll
                        for (int c = 0; c < NCH; ++c) {
#pragma unroll
                            for (int gq = 0; gq < 4; ++gq) {
                                const uint4 v = src ? src[c * 4 + gq] : make_uint4(0, 0, 0, 0);
                                *reinterpret_cast<uint4*>(dst + c * 8192 + ((gq ^ ((t >> 1) & 3)) << 4)) = v;
                            }
                        }
                        m[mt] = -INFINITY;
                        l[mt] = 0.f;
                    }
                    fence_proxy_async_smem();
                    mbar_arrive(q_full);
                }
                if (!warp_wait(s_full + sb, (it >> 1) & 1, abort_flag, s.err)) { ok = false; break; }
                tc_fence_after();
                const int key0 = G.key_begin + i * kN;
                const int nvalid = min(kN, G.key_end - key0);
                if (it >= 2 && !warp_wait(pv_done + sb, ((it - 2) >> 1) & 1, abort_flag, s.err)) { ok = false; break; }
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
                    if (i > 0 && __any_sync(0xffffffffu, grow)) {
                        // O holds this row tile's earlier tiles: rescale it once PV(it-1) is done.
                        if (!warp_wait(pv_done + ((it - 1) & 1), ((it - 1) >> 1) & 1, abort_flag, s.err)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
#pragma unroll
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
                    // p = 2^(s*scale*log2e - m): one FMA and one ex2 per score.
                    const float nm = -m[mt];
                    float s4[4] = {0.f, 0.f, 0.f, 0.f};
                    uint8_t* prow = sP + (sb * MT + mt) * Lay::P_BUF + t * 64;
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
#pragma unroll
                        for (int gq = 0; gq < 4; ++gq) {
                            uint32_t w[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float x0 = ex2(fmaf(sc[c * 32 + gq * 8 + 2 * e], c2, nm));
                                const float x1 = ex2(fmaf(sc[c * 32 + gq * 8 + 2 * e + 1], c2, nm));
                                s4[e] += x0 + x1;
                                __nv_bfloat162 b2 = __floats2bfloat162_rn(x0, x1);
                                w[e] = *reinterpret_cast<uint32_t*>(&b2);
                            }
                            *reinterpret_cast<uint4*>(prow + c * 8192 + ((gq ^ ((t >> 1) & 3)) << 4)) =
                                make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    }
                    l[mt] = l[mt] * alpha + ((s4[0] + s4[1]) + (s4[2] + s4[3]));
                }
                if (!ok) break;
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(p_full + sb);
                if (i == ntiles - 1) {
                    // Row-tile epilogue: the partial (m, l, o) of every real row.
                    if (!warp_wait(pv_done + sb, (it >> 1) & 1, abort_flag, s.err)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) {
                        const int row = rows[mt];
                        float o[D];
#pragma unroll
                        for (int c0 = 0; c0 < D; c0 += 32) tmem_ld32(lane_addr + Lay::O_COL(mt) + c0, o + c0);
                        tmem_wait_ld();
                        if (row >= 0) {
                            const int64_t pi = ((int64_t)row * s.H + h) * a.nseg + split;
                            a.part_ml[pi] = make_float2(m[mt], l[mt]);
                            float4* dst = reinterpret_cast<float4*>(a.part_o + pi * D);
#pragma unroll
                            for (int c = 0; c < D / 4; ++c)
                                dst[c] = make_float4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
                        }
                    }
                    tc_fence_before();
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5) tmem_dealloc(tmem, Lay::TMEM_COLS);

    // ---- count this split's arrival for every (branch, window row chunk) of the
    // group; where it is the last contributor, merge those rows.
    if (total_it > 0 && !*abort_flag) {
        const int ndeep = deep_splits_used(G.A, a.chunk, a.nsplit);
        if (warp == 0) {
            __threadfence();  // releases the partials written before the barrier above
            for (int i = lane; i < G.nb; i += 32) {
                int mask = 0;
                const int nrc = (bt[i].ntok + kWinRows - 1) / kWinRows;
                for (int rc = 0; rc < nrc; ++rc) {
                    int* cnt = a.cnt + ((int64_t)(G.first + i) * a.nrowchunks + rc) * s.H + h;
                    if (atomicAdd(cnt, 1) == ndeep) {
                        *cnt = 0;
                        mask |= 1 << rc;
                    }
                }
                bt[i].last_mask = mask;
            }
            __threadfence();
        }
        __syncthreads();
        const int nseg = a.nseg;
        for (int rl = threadIdx.x; rl < G.nrows; rl += kThreads) {
            int bi = 0, j = 0;
            const int row = group_row(bt, G.nb, rl, &bi, &j);
            if (row < 0 || !((bt[bi].last_mask >> (j / kWinRows)) & 1)) continue;
            const int64_t base = ((int64_t)row * s.H + h) * nseg;
            // Deep splits in order, then the window partial -- the same operation order as
            // the window-side merge, so the result does not depend on who merges.
            float mls[2 * 9];
            const int np = ndeep < 8 ? ndeep : 8;
            float M = -INFINITY;
            for (int sg = 0; sg <= np; ++sg) {
                const float2 ml = __ldcg(a.part_ml + base + (sg < np ? sg : a.nsplit));
                mls[2 * sg] = ml.x;
                mls[2 * sg + 1] = ml.y;
            }
            for (int sg = 0; sg < np; ++sg) M = fmaxf(M, mls[2 * sg]);
            M = fmaxf(M, mls[2 * np]);
            float L = 0.f;
            for (int sg = 0; sg <= np; ++sg) {
                mls[2 * sg] = ex2(mls[2 * sg] - M);
                L = fmaf(mls[2 * sg + 1], mls[2 * sg], L);
            }
            __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.O) + ((int64_t)row * s.H + h) * D;
#pragma unroll 2
            for (int c = 0; c < D; c += 8) {
                float acc[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = 0.f;
                for (int sg = 0; sg <= np; ++sg) {
                    const float4* src = reinterpret_cast<const float4*>(
                        a.part_o + (base + (sg < np ? sg : a.nsplit)) * D + c);
                    const float4 x0 = __ldcg(src), x1 = __ldcg(src + 1);
                    const float f = mls[2 * sg];
                    acc[0] = fmaf(x0.x, f, acc[0]); acc[1] = fmaf(x0.y, f, acc[1]);
                    acc[2] = fmaf(x0.z, f, acc[2]); acc[3] = fmaf(x0.w, f, acc[3]);
                    acc[4] = fmaf(x1.x, f, acc[4]); acc[5] = fmaf(x1.y, f, acc[5]);
                    acc[6] = fmaf(x1.z, f, acc[6]); acc[7] = fmaf(x1.w, f, acc[7]);
                }
                uint32_t w4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[2 * e] / L, acc[2 * e + 1] / L);
                    w4[e] = *reinterpret_cast<uint32_t*>(&b2);
                }
                *reinterpret_cast<uint4*>(orow + c) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
            if (a.lse) a.lse[(int64_t)row * s.H + h] = (M + log2f(L)) * 0.69314718055994531f;
        }
    }
}

template <int D, int MT, int ST>
cudaError_t launch_deep_t(const CUtensorMap& tk, const CUtensorMap& tv, const VerifyArgs& a, int gslots, bool pdl,
                          cudaStream_t st) {
    using Lay = DeepLayout<D, MT, ST>;
    static_assert(Lay::SMEM <= 232448, "shared memory budget");
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(deep_kernel<D, MT, ST>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             Lay::SMEM);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(deep_kernel<D, MT, ST>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(gslots, a.s.H, a.nsplit);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = Lay::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    cudaError_t e = cudaLaunchKernelEx(&cfg, deep_kernel<D, MT, ST>, tk, tv, a);
    ripe_count_launch();
    return e;
}

}  // namespace

bool deep_tc_supported(int dtype, int d) {
    return dtype == RIPE_BF16 && (d == 64 || d == 96 || d == 128);
}

cudaError_t launch_deep_tc(const void* tmK, const void* tmV, const VerifyArgs& a, int gslots, int mt, bool pdl,
                           cudaStream_t st) {
    const CUtensorMap& tk = *reinterpret_cast<const CUtensorMap*>(tmK);
    const CUtensorMap& tv = *reinterpret_cast<const CUtensorMap*>(tmV);
    const int d = a.s.d;
    if (mt == 1) {
        if (d == 64) return launch_deep_t<64, 1, 4>(tk, tv, a, gslots, pdl, st);
        if (d == 96) return launch_deep_t<96, 1, 3>(tk, tv, a, gslots, pdl, st);
        if (d == 128) return launch_deep_t<128, 1, 3>(tk, tv, a, gslots, pdl, st);
    } else {
        if (d == 64) return launch_deep_t<64, 2, 4>(tk, tv, a, gslots, pdl, st);
        if (d == 96) return launch_deep_t<96, 2, 3>(tk, tv, a, gslots, pdl, st);
        if (d == 128) return launch_deep_t<128, 2, 3>(tk, tv, a, gslots, pdl, st);
    }
    return cudaErrorInvalidValue;
}

// Tensor maps of the deep planes: 2-D [rows = L*Bmax*H*Tmax][d] bf16, box 32 x 64
// with the 64-byte swizzle the MMA descriptors above expect.
int make_deep_tensor_maps(ripe_cache_s* c) {
    typedef CUresult (*EncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
    static EncodeFn encode = nullptr;
    if (!encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
            return -1;
        encode = reinterpret_cast<EncodeFn>(fn);
    }
    const cuuint64_t rows = (cuuint64_t)c->L * c->Bmax * c->H * c->Tmax;
    if (rows >= (1ull << 31)) return -2;
    const cuuint64_t dims[2] = {(cuuint64_t)c->d, rows};
    const cuuint64_t strides[1] = {(cuuint64_t)c->d * 2};
    const cuuint32_t box[2] = {32, (cuuint32_t)kN};
    const cuuint32_t estr[2] = {1, 1};
    CUtensorMap* maps[2] = {reinterpret_cast<CUtensorMap*>(c->tmap_k), reinterpret_cast<CUtensorMap*>(c->tmap_v)};
    void* bases[2] = {c->kdeep, c->vdeep};
    for (int i = 0; i < 2; ++i) {
        CUresult r = encode(maps[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, bases[i], dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return -3;
    }
    return 0;
}
