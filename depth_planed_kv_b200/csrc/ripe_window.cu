// ripe_window.cu -- the window planes and the draft block of RIPE verify-attention
// on CUDA cores, and the final merge of each row's partial results.
//
// A query at loop depth r reads plane r of the positions still inside the window
// (RIPE abstract, sentence introducing RIPE) and the draft-block tokens of its own
// branch at plane r.  Those keys differ from depth to depth, so there is nothing
// to stack across rows: one CTA takes the k (<= 16) rows of one branch and head,
// and the work is 4-16 dot products per key -- CUDA-core territory.
//
// Data movement: the CTA's keys (a run of ring slots that wraps at most once, or a
// run of the deep plane for rows at depth R, then the block tokens) arrive by
// 16-byte asynchronous copies spread over all threads: K rows land at a padded
// stride (an odd number of 16-byte units, so one 16-byte vector per lane hits
// distinct banks), V rows densely.  (Bulk copies of single 192-byte rows were
// tried first: the copy engine then becomes the bottleneck.)
// Compute per tile: scores with thread = key (K row read once, q broadcast from
// shared memory), the online softmax with warp = row, P.V with thread = channel.
//
// Merge: the window CTA and the deep CTAs of the same (branch, row chunk, head)
// each write a partial (m, l, o) and then count their arrival; whoever arrives
// last merges -- M = max m, L = sum l 2^(m-M), O = sum o 2^(m-M) / L -- and
// writes O and the LSE.  No one waits for anyone.
#include "ripe_launch.h"
#include "ripe_verify.cuh"
#include "sm100_ptx.cuh"

namespace {

constexpr int kThreads = 128;
constexpr int kRowChunk = 16;  // rows of a branch per window CTA (the launch's row chunks)

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

template <int D, int NR>
struct WinLayout {
    static constexpr int ROWB = D * 2;       // bf16 row
    static constexpr int KSTR = ROWB + 16;   // padded K row stride: odd number of 16-byte units
    static constexpr int NVEC = ROWB / 16;
    // K tile, V tile, q rows (fp32), scores [row][key], probabilities [key][row], (m, l) per row
    static size_t bytes(int KT) {
        return 128 + (size_t)KT * (KSTR + ROWB) + (size_t)NR * D * 4 + (size_t)2 * NR * KT * 4 + NR * 8;
    }
};

// NR = rows per CTA (4, 8 or 16): every row loop has a compile-time trip count.
template <int D, int NR>
__global__ void __launch_bounds__(kThreads) window_kernel(VerifyArgs a, int KT) {
    using namespace sm100;
    using Lay = WinLayout<D, NR>;
    constexpr int kRows = NR;
    constexpr int ROWB = Lay::ROWB, KSTR = Lay::KSTR, NVEC = Lay::NVEC;
    extern __shared__ __align__(128) uint8_t smem[];
    int* flags = reinterpret_cast<int*>(smem + 8);  // [0] merge here, [1] abort
    uint8_t* sK = smem + 128;
    uint8_t* sV = sK + (size_t)KT * KSTR;
    float* q_s = reinterpret_cast<float*>(sV + (size_t)KT * ROWB);
    float* sc = q_s + kRows * D;                // scores, [row][key]
    float* pt = sc + (size_t)kRows * KT;        // probabilities, [key][row]
    float* alph = pt + (size_t)kRows * KT;

    const StoreView& s = a.s;
    const int H = s.H;
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    int w = blockIdx.x;
    const int h = w % H; w /= H;
    const int rc = w % a.nrowchunks;
    const int bi = w / a.nrowchunks;

    const Branch br = load_branch(a.ba, s.R, s.Bmax, bi);
    if (!br.ok && tid == 0 && rc == 0 && h == 0) set_device_error(s.err, RIPE_DEVERR_BRANCH);
    const int j0 = rc * kRowChunk;
    const bool active = br.ok && j0 < br.ntok;

    if (active) {
        const int nr = min(kRows, br.ntok - j0);
        const int b = br.seq, r = br.depth;
        const int T = context_length(s.len, a.ctx, s.err, b, h == 0 && rc == 0 && tid == 0);
        const int A = min(s.ws[b], T);
        const int nwin = T - A;
        const int nk = nwin + j0 + nr;  // block tokens 0..j0+nr-1 are visible to some row here
        const bool ring = r < s.R;
        const int ntile = (nk + KT - 1) / KT;
        const int slot0 = A % s.Wcap;  // ring slot of the first window position
        const int64_t ring_base = ring ? ring_row(s, a.layer, b, h, r, 0) : 0;
        if (tid == 0) flags[1] = 0;
        float mrow[kRows / 4], lrow[kRows / 4];  // warp w: rows w, w+4, w+8, w+12
#pragma unroll
        for (int i = 0; i < kRows / 4; ++i) { mrow[i] = -INFINITY; lrow[i] = 0.f; }
        float o[kRows];
#pragma unroll
        for (int i = 0; i < kRows; ++i) o[i] = 0.f;

        for (int t = 0; t < ntile; ++t) {
            const int k0 = t * KT, nkt = min(nk - k0, KT);
            // All threads: 16-byte asynchronous copies of the tile's K rows (padded
            // stride) and V rows (dense); consecutive threads take consecutive 16-byte
            // pieces of a row, so each run of key rows is read coalesced.
            for (int e = tid; e < nkt * NVEC; e += kThreads) {
                const int kk = e / NVEC, v = e - kk * NVEC;
                const int key = k0 + kk;
                const char *ks, *vs;
                if (key < nwin) {
                    const int p = A + key;
                    int64_t off;
                    if (ring) {
                        int slot = slot0 + key;
                        if (slot >= s.Wcap) slot -= s.Wcap;
                        off = ring_base + (int64_t)slot * ROWB;
                        ks = s.kwin + off; vs = s.vwin + off;
                    } else {
                        off = deep_row(s, a.layer, b, h, p);
                        ks = s.kdeep + off; vs = s.vdeep + off;
                    }
                } else {
                    const int64_t row = br.row0 + (int64_t)(key - nwin) * br.stride;
                    const int64_t off = (row * H + h) * ROWB;
                    ks = a.Kb + off; vs = a.Vb + off;
                }
                cp_async16(sK + (size_t)kk * KSTR + 16 * v, ks + 16 * v);
                cp_async16(sV + (size_t)kk * ROWB + 16 * v, vs + 16 * v);
            }
            cp_async_commit();
            if (t == 0) {
                // q rows (pre-scaled to log2 units) while the first tile is in flight;
                // rows past nr are zero so every row loop can run all NR rows.
                constexpr int QV = D / 8;  // 16-byte vectors per q row
                for (int e = tid; e < kRows * QV; e += kThreads) {
                    const int rr = e / QV, v = e - rr * QV;
                    uint4 x = make_uint4(0, 0, 0, 0);
                    if (rr < nr) {
                        const int64_t row = br.row0 + (int64_t)(j0 + rr) * br.stride;
                        x = *reinterpret_cast<const uint4*>(a.Q + (row * H + h) * ROWB + 16 * v);
                    }
                    const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
                    float4 lo, hi;
                    lo.x = __uint_as_float(xw[0] << 16) * a.scale_log2;
                    lo.y = __uint_as_float(xw[0] & 0xFFFF0000u) * a.scale_log2;
                    lo.z = __uint_as_float(xw[1] << 16) * a.scale_log2;
                    lo.w = __uint_as_float(xw[1] & 0xFFFF0000u) * a.scale_log2;
                    hi.x = __uint_as_float(xw[2] << 16) * a.scale_log2;
                    hi.y = __uint_as_float(xw[2] & 0xFFFF0000u) * a.scale_log2;
                    hi.z = __uint_as_float(xw[3] << 16) * a.scale_log2;
                    hi.w = __uint_as_float(xw[3] & 0xFFFF0000u) * a.scale_log2;
                    *reinterpret_cast<float4*>(q_s + rr * D + 8 * v) = lo;
                    *reinterpret_cast<float4*>(q_s + rr * D + 8 * v + 4) = hi;
                }
            }
            cp_async_wait_all();
            __syncthreads();
            // A. scores in log2 units: thread = key; q rows broadcast from shared memory
            for (int kk = tid; kk < nkt; kk += kThreads) {
                float acc[kRows];
#pragma unroll
                for (int rr = 0; rr < kRows; ++rr) acc[rr] = 0.f;
                const uint4* krow = reinterpret_cast<const uint4*>(sK + (size_t)kk * KSTR);
#pragma unroll 2
                for (int v = 0; v < NVEC; ++v) {
                    const uint4 x = krow[v];
                    const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
                    float kf[8];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        kf[2 * e] = __uint_as_float(xw[e] << 16);
                        kf[2 * e + 1] = __uint_as_float(xw[e] & 0xFFFF0000u);
                    }
#pragma unroll
                    for (int rr = 0; rr < kRows; ++rr) {
                        const float4 qa = *reinterpret_cast<const float4*>(q_s + rr * D + 8 * v);
                        const float4 qb = *reinterpret_cast<const float4*>(q_s + rr * D + 8 * v + 4);
                        acc[rr] = fmaf(qa.x, kf[0], acc[rr]);
                        acc[rr] = fmaf(qa.y, kf[1], acc[rr]);
                        acc[rr] = fmaf(qa.z, kf[2], acc[rr]);
                        acc[rr] = fmaf(qa.w, kf[3], acc[rr]);
                        acc[rr] = fmaf(qb.x, kf[4], acc[rr]);
                        acc[rr] = fmaf(qb.y, kf[5], acc[rr]);
                        acc[rr] = fmaf(qb.z, kf[6], acc[rr]);
                        acc[rr] = fmaf(qb.w, kf[7], acc[rr]);
                    }
                }
                const int key = k0 + kk;
#pragma unroll
                for (int rr = 0; rr < kRows; ++rr) {
                    const bool masked = rr >= nr || (key >= nwin && key - nwin > j0 + rr);
                    sc[rr * KT + kk] = masked ? -INFINITY : acc[rr];
                }
            }
            __syncthreads();
            // B. online softmax: warp = row; probabilities go to pt[key][row]
#pragma unroll
            for (int i = 0; i < kRows / 4; ++i) {
                const int rr = warp + 4 * i;
                const float* srow = sc + (size_t)rr * KT;
                float mt = -INFINITY;
                for (int kk = lane; kk < nkt; kk += 32) mt = fmaxf(mt, srow[kk]);
                mt = warp_max(mt);
                const float mn = fmaxf(mrow[i], mt);
                float alpha = 1.f;
                if (mn == -INFINITY) {
                    for (int kk = lane; kk < nkt; kk += 32) pt[kk * kRows + rr] = 0.f;
                } else {
                    alpha = ex2(mrow[i] - mn);
                    float sum = 0.f;
                    for (int kk = lane; kk < nkt; kk += 32) {
                        const float p = ex2(srow[kk] - mn);
                        pt[kk * kRows + rr] = p;
                        sum += p;
                    }
                    lrow[i] = lrow[i] * alpha + warp_sum(sum);
                    mrow[i] = mn;
                }
                if (lane == 0) alph[rr] = alpha;
            }
            __syncthreads();
            // C. o = alpha*o + P V: thread = channel, all rows
            if (tid < D) {
#pragma unroll
                for (int rr = 0; rr < kRows; ++rr) o[rr] *= alph[rr];
                const __nv_bfloat16* vcol = reinterpret_cast<const __nv_bfloat16*>(sV) + tid;
#pragma unroll 4
                for (int kk = 0; kk < nkt; ++kk) {
                    const float v = __bfloat162float(vcol[(size_t)kk * D]);
                    const float4* pk = reinterpret_cast<const float4*>(pt + kk * kRows);
#pragma unroll
                    for (int q4 = 0; q4 < kRows / 4; ++q4) {
                        const float4 p = pk[q4];
                        o[4 * q4] = fmaf(p.x, v, o[4 * q4]);
                        o[4 * q4 + 1] = fmaf(p.y, v, o[4 * q4 + 1]);
                        o[4 * q4 + 2] = fmaf(p.z, v, o[4 * q4 + 2]);
                        o[4 * q4 + 3] = fmaf(p.w, v, o[4 * q4 + 3]);
                    }
                }
            }
            __syncthreads();
        }

        // Partial of this split (window + block) for every row.
        const int seg = a.nsplit;
        if (tid < D) {
#pragma unroll
            for (int rr = 0; rr < kRows; ++rr) {
                if (rr < nr) {
                    const int64_t row = br.row0 + (int64_t)(j0 + rr) * br.stride;
                    a.part_o[((row * H + h) * a.nseg + seg) * D + tid] = o[rr];
                }
            }
        }
        float* ml_s = alph;  // reuse: (m, l) of each row for the merge
#pragma unroll
        for (int i = 0; i < kRows / 4; ++i) {
            const int rr = warp + 4 * i;
            if (rr >= nr) break;
            if (lane == 0) {
                const int64_t row = br.row0 + (int64_t)(j0 + rr) * br.stride;
                a.part_ml[(row * H + h) * a.nseg + seg] = make_float2(mrow[i], lrow[i]);
            }
        }
        __syncthreads();  // alph no longer read
#pragma unroll
        for (int i = 0; i < kRows / 4; ++i) {
            const int rr = warp + 4 * i;
            if (rr < nr && lane == 0) {
                ml_s[2 * rr] = mrow[i];
                ml_s[2 * rr + 1] = lrow[i];
            }
        }
        __syncthreads();
        const int ndeep = deep_splits_used(A, a.chunk, a.nsplit);
        if (tid == 0) {
            int* cnt = a.cnt + ((int64_t)bi * a.nrowchunks + rc) * H + h;
            __threadfence();  // releases every thread's partial (ordered before by the barrier)
            const int old = atomicAdd(cnt, 1);
            const int last = old == ndeep;
            if (last) *cnt = 0;
            flags[0] = last;
            __threadfence();
        }
        __syncthreads();
        if (flags[0]) {
            // Last to arrive: merge with the deep partials (read past L1, they come from
            // other CTAs).  Row by row, all of a row's loads are issued before use.
            constexpr int MAXS = 8;
            if (tid < D) {
#pragma unroll 1
                for (int rr = 0; rr < nr; ++rr) {
                    const int64_t row = br.row0 + (int64_t)(j0 + rr) * br.stride;
                    const int64_t base = (row * H + h) * a.nseg;
                    float mv[MAXS], lv[MAXS], ov[MAXS];
#pragma unroll
                    for (int sg = 0; sg < MAXS; ++sg) {
                        mv[sg] = -INFINITY;
                        lv[sg] = 0.f;
                        ov[sg] = 0.f;
                        if (sg < ndeep) {
                            const float2 ml = __ldcg(a.part_ml + base + sg);
                            mv[sg] = ml.x;
                            lv[sg] = ml.y;
                            ov[sg] = __ldcg(a.part_o + (base + sg) * D + tid);
                        }
                    }
                    float orow = 0.f;
#pragma unroll
                    for (int q = 0; q < kRows; ++q)
                        if (q == rr) orow = o[q];
                    // Same operation order as the deep-side merge (deep splits in order,
                    // then the window partial), so the result does not depend on who merges.
                    float M = -INFINITY;
#pragma unroll
                    for (int sg = 0; sg < MAXS; ++sg) M = fmaxf(M, mv[sg]);
                    M = fmaxf(M, ml_s[2 * rr]);
                    float L = 0.f, acc = 0.f;
#pragma unroll
                    for (int sg = 0; sg < MAXS; ++sg) {
                        if (sg < ndeep) {
                            const float f = ex2(mv[sg] - M);
                            L = fmaf(lv[sg], f, L);
                            acc = fmaf(ov[sg], f, acc);
                        }
                    }
                    const float fo = ex2(ml_s[2 * rr] - M);
                    L = fmaf(ml_s[2 * rr + 1], fo, L);
                    acc = fmaf(orow, fo, acc);
                    reinterpret_cast<__nv_bfloat16*>(a.O)[(row * H + h) * D + tid] = __float2bfloat16_rn(acc / L);
                    if (tid == 0 && a.lse) a.lse[row * H + h] = (M + log2f(L)) * 0.69314718055994531f;
                }
            }
        }
    }

    // Completion: the last CTA of this grid waits for the deep-plane grid it may run
    // beside (programmatic dependent launch), so that this grid ending implies both ended.
    __syncthreads();
    if (tid == 0) {
        const int n = atomicAdd(a.done, 1);
        if (n == (int)gridDim.x - 1) {
            *a.done = 0;
            grid_dependency_wait();
        }
    }
    grid_launch_dependents();
}

// ---------------------------------------------------------------------------
// Grouped variant: G units (consecutive branches -- for all-depths calls,
// consecutive loop depths -- of one head and row chunk) per CTA of 256 threads,
// so every phase has work for all threads and the barriers, copies, counters and
// merges are shared by G units.  Used when every unit's keys fit one tile.
// ---------------------------------------------------------------------------

template <int D, int NR, int G>
struct GroupLayout {
    static constexpr int ROWB = D * 2;
    static constexpr int KSTR = ROWB + 16;
    static constexpr int NVEC = ROWB / 16;
    // per unit: K (padded), V, q (fp32), scores [row][key], probabilities [key][row]
    __host__ __device__ static size_t unit_bytes(int KTU) {
        return (size_t)KTU * (KSTR + ROWB) + (size_t)NR * D * 4 + (size_t)2 * NR * KTU * 4;
    }
    __host__ __device__ static size_t bytes(int KTU) { return 512 + G * unit_bytes(KTU) + G * NR * 8; }
};

struct UnitInfo {
    const char *kring, *vring;  // plane r ring base (r < R) or deep plane base (r == R)
    int nk, nwin, nr, j0, row0, stride, bi, rc, h, A, slot0, ring, ndeep, last;
};

template <int D, int NR, int G>
__global__ void __launch_bounds__(64 * G) wgroup_kernel(VerifyArgs a, int KTU) {
    constexpr int kGThreads = 64 * G;  // two warps per unit
    using namespace sm100;
    using Lay = GroupLayout<D, NR, G>;
    constexpr int ROWB = Lay::ROWB, KSTR = Lay::KSTR, NVEC = Lay::NVEC;
    constexpr int NCP = D / 2;  // channel pairs per unit
    extern __shared__ __align__(128) uint8_t smem[];
    UnitInfo* ui = reinterpret_cast<UnitInfo*>(smem);  // G entries (< 512 bytes)
    uint8_t* ubase = smem + 512;
    float* mls = reinterpret_cast<float*>(ubase + G * Lay::unit_bytes(KTU));  // [G][NR][2]
    auto uK = [&](int u) { return ubase + u * Lay::unit_bytes(KTU); };
    auto uV = [&](int u) { return uK(u) + (size_t)KTU * KSTR; };
    auto uQ = [&](int u) { return reinterpret_cast<float*>(uV(u) + (size_t)KTU * ROWB); };
    auto uS = [&](int u) { return uQ(u) + NR * D; };
    auto uP = [&](int u) { return uS(u) + (size_t)NR * KTU; };

    const StoreView& s = a.s;
    const int H = s.H;
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int ngroups_b = (a.ba.nbranch + G - 1) / G;

    // ---- unit descriptors (one thread per unit)
    if (tid < G) {
        int64_t gidx = blockIdx.x;
        const int gb = (int)(gidx % ngroups_b);
        gidx /= ngroups_b;
        const int rc = (int)(gidx % a.nrowchunks);
        const int h = (int)(gidx / a.nrowchunks);
        const int bi = gb * G + tid;
        UnitInfo info{};
        info.nk = 0;
        if (bi < a.ba.nbranch) {
            const Branch br = load_branch(a.ba, s.R, s.Bmax, bi);
            if (!br.ok && rc == 0 && h == 0) set_device_error(s.err, RIPE_DEVERR_BRANCH);
            const int j0 = rc * kRowChunk;
            if (br.ok && j0 < br.ntok) {
                const int b = br.seq, r = br.depth;
                const int T = context_length(s.len, a.ctx, s.err, b, h == 0 && rc == 0);
                const int A = min(s.ws[b], T);
                info.nr = min(NR, br.ntok - j0);
                info.j0 = j0;
                info.nwin = T - A;
                info.nk = info.nwin + j0 + info.nr;
                info.row0 = br.row0;
                info.stride = br.stride;
                info.bi = bi;
                info.rc = rc;
                info.h = h;
                info.A = A;
                info.ring = r < s.R;
                info.slot0 = A % s.Wcap;
                info.kring = info.ring ? s.kwin + ring_row(s, a.layer, b, h, r, 0) : s.kdeep + deep_row(s, a.layer, b, h, A);
                info.vring = info.ring ? s.vwin + ring_row(s, a.layer, b, h, r, 0) : s.vdeep + deep_row(s, a.layer, b, h, A);
                info.ndeep = deep_splits_used(A, a.chunk, a.nsplit);
            }
        }
        ui[tid] = info;
    }
    __syncthreads();
    int nkmax = 0, total = 0;
#pragma unroll
    for (int u = 0; u < G; ++u) {
        nkmax = max(nkmax, ui[u].nk);
        total += ui[u].nk;
    }

    if (total > 0) {
        // ---- copies: one K/V row per thread-iteration (K padded, V dense)
        for (int pidx = tid; pidx < total; pidx += kGThreads) {
            int u = 0, key = pidx;
#pragma unroll
            for (int q = 0; q < G - 1; ++q)
                if (u == q && key >= ui[q].nk) { key -= ui[q].nk; u = q + 1; }
            const UnitInfo& U = ui[u];
            const char *kp, *vp;
            if (key < U.nwin) {
                if (U.ring) {
                    int slot = U.slot0 + key;
                    if (slot >= s.Wcap) slot -= s.Wcap;
                    kp = U.kring + (int64_t)slot * ROWB;
                    vp = U.vring + (int64_t)slot * ROWB;
                } else {
                    kp = U.kring + (int64_t)key * ROWB;
                    vp = U.vring + (int64_t)key * ROWB;
                }
            } else {
                const int64_t row = U.row0 + (int64_t)(key - U.nwin) * U.stride;
                kp = a.Kb + (row * H + U.h) * ROWB;
                vp = a.Vb + (row * H + U.h) * ROWB;
            }
            uint8_t* dk = uK(u) + (size_t)key * KSTR;
            uint8_t* dv = uV(u) + (size_t)key * ROWB;
#pragma unroll
            for (int v = 0; v < NVEC; ++v) {
                cp_async16(dk + 16 * v, kp + 16 * v);
                cp_async16(dv + 16 * v, vp + 16 * v);
            }
        }
        cp_async_commit();
        // ---- q rows (log2 units; rows past nr are zero) while the copies fly
        for (int e = tid; e < G * NR * NVEC; e += kGThreads) {
            const int u = e / (NR * NVEC), rem = e - u * NR * NVEC;
            const int rr = rem / NVEC, v = rem - rr * NVEC;
            const UnitInfo& U = ui[u];
            uint4 x = make_uint4(0, 0, 0, 0);
            if (U.nk > 0 && rr < U.nr) {
                const int64_t row = U.row0 + (int64_t)(U.j0 + rr) * U.stride;
                x = *reinterpret_cast<const uint4*>(a.Q + (row * H + U.h) * ROWB + 16 * v);
            }
            const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
            float* dst = uQ(u) + rr * D + 8 * v;
            float4 lo, hi;
            lo.x = __uint_as_float(xw[0] << 16) * a.scale_log2;
            lo.y = __uint_as_float(xw[0] & 0xFFFF0000u) * a.scale_log2;
            lo.z = __uint_as_float(xw[1] << 16) * a.scale_log2;
            lo.w = __uint_as_float(xw[1] & 0xFFFF0000u) * a.scale_log2;
            hi.x = __uint_as_float(xw[2] << 16) * a.scale_log2;
            hi.y = __uint_as_float(xw[2] & 0xFFFF0000u) * a.scale_log2;
            hi.z = __uint_as_float(xw[3] << 16) * a.scale_log2;
            hi.w = __uint_as_float(xw[3] & 0xFFFF0000u) * a.scale_log2;
            *reinterpret_cast<float4*>(dst) = lo;
            *reinterpret_cast<float4*>(dst + 4) = hi;
        }
        cp_async_wait_all();
        __syncthreads();

        // ---- A. scores: thread = (unit, key); the K row read once for all rows
        for (int pidx = tid; pidx < total; pidx += kGThreads) {
            int u = 0, key = pidx;
#pragma unroll
            for (int q = 0; q < G - 1; ++q)
                if (u == q && key >= ui[q].nk) { key -= ui[q].nk; u = q + 1; }
            const UnitInfo& U = ui[u];
            const float* qb = uQ(u);
            const uint4* krow = reinterpret_cast<const uint4*>(uK(u) + (size_t)key * KSTR);
            float acc[NR];
#pragma unroll
            for (int rr = 0; rr < NR; ++rr) acc[rr] = 0.f;
#pragma unroll 4
            for (int v = 0; v < NVEC; ++v) {
                const uint4 x = krow[v];
                const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
                float kf[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    kf[2 * e] = __uint_as_float(xw[e] << 16);
                    kf[2 * e + 1] = __uint_as_float(xw[e] & 0xFFFF0000u);
                }
#pragma unroll
                for (int rr = 0; rr < NR; ++rr) {
                    const float4 qa = *reinterpret_cast<const float4*>(qb + rr * D + 8 * v);
                    const float4 qc = *reinterpret_cast<const float4*>(qb + rr * D + 8 * v + 4);
                    acc[rr] = fmaf(qa.x, kf[0], acc[rr]);
                    acc[rr] = fmaf(qa.y, kf[1], acc[rr]);
                    acc[rr] = fmaf(qa.z, kf[2], acc[rr]);
                    acc[rr] = fmaf(qa.w, kf[3], acc[rr]);
                    acc[rr] = fmaf(qc.x, kf[4], acc[rr]);
                    acc[rr] = fmaf(qc.y, kf[5], acc[rr]);
                    acc[rr] = fmaf(qc.z, kf[6], acc[rr]);
                    acc[rr] = fmaf(qc.w, kf[7], acc[rr]);
                }
            }
            float* sc = uS(u);
#pragma unroll
            for (int rr = 0; rr < NR; ++rr) {
                const bool masked = rr >= U.nr || (key >= U.nwin && key - U.nwin > U.j0 + rr);
                sc[rr * KTU + key] = masked ? -INFINITY : acc[rr];
            }
        }
        __syncthreads();

        // ---- B. softmax: warp = (unit, row)
        for (int pr = warp; pr < G * NR; pr += kGThreads / 32) {
            const int u = pr / NR, rr = pr - u * NR;
            const UnitInfo& U = ui[u];
            const int nk = U.nk;
            const float* srow = uS(u) + rr * KTU;
            float* pt = uP(u);
            float mt = -INFINITY;
            for (int kk = lane; kk < nk; kk += 32) mt = fmaxf(mt, srow[kk]);
            mt = warp_max(mt);
            float sum = 0.f;
            for (int kk = lane; kk < nk; kk += 32) {
                const float p = mt == -INFINITY ? 0.f : ex2(srow[kk] - mt);
                pt[kk * NR + rr] = p;
                sum += p;
            }
            sum = warp_sum(sum);
            if (lane == 0) {
                mls[(u * NR + rr) * 2] = mt;
                mls[(u * NR + rr) * 2 + 1] = sum;
            }
        }
        __syncthreads();

        // ---- C. o = P V: thread = (unit, channel pair)
        for (int pc = tid; pc < G * NCP; pc += kGThreads) {
            const int u = pc / NCP, cp2 = pc - u * NCP;
            const UnitInfo& U = ui[u];
            if (U.nk == 0) continue;
            const uint32_t* vcol = reinterpret_cast<const uint32_t*>(uV(u)) + cp2;
            const float4* pk = reinterpret_cast<const float4*>(uP(u));
            float o0[NR], o1[NR];
#pragma unroll
            for (int rr = 0; rr < NR; ++rr) { o0[rr] = 0.f; o1[rr] = 0.f; }
#pragma unroll 4
            for (int kk = 0; kk < U.nk; ++kk) {
                const uint32_t w2 = vcol[kk * (ROWB / 4)];
                const float v0 = __uint_as_float(w2 << 16), v1 = __uint_as_float(w2 & 0xFFFF0000u);
#pragma unroll
                for (int q4 = 0; q4 < NR / 4; ++q4) {
                    const float4 p = pk[kk * (NR / 4) + q4];
                    o0[4 * q4] = fmaf(p.x, v0, o0[4 * q4]);         o1[4 * q4] = fmaf(p.x, v1, o1[4 * q4]);
                    o0[4 * q4 + 1] = fmaf(p.y, v0, o0[4 * q4 + 1]); o1[4 * q4 + 1] = fmaf(p.y, v1, o1[4 * q4 + 1]);
                    o0[4 * q4 + 2] = fmaf(p.z, v0, o0[4 * q4 + 2]); o1[4 * q4 + 2] = fmaf(p.z, v1, o1[4 * q4 + 2]);
                    o0[4 * q4 + 3] = fmaf(p.w, v0, o0[4 * q4 + 3]); o1[4 * q4 + 3] = fmaf(p.w, v1, o1[4 * q4 + 3]);
                }
            }
            // partial of this split (window + block)
            const int seg = a.nsplit;
#pragma unroll
            for (int rr = 0; rr < NR; ++rr) {
                if (rr < U.nr) {
                    const int64_t row = U.row0 + (int64_t)(U.j0 + rr) * U.stride;
                    const int64_t pi = (row * H + U.h) * a.nseg + seg;
                    *reinterpret_cast<float2*>(a.part_o + pi * D + 2 * cp2) = make_float2(o0[rr], o1[rr]);
                    if (cp2 == 0) a.part_ml[pi] = make_float2(mls[(u * NR + rr) * 2], mls[(u * NR + rr) * 2 + 1]);
                }
            }
            // keep o for a possible merge: stash it in the (now free) K tile
            float* stash = reinterpret_cast<float*>(uK(u));
#pragma unroll
            for (int rr = 0; rr < NR; ++rr) {
                stash[rr * D + 2 * cp2] = o0[rr];
                stash[rr * D + 2 * cp2 + 1] = o1[rr];
            }
        }
        __syncthreads();

        // ---- arrivals: one thread per unit
        if (tid < G) {
            UnitInfo& U = ui[tid];
            if (U.nk > 0) {
                int* cnt = a.cnt + ((int64_t)U.bi * a.nrowchunks + U.rc) * H + U.h;
                __threadfence();  // releases the CTA's partials (ordered before by the barrier)
                U.last = atomicAdd(cnt, 1) == U.ndeep;
                if (U.last) *cnt = 0;
                __threadfence();
            } else {
                U.last = 0;
            }
        }
        __syncthreads();

        // ---- merge where this CTA arrived last: thread = (unit, channel pair);
        // deep splits in order, then the window partial (same order as the deep side).
        for (int pc = tid; pc < G * NCP; pc += kGThreads) {
            const int u = pc / NCP, cp2 = pc - u * NCP;
            const UnitInfo& U = ui[u];
            if (U.nk == 0 || !U.last) continue;
            const float* stash = reinterpret_cast<const float*>(uK(u));
            for (int rr = 0; rr < U.nr; ++rr) {
                const int64_t row = U.row0 + (int64_t)(U.j0 + rr) * U.stride;
                const int64_t base = (row * H + U.h) * a.nseg;
                const float mw = mls[(u * NR + rr) * 2], lw = mls[(u * NR + rr) * 2 + 1];
                float M = mw;
                for (int sg = 0; sg < U.ndeep; ++sg) M = fmaxf(M, __ldcg(a.part_ml + base + sg).x);
                float L = 0.f, acc0 = 0.f, acc1 = 0.f;
                for (int s0 = 0; s0 < U.ndeep; s0 += 4) {
                    float mv[4], lv[4];
                    float2 ov[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        if (s0 + q < U.ndeep) {
                            const float2 ml = __ldcg(a.part_ml + base + s0 + q);
                            mv[q] = ml.x;
                            lv[q] = ml.y;
                            ov[q] = __ldcg(reinterpret_cast<const float2*>(a.part_o + (base + s0 + q) * D) + cp2);
                        }
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        if (s0 + q < U.ndeep) {
                            const float f = ex2(mv[q] - M);
                            L = fmaf(lv[q], f, L);
                            acc0 = fmaf(ov[q].x, f, acc0);
                            acc1 = fmaf(ov[q].y, f, acc1);
                        }
                    }
                }
                const float fo = ex2(mw - M);
                L = fmaf(lw, fo, L);
                acc0 = fmaf(stash[rr * D + 2 * cp2], fo, acc0);
                acc1 = fmaf(stash[rr * D + 2 * cp2 + 1], fo, acc1);
                *reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<__nv_bfloat16*>(a.O) + (row * H + U.h) * D +
                                                   2 * cp2) = __floats2bfloat162_rn(acc0 / L, acc1 / L);
                if (cp2 == 0 && a.lse) a.lse[row * H + U.h] = (M + log2f(L)) * 0.69314718055994531f;
            }
        }
    }
    (void)nkmax;

    // Completion: the last CTA of this grid waits for the deep-plane grid it may run beside.
    __syncthreads();
    if (tid == 0) {
        const int n = atomicAdd(a.done, 1);
        if (n == (int)gridDim.x - 1) {
            *a.done = 0;
            grid_dependency_wait();
        }
    }
    grid_launch_dependents();
}

}  // namespace

bool window_supported(int dtype, int d) { return dtype == RIPE_BF16 && (d == 64 || d == 96 || d == 128); }

template <int D, int NR, int G>
cudaError_t launch_group_t(cudaLaunchConfig_t cfg, const VerifyArgs& a, int KTU) {
    static bool set = false;
    if (!set) {
        cudaFuncSetAttribute(wgroup_kernel<D, NR, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        cudaFuncSetAttribute(wgroup_kernel<D, NR, G>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
        set = true;
    }
    const int64_t groups = (int64_t)(a.ba.nbranch + G - 1) / G * a.nrowchunks * a.s.H;
    if (groups > 0x7fffffff) return cudaErrorInvalidConfiguration;
    cfg.gridDim = dim3((unsigned)groups);
    cfg.blockDim = dim3(64 * G);
    cfg.dynamicSmemBytes = GroupLayout<D, NR, G>::bytes(KTU);
    return cudaLaunchKernelEx(&cfg, wgroup_kernel<D, NR, G>, a, KTU);
}

template <int D, int NR>
cudaError_t launch_group_d(cudaLaunchConfig_t cfg, const VerifyArgs& a, int KTU, int G) {
    if (G == 4) return launch_group_t<D, NR, 4>(cfg, a, KTU);
    if (G == 2) return launch_group_t<D, NR, 2>(cfg, a, KTU);
    return launch_group_t<D, NR, 1>(cfg, a, KTU);
}

cudaError_t launch_window(const VerifyArgs& a, int nbranch, int keys_ub, bool pdl, cudaStream_t st) {
    const int64_t grid = (int64_t)nbranch * a.nrowchunks * a.s.H;
    if (grid == 0) return cudaSuccess;
    if (grid > 0x7fffffff) return cudaErrorInvalidConfiguration;
    int KT = (keys_ub + 7) / 8 * 8;
    if (KT > 160) KT = 128;
    if (KT < 8) KT = 8;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    const int rows = a.ba.max_ntok < kRowChunk ? a.ba.max_ntok : kRowChunk;
    const int NR = rows <= 4 ? 4 : rows <= 8 ? 8 : 16;

    // Grouped kernel when every unit's keys fit one tile and NR <= 8: as many units
    // per CTA as keep the CTA within ~70 KB of shared memory (three per SM).
    if (keys_ub <= 160 && NR <= 8) {
        int KTU = (keys_ub + 7) / 8 * 8;
        const int min_ktu = (NR * a.s.d * 4 + (2 * a.s.d + 16) - 1) / (2 * a.s.d + 16);  // o stash fits the K tile
        if (KTU < min_ktu) KTU = (min_ktu + 7) / 8 * 8;
        const size_t unit = (size_t)KTU * (4 * a.s.d + 16) + (size_t)NR * a.s.d * 4 + (size_t)2 * NR * KTU * 4;
        int G = 4;
        while (G > 1 && 512 + G * unit + G * NR * 8 > 72 * 1024) G /= 2;
        cudaError_t e = cudaErrorInvalidValue;
        switch (a.s.d * 16 + NR) {
            case 64 * 16 + 4: e = launch_group_d<64, 4>(cfg, a, KTU, G); break;
            case 64 * 16 + 8: e = launch_group_d<64, 8>(cfg, a, KTU, G); break;
            case 96 * 16 + 4: e = launch_group_d<96, 4>(cfg, a, KTU, G); break;
            case 96 * 16 + 8: e = launch_group_d<96, 8>(cfg, a, KTU, G); break;
            case 128 * 16 + 4: e = launch_group_d<128, 4>(cfg, a, KTU, G); break;
            case 128 * 16 + 8: e = launch_group_d<128, 8>(cfg, a, KTU, G); break;
        }
        ripe_count_launch();
        return e;
    }

    static bool attrs_set = false;
    if (!attrs_set) {
#define RIPE_WIN_ATTR(D_, NR_)                                                                             \
        cudaFuncSetAttribute(window_kernel<D_, NR_>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024); \
        cudaFuncSetAttribute(window_kernel<D_, NR_>, cudaFuncAttributePreferredSharedMemoryCarveout,          \
                             cudaSharedmemCarveoutMaxShared);
        RIPE_WIN_ATTR(64, 4) RIPE_WIN_ATTR(64, 8) RIPE_WIN_ATTR(64, 16)
        RIPE_WIN_ATTR(96, 4) RIPE_WIN_ATTR(96, 8) RIPE_WIN_ATTR(96, 16)
        RIPE_WIN_ATTR(128, 4) RIPE_WIN_ATTR(128, 8) RIPE_WIN_ATTR(128, 16)
#undef RIPE_WIN_ATTR
        attrs_set = true;
    }
    cudaError_t e = cudaErrorInvalidValue;
#define RIPE_WIN_GO(D_, NR_)                                       \
    if (a.s.d == D_ && NR == NR_) {                                \
        cfg.dynamicSmemBytes = WinLayout<D_, NR_>::bytes(KT);      \
        e = cudaLaunchKernelEx(&cfg, window_kernel<D_, NR_>, a, KT); \
    }
    RIPE_WIN_GO(64, 4) RIPE_WIN_GO(64, 8) RIPE_WIN_GO(64, 16)
    RIPE_WIN_GO(96, 4) RIPE_WIN_GO(96, 8) RIPE_WIN_GO(96, 16)
    RIPE_WIN_GO(128, 4) RIPE_WIN_GO(128, 8) RIPE_WIN_GO(128, 16)
#undef RIPE_WIN_GO
    ripe_count_launch();
    return e;
}
