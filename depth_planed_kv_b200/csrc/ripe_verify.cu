// ripe_verify.cu -- verify-attention over the RIPE store: the CUDA-core split
// kernel (bf16 or f32, head sizes up to 128), the split merge, and the plan
// that decides how the deep region is split and which kernel reads it.
//
// Read rule (RIPE abstract, sentence introducing RIPE; LoopSpec article on
// mixed-depth branches): row j of branch (b, r) attends to positions
// [0, min(ws_b,T_b)) at plane R, [min(ws_b,T_b), T_b) at plane r, and block
// tokens 0..j of its branch at plane r.
//
// Partial results: every split of a row writes (m, l) and o[d] with
//   m = max of the split's scores (log2 domain, i.e. scaled by scale*log2 e),
//   l = sum 2^(s - m), o = sum 2^(s - m) v,
// and the merge combines them by their maxima.  Splits 0..nsplit-1 cover the
// deep region in chunks; split nsplit covers the window region and the block.
#include <math.h>

#include "ripe_internal.cuh"
#include "ripe_launch.h"
#include "ripe_verify.cuh"
#include "sm100_ptx.cuh"

namespace {

constexpr int kWarps = 4;
constexpr int kRowsPerWarp = 4;
constexpr int kRowsPerCta = kWarps * kRowsPerWarp;

template <typename Elem>
__device__ inline float to_f32(Elem x);
template <>
__device__ inline float to_f32<float>(float x) { return x; }
template <>
__device__ inline float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename Elem>
__device__ inline Elem from_f32(float x);
template <>
__device__ inline float from_f32<float>(float x) { return x; }
template <>
__device__ inline __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

__device__ inline float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ inline float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// One CTA: up to 16 rows of one branch, one head, one split of its keys.
//
// The split's keys (a contiguous run of the deep plane, or the window run of
// plane r -- the ring, which wraps at most once -- followed by the branch's
// draft-block tokens) stream into shared memory in tiles of KT keys by bulk
// asynchronous copies (one or two stages).  Per tile:
//   A. scores: thread = key; each K row is read once for all rows, 16 bytes at a
//      time with a per-key rotation of the starting vector (no bank conflicts
//      for any head size);
//   B. softmax: warp = row; tile max, rescale factor, probabilities in place;
//   C. P.V: warp = row group, lane = output channel; each V row read once per
//      warp for all of its rows.
// The split's partial (m, l, o) of every row goes to the scratch.
template <typename Elem, int MAXD>
__global__ void __launch_bounds__(kWarps * 32)
seg_kernel(VerifyArgs a, int seg_first, int seg_count, int KT, int ST) {
    using namespace sm100;
    constexpr int NV = MAXD / 32;
    constexpr int VE = 16 / sizeof(Elem);  // elements per 16-byte vector
    extern __shared__ __align__(128) uint8_t smem[];

    const StoreView& s = a.s;
    const int d = s.d, H = s.H;
    const int rowb = d * (int)sizeof(Elem);  // bytes per key row
    const int nvec = rowb / 16;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + 16);
    uint8_t* sK = smem + 128;
    uint8_t* sV = sK + (size_t)ST * KT * rowb;
    float* q_s = reinterpret_cast<float*>(sV + (size_t)ST * KT * rowb);
    float* sc = q_s + kRowsPerCta * d;

    int w = blockIdx.x;
    const int seg = seg_first + w % seg_count; w /= seg_count;
    const int h = w % H; w /= H;
    const int rc = w % a.nrowchunks;
    const int bi = w / a.nrowchunks;
    const Branch br = load_branch(a.ba, s.R, s.Bmax, bi);
    if (!br.ok) {
        if (threadIdx.x == 0 && rc == 0 && h == 0 && seg == a.nsplit) set_device_error(s.err, RIPE_DEVERR_BRANCH);
        return;
    }
    const int j0 = rc * kRowsPerCta;
    if (j0 >= br.ntok) return;
    const int nr = min(kRowsPerCta, br.ntok - j0);
    const int b = br.seq, r = br.depth;
    const int T = context_length(s.len, a.ctx, s.err, b, seg == a.nsplit && h == 0 && rc == 0 && threadIdx.x == 0);
    const int A = min(s.ws[b], T);

    int p0, p1, nblk = 0;
    bool ring = false;
    if (seg < a.nsplit) {
        p0 = seg * a.chunk;
        p1 = min(A, p0 + a.chunk);
        if (p0 >= p1) return;
    } else {
        p0 = A;
        p1 = T;
        nblk = j0 + nr;  // block tokens 0..j0+nr-1 are visible to some row here
        ring = r < s.R;
    }
    const int ncom = p1 - p0;
    const int nk = ncom + nblk;
    const int ntile = (nk + KT - 1) / KT;
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;

    if (tid == 0) {
        for (int i = 0; i < ST; ++i) mbar_init(full + i, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();

    // Issue the copies of tile t into stage t % ST (one thread).
    auto issue_tile = [&](int t) {
        const int st = t % ST;
        const int k0 = t * KT, k1 = min(nk, k0 + KT);
        uint8_t* dk = sK + (size_t)st * KT * rowb;
        uint8_t* dv = sV + (size_t)st * KT * rowb;
        mbar_expect_tx(full + st, (uint32_t)(2 * (k1 - k0) * rowb));
        int key = k0;
        while (key < min(k1, ncom)) {
            const int p = p0 + key;
            int n = min(k1, ncom) - key;
            int64_t off;
            const char *kb, *vb;
            if (ring) {
                const int slot = p % s.Wcap;
                n = min(n, s.Wcap - slot);
                off = ring_row(s, a.layer, b, h, r, slot);
                kb = s.kwin; vb = s.vwin;
            } else {
                // a fork reads its parent's deep plane below its fork position
                const int fp = s.fpos[b];
                if (p < fp) n = min(n, fp - p);
                off = deep_row(s, a.layer, deep_owner(s, b, p), h, p);
                kb = s.kdeep; vb = s.vdeep;
            }
            bulk_load(dk + (size_t)(key - k0) * rowb, kb + off, (uint32_t)(n * rowb), full + st);
            bulk_load(dv + (size_t)(key - k0) * rowb, vb + off, (uint32_t)(n * rowb), full + st);
            key += n;
        }
        for (; key < k1; ++key) {
            const int64_t row = br.row0 + (int64_t)(key - ncom) * br.stride;
            const int64_t off = (row * H + h) * rowb;
            bulk_load(dk + (size_t)(key - k0) * rowb, a.Kb + off, (uint32_t)rowb, full + st);
            bulk_load(dv + (size_t)(key - k0) * rowb, a.Vb + off, (uint32_t)rowb, full + st);
        }
    };
    if (tid == 0) {
        for (int t = 0; t < ST && t < ntile; ++t) issue_tile(t);
    }

    for (int e = tid; e < nr * d; e += blockDim.x) {
        const int rr = e / d, c = e % d;
        const int64_t row = br.row0 + (int64_t)(j0 + rr) * br.stride;
        q_s[rr * d + c] = to_f32(reinterpret_cast<const Elem*>(a.Q)[(row * H + h) * d + c]) * a.scale_log2;
    }

    float m[kRowsPerWarp], l[kRowsPerWarp], o[kRowsPerWarp][NV];
#pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) {
        m[i] = -INFINITY;
        l[i] = 0.f;
#pragma unroll
        for (int v = 0; v < NV; ++v) o[i][v] = 0.f;
    }

    for (int t = 0; t < ntile; ++t) {
        const int st = t % ST;
        const int k0 = t * KT, nkt = min(nk, k0 + KT) - k0;
        mbar_wait(full + st, (t / ST) & 1, abort_flag, s.err);
        __syncthreads();  // q_s written; a timed-out wait still keeps every thread in step
        const uint8_t* tk = sK + (size_t)st * KT * rowb;
        const uint8_t* tv = sV + (size_t)st * KT * rowb;
        // A. scores (log2 units): thread = key
        for (int kk = tid; kk < nkt; kk += blockDim.x) {
            float acc[kRowsPerCta];
#pragma unroll
            for (int rr = 0; rr < kRowsPerCta; ++rr) acc[rr] = 0.f;
            const uint4* krow = reinterpret_cast<const uint4*>(tk + (size_t)kk * rowb);
            for (int v = 0; v < nvec; ++v) {
                int vv = v + kk;
                vv -= (vv / nvec) * nvec;
                const uint4 x = krow[vv];
                float kf[VE];
                if constexpr (sizeof(Elem) == 2) {
                    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __bfloat1622float2(b2[e]);
                        kf[2 * e] = f.x;
                        kf[2 * e + 1] = f.y;
                    }
                } else {
                    kf[0] = __uint_as_float(x.x); kf[1] = __uint_as_float(x.y);
                    kf[2] = __uint_as_float(x.z); kf[3] = __uint_as_float(x.w);
                }
#pragma unroll
                for (int rr = 0; rr < kRowsPerCta; ++rr) {
                    if (rr < nr) {
                        const float* qv = q_s + rr * d + vv * VE;
#pragma unroll
                        for (int e = 0; e < VE; ++e) acc[rr] = fmaf(qv[e], kf[e], acc[rr]);
                    }
                }
            }
            const int key = k0 + kk;
#pragma unroll
            for (int rr = 0; rr < kRowsPerCta; ++rr) {
                if (rr < nr) {
                    const bool masked = key >= ncom && key - ncom > j0 + rr;
                    sc[rr * KT + kk] = masked ? -INFINITY : acc[rr];
                }
            }
        }
        __syncthreads();
        // B. online softmax: warp = row
        float alpha[kRowsPerWarp];
#pragma unroll
        for (int i = 0; i < kRowsPerWarp; ++i) {
            alpha[i] = 1.f;
            const int rr = warp + kWarps * i;
            if (rr >= nr) continue;
            float* srow = sc + rr * KT;
            float mt = -INFINITY;
            for (int kk = lane; kk < nkt; kk += 32) mt = fmaxf(mt, srow[kk]);
            mt = warp_max(mt);
            const float mn = fmaxf(m[i], mt);
            if (mn == -INFINITY) {
                for (int kk = lane; kk < nkt; kk += 32) srow[kk] = 0.f;
                continue;
            }
            alpha[i] = ex2(m[i] - mn);
            float sum = 0.f;
            for (int kk = lane; kk < nkt; kk += 32) {
                const float p = ex2(srow[kk] - mn);
                srow[kk] = p;
                sum += p;
            }
            l[i] = l[i] * alpha[i] + warp_sum(sum);
            m[i] = mn;
        }
        __syncwarp();
        // C. o = alpha*o + P V: warp = its rows, lane = channels
#pragma unroll
        for (int i = 0; i < kRowsPerWarp; ++i)
#pragma unroll
            for (int v = 0; v < NV; ++v) o[i][v] *= alpha[i];
        const int nrw = nr > warp ? (nr - warp + kWarps - 1) / kWarps : 0;
        for (int kk = 0; kk < nkt; ++kk) {
            const Elem* vrow = reinterpret_cast<const Elem*>(tv + (size_t)kk * rowb);
            float vv[NV];
#pragma unroll
            for (int v = 0; v < NV; ++v) {
                const int c = lane + 32 * v;
                vv[v] = c < d ? to_f32(vrow[c]) : 0.f;
            }
#pragma unroll
            for (int i = 0; i < kRowsPerWarp; ++i) {
                if (i < nrw) {
                    const float p = sc[(warp + kWarps * i) * KT + kk];
#pragma unroll
                    for (int v = 0; v < NV; ++v) o[i][v] = fmaf(p, vv[v], o[i][v]);
                }
            }
        }
        __syncthreads();
        if (tid == 0 && t + ST < ntile) issue_tile(t + ST);
    }

#pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) {
        const int rr = warp + kWarps * i;
        if (rr >= nr) break;
        const int64_t row = br.row0 + (int64_t)(j0 + rr) * br.stride;
        const int64_t pi = (row * H + h) * a.nseg + seg;
        if (lane == 0) a.part_ml[pi] = make_float2(m[i], l[i]);
#pragma unroll
        for (int v = 0; v < NV; ++v) {
            const int c = lane + 32 * v;
            if (c < d) a.part_o[pi * d + c] = o[i][v];
        }
    }
}

// Combine the splits of every row: M = max m_s, L = sum l_s 2^(m_s-M),
// O = sum 2^(m_s-M) o_s / L, lse = (M + log2 L) ln 2.
template <typename Elem>
__global__ void __launch_bounds__(128) merge_kernel(VerifyArgs a) {
    const StoreView& s = a.s;
    const int d = s.d, H = s.H;
    const int h = blockIdx.x % H;
    const int bi = blockIdx.x / H;
    const Branch br = load_branch(a.ba, s.R, s.Bmax, bi);
    if (!br.ok) return;
    const int T = context_length(s.len, a.ctx, s.err, br.seq, false);
    const int A = min(s.ws[br.seq], T);
    const int nvalid = min(a.nsplit, (A + a.chunk - 1) / a.chunk);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    for (int j = warp; j < br.ntok; j += 4) {
        const int64_t row = br.row0 + (int64_t)j * br.stride;
        const int64_t base = (row * H + h) * a.nseg;
        float M = -INFINITY;
        for (int sg = 0; sg <= a.nsplit; ++sg) {
            if (sg < a.nsplit && sg >= nvalid) continue;
            const float2 ml = a.part_ml[base + sg];
            if (ml.y > 0.f) M = fmaxf(M, ml.x);
        }
        float L = 0.f;
        for (int sg = 0; sg <= a.nsplit; ++sg) {
            if (sg < a.nsplit && sg >= nvalid) continue;
            const float2 ml = a.part_ml[base + sg];
            if (ml.y > 0.f) L += exp2f(ml.x - M) * ml.y;
        }
        for (int c = lane; c < d; c += 32) {
            float acc = 0.f;
            for (int sg = 0; sg <= a.nsplit; ++sg) {
                if (sg < a.nsplit && sg >= nvalid) continue;
                const float2 ml = a.part_ml[base + sg];
                if (ml.y > 0.f) acc = fmaf(exp2f(ml.x - M), a.part_o[(base + sg) * d + c], acc);
            }
            reinterpret_cast<Elem*>(a.O)[(row * H + h) * d + c] = from_f32<Elem>(acc / L);
        }
        if (a.lse && lane == 0) a.lse[row * H + h] = (M + log2f(L)) * 0.69314718055994531f;
    }
}

// Key tile and stage count of the CUDA-core kernel: one stage when a split's keys
// fit a tile of at most 128, else two stages of 128-key tiles.
struct SegShape {
    int KT, ST;
    size_t smem;
};

SegShape seg_shape(int d, int esize, int keys_ub) {
    SegShape g;
    if (keys_ub <= 128) {
        g.KT = (keys_ub + 7) / 8 * 8;
        if (g.KT < 8) g.KT = 8;
        g.ST = 1;
    } else {
        g.KT = 128;
        g.ST = 2;
    }
    auto bytes = [&](int KT, int ST) {
        return 128 + (size_t)2 * ST * KT * d * esize + (size_t)kRowsPerCta * d * 4 + (size_t)kRowsPerCta * KT * 4;
    };
    while (bytes(g.KT, g.ST) > 150 * 1024 && g.KT > 16) g.KT = (g.KT / 2 + 7) / 8 * 8;
    g.smem = bytes(g.KT, g.ST);
    return g;
}

template <typename Elem>
cudaError_t launch_seg(const VerifyArgs& a, int seg_first, int seg_count, int nbranch, int keys_ub,
                       cudaStream_t st) {
    const int64_t grid = (int64_t)nbranch * a.nrowchunks * a.s.H * seg_count;
    if (grid == 0) return cudaSuccess;
    if (grid > 0x7fffffff) return cudaErrorInvalidConfiguration;
    const SegShape g = seg_shape(a.s.d, (int)sizeof(Elem), keys_ub);
    // The dynamic shared-memory limit is a per-device attribute of each instantiation.
    auto configure = [](const void* fn) {
        cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        if (e != cudaSuccess) return e;
        return cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                                    cudaSharedmemCarveoutMaxShared);
    };
    if (a.s.d <= 64) {
        static PerDeviceOnce cfg;
        cudaError_t e = per_device_once(cfg, [&] { return configure((const void*)seg_kernel<Elem, 64>); });
        if (e != cudaSuccess) return e;
        seg_kernel<Elem, 64><<<(unsigned)grid, kWarps * 32, g.smem, st>>>(a, seg_first, seg_count, g.KT, g.ST);
    } else {
        static PerDeviceOnce cfg;
        cudaError_t e = per_device_once(cfg, [&] { return configure((const void*)seg_kernel<Elem, 128>); });
        if (e != cudaSuccess) return e;
        seg_kernel<Elem, 128><<<(unsigned)grid, kWarps * 32, g.smem, st>>>(a, seg_first, seg_count, g.KT, g.ST);
    }
    ripe_count_launch();
    return cudaGetLastError();
}

// The persistent kernel serves an all-depths call whose k*R rows of a sequence
// fit two 128-row M tiles.  The plan splits the deep region into nsplit chunks and balances the
// bytes each CTA streams: pd CTAs take deep items (sequence, head, chunk) pd
// apart plus n_lo window units each; the others take n_hi window units.  A deep
// item also costs a fixed latency (Q load, pipeline fill, epilogue), counted as
// bytes of streaming.  The kernel's last chunk runs to the end of the deep
// region, so the chunk length only shapes the balance: it is sized for the
// deep region an evicted store has at the host's length bound (len_ub - W).
bool plan_persist(const ripe_cache_s* c, int nseq, int k, int len_ub, VerifyPlan& p) {
    const int A_ub = len_ub - c->W > 0 ? len_ub - c->W : 0;
    const int R = c->R, H = c->H, d = c->d;
    const int kR = k * R, QS = (k + 7) / 8;
    if (kR > 256 || nseq < 1) return false;
    const int mt = kR > 128 ? 2 : 1;
    int nww_deep = 0, nww_other = 0;
    persist_shape(d, mt, &nww_deep, &nww_other);
    if (nww_other == 0) return false;
    const int P = device_sm_count();
    if (P < 1) return false;
    const double kv = 4.0 * d, row = 2.0 * d;
    const int wl = len_ub < c->W ? len_ub : c->W;
    // A window unit costs its bytes, but at least a fixed ~20 KB-equivalent of issue
    // and compute time (measured: a unit of a few KB takes about as long as one
    // of 20 KB).
    const double bU_bytes = (wl + k) * kv + 2.0 * (k < 8 ? k : 8) * row;
    const double bU = bU_bytes > 20e3 ? bU_bytes : 20e3;
    const double item_fixed = 96e3;
    const int64_t NU = (int64_t)nseq * H * R * QS;
    if (NU > (1 << 30)) return false;
    double best = 1e300;
    bool found = false;
    for (int nd = 1; nd <= 8; ++nd) {
        int chunk = (A_ub + nd - 1) / nd;
        chunk = (chunk + 63) / 64 * 64;
        if (chunk < 64) chunk = 64;
        if (nd > 1 && (int64_t)chunk * (nd - 1) >= A_ub) break;  // a chunk would always be empty
        const int64_t ND = (int64_t)nseq * H * nd;
        const int pd = (int)(ND < P ? ND : P);
        const int64_t I = (ND + pd - 1) / pd;
        if (I > 32) continue;
        const double bD = chunk * kv + kR * row + item_fixed;
        const double LD = I * bD;
        int64_t n_lo, n_hi;
        double Tm;
        if (pd == P) {
            n_hi = 0;
            n_lo = (NU + P - 1) / P;
            Tm = LD + n_lo * bU;
        } else {
            const double T0 = LD > (ND * bD + NU * bU) / P ? LD : (ND * bD + NU * bU) / P;
            n_hi = (int64_t)ceil(T0 / bU);
            if (n_hi < 1) n_hi = 1;
            for (;;) {
                const double spare = n_hi * bU - LD;
                n_lo = spare > 0 ? (int64_t)floor(spare / bU) : 0;
                if (pd * n_lo + (int64_t)(P - pd) * n_hi >= NU) break;
                ++n_hi;
            }
            Tm = LD + n_lo * bU > n_hi * bU ? LD + n_lo * bU : n_hi * bU;
        }
        if (Tm < 0.98 * best) {  // more chunks only for a clear gain (their partials cost traffic)
            best = Tm;
            found = true;
            p.nsplit = nd;
            p.chunk = chunk;
            p.pd = pd;
            p.n_lo = (int)n_lo;
            p.n_hi = (int)n_hi;
            p.ndeep = (int)ND;
            const int64_t rest = NU - (int64_t)pd * n_lo;
            const int64_t others = rest > 0 ? (rest + n_hi - 1) / n_hi : 0;
            p.grid = (int)(pd + others < P ? pd + others : P);
        }
    }
    if (!found) return false;
    p.nunits = (int)NU;
    p.mt = mt;
    p.persist = true;
    return true;
}

}  // namespace

int device_sm_count() {
    static int count[64];
    static PerDeviceOnce once;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (per_device_once(once, [&] {
            return cudaDeviceGetAttribute(&count[dev], cudaDevAttrMultiProcessorCount, dev);
        }) != cudaSuccess)
        return 0;
    return count[dev];
}

VerifyPlan plan_verify(const ripe_cache_s* c, int nbranch, int nrows, int max_ntok, bool all_depths,
                       bool capacity, bool sliding) {
    VerifyPlan p{};
    p.max_ntok = max_ntok;
    p.nrowchunks = (max_ntok + kRowsPerCta - 1) / kRowsPerCta;
    if (p.nrowchunks < 1) p.nrowchunks = 1;
    const int len_ub = capacity ? c->Tmax : c->len_ub;
    const int A_ub = len_ub < c->Tmax ? len_ub : c->Tmax;
    p.a_ub = A_ub;
    p.win_ub = (len_ub < c->Wcap ? len_ub : c->Wcap) + max_ntok;
    p.fused = c->tc_ready && fused_supported(c->dtype, c->d);
    // All depths: the persistent kernel for the sliding window (only it serves that
    // form); where the deep region outweighs the windows over enough (sequence, head)
    // pairs to fill the SMs (long contexts); and where the windows, each one stage of
    // its ring, outweigh the deep region (short contexts, windows of tens of
    // positions).  Measured on B200, the cluster kernel is faster for windows too wide
    // for one stage and for windows of a few positions over a longer deep region.
    const int nseq = all_depths ? nbranch / c->R : 0;
    const int deep_ub = len_ub > c->W ? len_ub - c->W : 0;
    const bool deep_heavy = (int64_t)deep_ub >= (int64_t)c->R * (c->Wcap + max_ntok) &&
                            (int64_t)nseq * c->H >= device_sm_count();
    const int mt_ad = max_ntok * c->R > 128 ? 2 : 1;
    const bool window_heavy = persist_ring_ok(c->d, mt_ad, c->Wcap, max_ntok, sliding ? 1 : 0, c->full_box ? 1 : 0) &&
                              (int64_t)c->R * c->Wcap >= deep_ub;
    const int choice = c->all_depths_kernel;
    const bool want = sliding || choice == RIPE_ALL_DEPTHS_PERSISTENT ||
                      (choice == RIPE_ALL_DEPTHS_AUTO && (deep_heavy || window_heavy));
    if (p.fused && all_depths && want && plan_persist(c, nseq, max_ntok, len_ub, p)) {
        p.part_bytes = persist_work_bytes(nrows, c->H, c->d, p.nsplit + 1, nbranch / c->R);
        p.work_bytes = p.part_bytes;
        return p;
    }
    int64_t ns;
    if (p.fused) {
        // One CTA per (sequence group, head, split); splits (a cluster, at most 8)
        // only until the CTAs cover the 148 SMs once: each CTA holds one SM.
        p.gslots = all_depths ? nbranch / c->R : (nbranch < c->Bmax ? nbranch : c->Bmax);
        p.mt = (all_depths && max_ntok * c->R > 128) ? 2 : 1;
        const int64_t units = (int64_t)p.gslots * c->H;
        ns = units > 0 ? 148 / units : 1;
        if (ns > 8) ns = 8;
        if (ns < 1) ns = 1;
    } else {
        const int64_t items = (int64_t)nbranch * p.nrowchunks * c->H;
        const int64_t target = 148 * 8;
        ns = items > 0 ? (target + items - 1) / items : 1;
        const int64_t max_ns = (A_ub + 63) / 64;
        if (ns > max_ns) ns = max_ns;
        if (ns < 1) ns = 1;
        p.mt = 0;
        p.gslots = 0;
    }
    plan_set_splits(p, c, nrows, (int)ns);
    return p;
}

void plan_set_splits(VerifyPlan& p, const ripe_cache_s* c, int nrows, int nsplit) {
    const int A_ub = p.a_ub;
    const int align = p.fused ? 64 : 32;  // deep tile of the fused kernel / key tile of the CUDA-core kernel
    p.nsplit = nsplit;
    int chunk = (A_ub + nsplit - 1) / nsplit;
    chunk = (chunk + align - 1) / align * align;
    p.chunk = chunk < align ? align : chunk;
    p.part_bytes = verify_work_bytes(nrows, c->H, c->d, nsplit + 1);
    p.work_bytes = p.part_bytes;
}

cudaError_t launch_verify(const ripe_cache_s* c, const VerifyPlan& plan, int layer, const BranchArgs& ba,
                          const void* Q, const void* Kb, const void* Vb, const int32_t* ctx, float scale,
                          void* O, float* lse, void* work, cudaStream_t st) {
    VerifyArgs a;
    a.s = store_view(c);
    a.ba = ba;
    a.layer = layer;
    a.Q = (const char*)Q; a.Kb = (const char*)Kb; a.Vb = (const char*)Vb;
    a.O = (char*)O; a.lse = lse; a.ctx = ctx;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.nsplit = plan.nsplit; a.chunk = plan.chunk; a.nseg = plan.nsplit + 1;
    a.nrowchunks = plan.nrowchunks;
    a.q_tma = 0;
    char* wb = reinterpret_cast<char*>(work);
    a.part_ml = reinterpret_cast<float2*>(wb);
    a.part_o = reinterpret_cast<float*>(wb + verify_ml_bytes(ba.nrows, c->H, a.nseg));
    a.gE = plan.persist ? reinterpret_cast<int32_t*>(wb + verify_work_bytes(ba.nrows, c->H, c->d, a.nseg)) : nullptr;
    cudaError_t e;
    const int win_ub = plan.win_ub;
    if (plan.persist) {
        // The test hook is consumed by the launch it applies to.
        const long long probe = const_cast<ripe_cache_s*>(c)->probe_cycles.exchange(0);
        e = launch_persist(c->tmaps, a, plan.pd, plan.n_lo, plan.n_hi, plan.ndeep,
                           plan.nunits, plan.grid, plan.mt, probe, ba.sliding, c->full_box ? 1 : 0, st);
        if (e != cudaSuccess) return e;
    } else if (plan.fused) {
        // The whole call in one kernel; programmatic dependent launch lets its
        // prologue overlap the tail of the previous kernel in the stream.
        e = launch_fused(c->tmaps, a, plan.gslots, plan.mt, true, st);
        if (e != cudaSuccess) return e;
    } else {
        const int keys_ub = plan.chunk > win_ub ? plan.chunk : win_ub;
        if (c->dtype == RIPE_BF16) {
            e = launch_seg<__nv_bfloat16>(a, 0, a.nseg, ba.nbranch, keys_ub, st);
            if (e != cudaSuccess) return e;
            merge_kernel<__nv_bfloat16><<<ba.nbranch * c->H, 128, 0, st>>>(a);
        } else {
            e = launch_seg<float>(a, 0, a.nseg, ba.nbranch, keys_ub, st);
            if (e != cudaSuccess) return e;
            merge_kernel<float><<<ba.nbranch * c->H, 128, 0, st>>>(a);
        }
        ripe_count_launch();
    }
    return cudaGetLastError();
}
