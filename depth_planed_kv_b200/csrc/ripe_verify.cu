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

namespace {

constexpr int kWarps = 4;
constexpr int kRowsPerWarp = 4;
constexpr int kRowsPerCta = kWarps * kRowsPerWarp;
constexpr int kTile = 32;

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

// One CTA: up to 16 rows of one branch, one head, one split.  Keys stream
// through shared memory 32 at a time; each warp owns 4 rows; a lane owns one
// key for the scores and d/32 output channels for the weighted sum.
template <typename Elem, int MAXD>
__global__ void __launch_bounds__(kWarps * 32)
split_kernel(VerifyArgs a, int seg_first, int seg_count) {
    constexpr int NV = MAXD / 32;
    __shared__ float q_s[kRowsPerCta][MAXD];
    __shared__ float k_s[kTile][MAXD + 1];
    __shared__ float v_s[kTile][MAXD];

    const StoreView& s = a.s;
    const int d = s.d, H = s.H;
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

    int64_t p0, p1;
    int nblk = 0;
    bool ring = false;
    if (seg < a.nsplit) {
        p0 = (int64_t)seg * a.chunk;
        p1 = min((int64_t)A, p0 + a.chunk);
        if (p0 >= p1) return;
    } else {
        p0 = A;
        p1 = T;
        nblk = j0 + nr;  // block tokens 0..j0+nr-1 are visible to some row here
        ring = r < s.R;
    }
    const int ncom = (int)(p1 - p0);
    const int nk = ncom + nblk;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    for (int e = threadIdx.x; e < nr * d; e += blockDim.x) {
        const int rr = e / d, c = e % d;
        const int64_t row = br.row0 + (int64_t)(j0 + rr) * br.stride;
        q_s[rr][c] = to_f32(reinterpret_cast<const Elem*>(a.Q)[(row * H + h) * d + c]) * a.scale_log2;
    }

    float m[kRowsPerWarp], l[kRowsPerWarp], o[kRowsPerWarp][NV];
#pragma unroll
    for (int t = 0; t < kRowsPerWarp; ++t) {
        m[t] = -INFINITY;
        l[t] = 0.f;
#pragma unroll
        for (int v = 0; v < NV; ++v) o[t][v] = 0.f;
    }

    for (int k0 = 0; k0 < nk; k0 += kTile) {
        __syncthreads();
        for (int e = threadIdx.x; e < kTile * d; e += blockDim.x) {
            const int key = e / d, c = e % d;
            const int t = k0 + key;
            float kx = 0.f, vx = 0.f;
            if (t < nk) {
                const Elem *kp, *vp;
                if (t < ncom) {
                    const int64_t p = p0 + t;
                    if (ring) {
                        const int64_t off = ring_row(s, a.layer, b, h, r, (int)(p % s.Wcap));
                        kp = reinterpret_cast<const Elem*>(s.kwin + off);
                        vp = reinterpret_cast<const Elem*>(s.vwin + off);
                    } else {
                        const int64_t off = deep_row(s, a.layer, b, h, p);
                        kp = reinterpret_cast<const Elem*>(s.kdeep + off);
                        vp = reinterpret_cast<const Elem*>(s.vdeep + off);
                    }
                } else {
                    const int64_t row = br.row0 + (int64_t)(t - ncom) * br.stride;
                    kp = reinterpret_cast<const Elem*>(a.Kb) + (row * H + h) * d;
                    vp = reinterpret_cast<const Elem*>(a.Vb) + (row * H + h) * d;
                }
                kx = to_f32(kp[c]);
                vx = to_f32(vp[c]);
            }
            k_s[key][c] = kx;
            v_s[key][c] = vx;
        }
        __syncthreads();
        const int t = k0 + lane;
#pragma unroll
        for (int rw = 0; rw < kRowsPerWarp; ++rw) {
            const int rr = warp + kWarps * rw;
            if (rr >= nr) break;
            const int j = j0 + rr;
            const bool valid = t < nk && (t < ncom || (t - ncom) <= j);
            float sc = -INFINITY;
            if (valid) {
                float acc = 0.f;
                for (int c = 0; c < d; ++c) acc = fmaf(q_s[rr][c], k_s[lane][c], acc);
                sc = acc;
            }
            const float mt = warp_max(sc);
            const float mn = fmaxf(m[rw], mt);
            if (mn == -INFINITY) continue;
            const float alpha = exp2f(m[rw] - mn);
            const float p = valid ? exp2f(sc - mn) : 0.f;
            l[rw] = l[rw] * alpha + warp_sum(p);
            m[rw] = mn;
#pragma unroll
            for (int v = 0; v < NV; ++v) o[rw][v] *= alpha;
            const int kmax = min(kTile, nk - k0);
            for (int key = 0; key < kmax; ++key) {
                const float pk = __shfl_sync(0xffffffffu, p, key);
#pragma unroll
                for (int v = 0; v < NV; ++v) {
                    const int c = lane + 32 * v;
                    if (c < d) o[rw][v] = fmaf(pk, v_s[key][c], o[rw][v]);
                }
            }
        }
    }

#pragma unroll
    for (int rw = 0; rw < kRowsPerWarp; ++rw) {
        const int rr = warp + kWarps * rw;
        if (rr >= nr) break;
        const int64_t row = br.row0 + (int64_t)(j0 + rr) * br.stride;
        const int64_t pi = (row * H + h) * a.nseg + seg;
        if (lane == 0) a.part_ml[pi] = make_float2(m[rw], l[rw]);
#pragma unroll
        for (int v = 0; v < NV; ++v) {
            const int c = lane + 32 * v;
            if (c < d) a.part_o[pi * d + c] = o[rw][v];
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

template <typename Elem>
cudaError_t launch_split(const VerifyArgs& a, int seg_first, int seg_count, int nbranch, cudaStream_t st) {
    const int64_t grid = (int64_t)nbranch * a.nrowchunks * a.s.H * seg_count;
    if (grid == 0) return cudaSuccess;
    if (grid > 0x7fffffff) return cudaErrorInvalidConfiguration;
    if (a.s.d <= 64)
        split_kernel<Elem, 64><<<(unsigned)grid, kWarps * 32, 0, st>>>(a, seg_first, seg_count);
    else
        split_kernel<Elem, 128><<<(unsigned)grid, kWarps * 32, 0, st>>>(a, seg_first, seg_count);
    ripe_count_launch();
    return cudaGetLastError();
}

}  // namespace

VerifyPlan plan_verify(const ripe_cache_s* c, int nbranch, int nrows, int max_ntok, bool all_depths) {
    VerifyPlan p{};
    p.max_ntok = max_ntok;
    p.rows_chunk = kRowsPerCta;
    p.nrowchunks = (max_ntok + kRowsPerCta - 1) / kRowsPerCta;
    if (p.nrowchunks < 1) p.nrowchunks = 1;
    const int A_ub = c->len_ub < c->Tmax ? c->len_ub : c->Tmax;
    p.tc_deep = c->tc_ready && deep_tc_supported(c->dtype, c->d);
    int64_t ns;
    if (p.tc_deep) {
        // One deep CTA per (sequence group, head, split); splits only until the
        // CTAs cover the 148 SMs once (each CTA holds one SM's tensor memory).
        p.gslots = all_depths ? nbranch / c->R : (nbranch < c->Bmax ? nbranch : c->Bmax);
        p.mt = (all_depths && max_ntok * c->R > 128) ? 2 : 1;
        const int64_t units = (int64_t)p.gslots * c->H;
        ns = units > 0 ? 148 / units : 1;
        const int64_t max_ns = (A_ub + 255) / 256;
        if (ns > max_ns) ns = max_ns;
        if (ns < 1) ns = 1;
        p.nsplit = (int)ns;
        int chunk = (int)((A_ub + ns - 1) / ns);
        chunk = (chunk + 63) / 64 * 64;
        p.chunk = chunk < 64 ? 64 : chunk;
    } else {
        const int64_t items = (int64_t)nbranch * p.nrowchunks * c->H;
        const int64_t target = 148 * 8;
        ns = items > 0 ? (target + items - 1) / items : 1;
        const int64_t max_ns = (A_ub + 63) / 64;
        if (ns > max_ns) ns = max_ns;
        if (ns < 1) ns = 1;
        p.nsplit = (int)ns;
        int chunk = (int)((A_ub + ns - 1) / ns);
        chunk = (chunk + 31) / 32 * 32;
        p.chunk = chunk < 32 ? 32 : chunk;
        p.mt = 0;
        p.gslots = 0;
    }
    p.work_bytes = verify_work_bytes(nrows, c->H, c->d, p.nsplit + 1);
    return p;
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
    a.part_ml = reinterpret_cast<float2*>(work);
    a.part_o = reinterpret_cast<float*>(reinterpret_cast<char*>(work) +
                                        verify_ml_bytes(ba.nrows, c->H, a.nseg));
    cudaError_t e;
    if (plan.tc_deep) {
        // Deep region on the tensor cores, then the window/block split, then the merge.
        e = launch_deep_tc(c->tmap_k, c->tmap_v, a, plan.gslots, plan.mt, st);
        if (e != cudaSuccess) return e;
        e = launch_split<__nv_bfloat16>(a, a.nsplit, 1, ba.nbranch, st);
        if (e != cudaSuccess) return e;
        merge_kernel<__nv_bfloat16><<<ba.nbranch * c->H, 128, 0, st>>>(a);
        ripe_count_launch();
    } else if (c->dtype == RIPE_BF16) {
        e = launch_split<__nv_bfloat16>(a, 0, a.nseg, ba.nbranch, st);
        if (e != cudaSuccess) return e;
        merge_kernel<__nv_bfloat16><<<ba.nbranch * c->H, 128, 0, st>>>(a);
        ripe_count_launch();
    } else {
        e = launch_split<float>(a, 0, a.nseg, ba.nbranch, st);
        if (e != cudaSuccess) return e;
        merge_kernel<float><<<ba.nbranch * c->H, 128, 0, st>>>(a);
        ripe_count_launch();
    }
    return cudaGetLastError();
}
