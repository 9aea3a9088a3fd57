// ripe_store.cu -- RIPE store maintenance: append, evict, reset, truncate and
// the synthetic fill.  All are bandwidth-trivial next to verify; they move 16-byte
// vectors and touch per-sequence metadata with one thread per sequence.
#include "ripe_internal.cuh"
#include "ripe_launch.h"

namespace {

constexpr int kThreads = 256;

inline int grid_for(int64_t work, int threads) {
    int64_t g = (work + threads - 1) / threads;
    if (g > 148 * 64) g = 148 * 64;  // grid-stride beyond 64 CTAs per SM
    return (int)(g < 1 ? 1 : g);
}

// Positions T..T+n-1 of each listed sequence get their planes: the deepest into
// Kdeep/Vdeep, planes 1..R-1 of the last min(n, Wcap) positions into the ring.
// Reads len before append_meta_kernel updates it (stream order).
__global__ void append_copy_kernel(StoreView s, const int32_t* __restrict__ seq_ids,
                                   const int32_t* __restrict__ n_acc, int nseq, const char* __restrict__ K,
                                   const char* __restrict__ V, int kmax_in) {
    const int vecs = s.d * s.esize / 16;
    const int64_t total = (int64_t)s.L * nseq * kmax_in * s.R * s.H * vecs;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        int64_t x = e;
        const int v = (int)(x % vecs); x /= vecs;
        const int h = (int)(x % s.H); x /= s.H;
        const int rp = (int)(x % s.R); x /= s.R;
        const int t = (int)(x % kmax_in); x /= kmax_in;
        const int i = (int)(x % nseq);
        const int l = (int)(x / nseq);
        const int b = seq_ids[i];
        const int n = n_acc[i];
        if (b < 0 || b >= s.Bmax || n < 0 || n > kmax_in || t >= n) continue;
        const int T = s.len[b];
        if (T + n > s.Tmax) continue;
        const int64_t p = (int64_t)T + t;
        const int64_t src = e * 16;  // input is dense [L][nseq][kmax_in][R][H][d]
        const uint4 kv = *reinterpret_cast<const uint4*>(K + src);
        const uint4 vv = *reinterpret_cast<const uint4*>(V + src);
        if (rp == s.R - 1) {
            const int64_t dst = deep_row(s, l, b, h, p) + v * 16;
            *reinterpret_cast<uint4*>(s.kdeep + dst) = kv;
            *reinterpret_cast<uint4*>(s.vdeep + dst) = vv;
        } else if (t >= n - s.Wcap) {
            const int64_t dst = ring_row(s, l, b, h, rp + 1, (int)(p % s.Wcap)) + v * 16;
            *reinterpret_cast<uint4*>(s.kwin + dst) = kv;
            *reinterpret_cast<uint4*>(s.vwin + dst) = vv;
        }
    }
}

__global__ void append_meta_kernel(StoreView s, const int32_t* __restrict__ seq_ids,
                                   const int32_t* __restrict__ n_acc, int nseq, int kmax_in) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= nseq) return;
    const int b = seq_ids[i];
    const int n = n_acc[i];
    if (b < 0 || b >= s.Bmax) { set_device_error(s.err, RIPE_DEVERR_SEQ_RANGE); return; }
    if (n < 0 || n > kmax_in) { set_device_error(s.err, RIPE_DEVERR_COUNT); return; }
    const int T = s.len[b];
    if (T + n > s.Tmax) { set_device_error(s.err, RIPE_DEVERR_CAPACITY); return; }
    const int nl = T + n;
    s.len[b] = nl;
    // Positions below nl - Wcap no longer (or never) hold their planes in the ring.
    if (nl - s.Wcap > s.ws[b]) s.ws[b] = nl - s.Wcap;
    if (nl - s.Wcap > s.rfloor[b]) s.rfloor[b] = nl - s.Wcap;
}

__global__ void evict_kernel(StoreView s, const int32_t* __restrict__ seq_ids, int nseq) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= nseq) return;
    const int b = seq_ids[i];
    if (b < 0 || b >= s.Bmax) { set_device_error(s.err, RIPE_DEVERR_SEQ_RANGE); return; }
    const int lo = s.len[b] - s.W;
    if (lo > s.ws[b]) s.ws[b] = lo;
}

__global__ void reset_kernel(StoreView s, const int32_t* __restrict__ seq_ids, int nseq) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= nseq) return;
    const int b = seq_ids[i];
    if (b < 0 || b >= s.Bmax) { set_device_error(s.err, RIPE_DEVERR_SEQ_RANGE); return; }
    s.len[b] = 0;
    s.ws[b] = 0;
    s.rfloor[b] = 0;
    s.fbase[b] = b;  // a released fork no longer reads its parent
    s.fpos[b] = 0;
}

// Every sequence starts as its own deep-plane owner (not a fork).
__global__ void init_meta_kernel(StoreView s) {
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b < s.Bmax) s.fbase[b] = b;
}

// A (parent, child) pair of ripe_fork is valid when both ids are in range and
// distinct and the parent is not itself a fork.
__device__ __forceinline__ bool fork_pair_ok(const StoreView& s, int p, int c) {
    return p >= 0 && p < s.Bmax && c >= 0 && c < s.Bmax && p != c && s.fbase[p] == p;
}

// Branch fork (LoopSpec article, deployment section: a KV cache per branch): the
// child takes copies of the parent's deep rows from its fork position
// f = floor64(T) to T and of the parent's whole ring; rows below f stay in the
// parent and are read through fbase/fpos.  16-byte vectors; per pair and (layer,
// head) 64 deep rows (those at f + i < T) and (R-1)*Wcap ring rows.
__global__ void fork_copy_kernel(StoreView s, const int32_t* __restrict__ parents,
                                 const int32_t* __restrict__ children, int nseq) {
    const int vecs = s.d * s.esize / 16;
    const int ring_rows = (s.R - 1) * s.Wcap;
    const int rows = 64 + ring_rows;
    const int64_t total = (int64_t)nseq * s.L * s.H * rows * vecs;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        int64_t x = e;
        const int v = (int)(x % vecs); x /= vecs;
        const int row = (int)(x % rows); x /= rows;
        const int h = (int)(x % s.H); x /= s.H;
        const int l = (int)(x % s.L);
        const int i = (int)(x / s.L);
        const int p = parents[i], c = children[i];
        if (!fork_pair_ok(s, p, c)) continue;
        if (row < 64) {
            const int T = s.len[p];
            const int64_t pos = (int64_t)(T / 64 * 64) + row;
            if (pos >= T) continue;
            const int64_t src = deep_row(s, l, p, h, pos) + v * 16, dst = deep_row(s, l, c, h, pos) + v * 16;
            *reinterpret_cast<uint4*>(s.kdeep + dst) = *reinterpret_cast<const uint4*>(s.kdeep + src);
            *reinterpret_cast<uint4*>(s.vdeep + dst) = *reinterpret_cast<const uint4*>(s.vdeep + src);
        } else {
            const int rr = row - 64;
            const int r = rr / s.Wcap + 1, slot = rr % s.Wcap;
            const int64_t src = ring_row(s, l, p, h, r, slot) + v * 16, dst = ring_row(s, l, c, h, r, slot) + v * 16;
            *reinterpret_cast<uint4*>(s.kwin + dst) = *reinterpret_cast<const uint4*>(s.kwin + src);
            *reinterpret_cast<uint4*>(s.vwin + dst) = *reinterpret_cast<const uint4*>(s.vwin + src);
        }
    }
}

__global__ void fork_meta_kernel(StoreView s, const int32_t* __restrict__ parents,
                                 const int32_t* __restrict__ children, int nseq) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= nseq) return;
    const int p = parents[i], c = children[i];
    if (!fork_pair_ok(s, p, c)) { set_device_error(s.err, RIPE_DEVERR_FORK); return; }
    const int T = s.len[p];
    s.len[c] = T;
    s.ws[c] = s.ws[p];
    s.rfloor[c] = s.rfloor[p];
    s.fbase[c] = p;
    s.fpos[c] = T / 64 * 64;
}

// Rollback to the confirmed prefix (LoopSpec article, section on the second
// branch): the state an evict at the confirmed length leaves, as far as the ring
// still holds the planes -- positions pushed out of the window only by the
// rejected tokens return to it.  len = min(len, T'), rfloor = min(rfloor, len),
// ws = min(ws, max(len - W, rfloor)).  T' >= len changes nothing.
__global__ void truncate_kernel(StoreView s, const int32_t* __restrict__ seq_ids,
                                const int32_t* __restrict__ new_len, int nseq) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= nseq) return;
    const int b = seq_ids[i];
    if (b < 0 || b >= s.Bmax) { set_device_error(s.err, RIPE_DEVERR_SEQ_RANGE); return; }
    int T = s.len[b];
    const int t = new_len[i];
    // A fork is never cut below its fork position (release it instead).
    if (t < 0 || (s.fbase[b] != b && t < s.fpos[b])) { set_device_error(s.err, RIPE_DEVERR_COUNT); return; }
    if (t < T) T = t;
    const int rf = min(s.rfloor[b], T);
    s.len[b] = T;
    s.rfloor[b] = rf;
    s.ws[b] = min(s.ws[b], max(T - s.W, rf));
}

struct Coefs { float c[64]; };

// Synthetic fill of one sequence: the state one append of T positions leaves.
template <typename Elem>
__global__ void synth_fill_kernel(StoreView s, int b, int T, uint64_t seed, Coefs cf) {
    const uint64_t keyK = splitmix64_out((seed << 16) + 1), keyV = splitmix64_out((seed << 16) + 2);
    const uint64_t nkK = splitmix64_out((seed << 16) + 3), nkV = splitmix64_out((seed << 16) + 4);
    const int lo = T - s.Wcap > 0 ? T - s.Wcap : 0;
    const int nwin = T - lo;
    // Work: deep elements (L*H*T*d), then ring elements (L*H*(R-1)*nwin*d).
    const int64_t deep_n = (int64_t)s.L * s.H * T * s.d;
    const int64_t ring_n = (int64_t)s.L * s.H * (s.R - 1) * nwin * s.d;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < deep_n + ring_n;
         e += (int64_t)gridDim.x * blockDim.x) {
        if (e < deep_n) {
            int64_t x = e;
            const int c = (int)(x % s.d); x /= s.d;
            const int64_t p = x % T; x /= T;
            const int h = (int)(x % s.H);
            const int l = (int)(x / s.H);
            const uint64_t idx = synth_index(l, 0, b, h, p, c);
            const float zk = synth_normal(keyK, idx), zv = synth_normal(keyV, idx);
            Elem* kd = reinterpret_cast<Elem*>(s.kdeep + deep_row(s, l, b, h, p)) + c;
            Elem* vd = reinterpret_cast<Elem*>(s.vdeep + deep_row(s, l, b, h, p)) + c;
            if constexpr (sizeof(Elem) == 2) { *kd = __float2bfloat16_rn(zk); *vd = __float2bfloat16_rn(zv); }
            else { *kd = zk; *vd = zv; }
        } else {
            int64_t x = e - deep_n;
            const int c = (int)(x % s.d); x /= s.d;
            const int64_t p = lo + x % nwin; x /= nwin;
            const int r = (int)(x % (s.R - 1)) + 1; x /= (s.R - 1);
            const int h = (int)(x % s.H);
            const int l = (int)(x / s.H);
            const uint64_t di = synth_index(l, 0, b, h, p, c), ni = synth_index(l, r, b, h, p, c);
            const float k = __fadd_rn(__fmul_rn(cf.c[r - 1], synth_normal(nkK, ni)), synth_normal(keyK, di));
            const float v = __fadd_rn(__fmul_rn(cf.c[r - 1], synth_normal(nkV, ni)), synth_normal(keyV, di));
            const int64_t off = ring_row(s, l, b, h, r, (int)(p % s.Wcap));
            Elem* kw = reinterpret_cast<Elem*>(s.kwin + off) + c;
            Elem* vw = reinterpret_cast<Elem*>(s.vwin + off) + c;
            if constexpr (sizeof(Elem) == 2) { *kw = __float2bfloat16_rn(k); *vw = __float2bfloat16_rn(v); }
            else { *kw = k; *vw = v; }
        }
    }
}

__global__ void set_meta_kernel(StoreView s, int b, int T) {
    s.len[b] = T;
    s.ws[b] = T - s.Wcap > 0 ? T - s.Wcap : 0;
    s.rfloor[b] = s.ws[b];
    s.fbase[b] = b;
    s.fpos[b] = 0;
}

}  // namespace

cudaError_t launch_append(const ripe_cache_s* c, const int32_t* seq_ids, const int32_t* n_acc, int nseq,
                          const void* K, const void* V, int kmax_in, cudaStream_t st) {
    StoreView s = store_view(c);
    const int64_t total = (int64_t)s.L * nseq * kmax_in * s.R * s.H * (s.d * s.esize / 16);
    append_copy_kernel<<<grid_for(total, kThreads), kThreads, 0, st>>>(
        s, seq_ids, n_acc, nseq, (const char*)K, (const char*)V, kmax_in);
    append_meta_kernel<<<(nseq + 127) / 128, 128, 0, st>>>(s, seq_ids, n_acc, nseq, kmax_in);
    ripe_count_launch(2);
    return cudaGetLastError();
}

cudaError_t launch_evict(const ripe_cache_s* c, const int32_t* seq_ids, int nseq, cudaStream_t st) {
    evict_kernel<<<(nseq + 127) / 128, 128, 0, st>>>(store_view(c), seq_ids, nseq);
    ripe_count_launch();
    return cudaGetLastError();
}

cudaError_t launch_reset(const ripe_cache_s* c, const int32_t* seq_ids, int nseq, cudaStream_t st) {
    reset_kernel<<<(nseq + 127) / 128, 128, 0, st>>>(store_view(c), seq_ids, nseq);
    ripe_count_launch();
    return cudaGetLastError();
}

cudaError_t launch_init_meta(const ripe_cache_s* c, cudaStream_t st) {
    init_meta_kernel<<<(c->Bmax + 127) / 128, 128, 0, st>>>(store_view(c));
    ripe_count_launch();
    return cudaGetLastError();
}

cudaError_t launch_fork(const ripe_cache_s* c, const int32_t* parents, const int32_t* children, int nseq,
                        cudaStream_t st) {
    StoreView s = store_view(c);
    const int64_t total = (int64_t)nseq * s.L * s.H * (64 + (s.R - 1) * s.Wcap) * (s.d * s.esize / 16);
    fork_copy_kernel<<<grid_for(total, kThreads), kThreads, 0, st>>>(s, parents, children, nseq);
    fork_meta_kernel<<<(nseq + 127) / 128, 128, 0, st>>>(s, parents, children, nseq);
    ripe_count_launch(2);
    return cudaGetLastError();
}

cudaError_t launch_truncate(const ripe_cache_s* c, const int32_t* seq_ids, const int32_t* new_len, int nseq,
                            cudaStream_t st) {
    truncate_kernel<<<(nseq + 127) / 128, 128, 0, st>>>(store_view(c), seq_ids, new_len, nseq);
    ripe_count_launch();
    return cudaGetLastError();
}

cudaError_t launch_synth_fill(const ripe_cache_s* c, int b, int T, uint64_t seed, const float* coef,
                              cudaStream_t st) {
    StoreView s = store_view(c);
    Coefs cf;
    for (int r = 0; r < 64; ++r) cf.c[r] = r < s.R ? coef[r] : 0.f;
    const int lo = T - s.Wcap > 0 ? T - s.Wcap : 0;
    const int64_t work = (int64_t)s.L * s.H * T * s.d + (int64_t)s.L * s.H * (s.R - 1) * (T - lo) * s.d;
    if (work > 0) {
        if (c->dtype == RIPE_BF16)
            synth_fill_kernel<__nv_bfloat16><<<grid_for(work, kThreads), kThreads, 0, st>>>(s, b, T, seed, cf);
        else
            synth_fill_kernel<float><<<grid_for(work, kThreads), kThreads, 0, st>>>(s, b, T, seed, cf);
        ripe_count_launch();
    }
    set_meta_kernel<<<1, 1, 0, st>>>(s, b, T);
    ripe_count_launch();
    return cudaGetLastError();
}
