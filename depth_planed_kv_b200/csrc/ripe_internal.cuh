// ripe_internal.cuh -- cache object, kernel argument blocks and device helpers
// shared by the libripe translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "../../include/ripe.h"

struct ripe_cache_s {
    int L, R, H, d, W, Tmax, Bmax, kmax, dtype, Wcap, esize;
    int device;
    size_t bytes;
    bool owns;
    char* base;
    char *kdeep, *vdeep, *kwin, *vwin;
    int32_t *len, *ws, *rfloor, *fbase, *fpos, *err;
    // Host-side upper bound of len over all sequences (grows with append/fill);
    // sizes the deep-region split grid without reading device metadata.
    int len_ub;
    // Verify scratch (per-split partial results), grown on demand.
    void* work;
    size_t work_bytes;
    // TMA descriptors (CUtensorMap), when the sm_100a kernels serve this cache
    // (bf16, d in {64, 96, 128}): deep K, V planes in 64-row boxes (deep region),
    // ring K, V planes and deep K, V planes in 16-row boxes (window tiles of the
    // cluster kernel), and the same four in 8-row boxes (window chunks of the
    // persistent kernel), and ring and deep planes in boxes of Wcap rows (a whole
    // ring plane in one box; only when Wcap <= 256, see full_box).
    alignas(64) unsigned char tmaps[14][128];
    bool full_box;
    bool tc_ready;
    // Test hook (ripe_debug_stall_next_verify): clock cycles of a wait that nothing
    // ends, taken by the next persistent-kernel verify; 0 = off.
    std::atomic<long long> probe_cycles{0};
    int all_depths_kernel = 0;  // RIPE_ALL_DEPTHS_* (ripe_cache_set_all_depths_kernel)
};

// Store geometry, passed by value to kernels.
struct StoreView {
    char *kdeep, *vdeep, *kwin, *vwin;
    // len: committed length; ws: window start; rfloor: lowest position whose ring
    // slots still hold its own planes (ws >= rfloor; evict leaves it alone);
    // fbase, fpos: a fork reads its deep positions below fpos from sequence fbase
    // (fbase = itself and fpos = 0 for a sequence that is not a fork).
    int32_t *len, *ws, *rfloor, *fbase, *fpos, *err;
    int L, R, H, d, Tmax, Bmax, Wcap, W, esize;
};

static inline StoreView store_view(const ripe_cache_s* c) {
    StoreView s;
    s.kdeep = c->kdeep; s.vdeep = c->vdeep; s.kwin = c->kwin; s.vwin = c->vwin;
    s.len = c->len; s.ws = c->ws; s.rfloor = c->rfloor; s.fbase = c->fbase; s.fpos = c->fpos; s.err = c->err;
    s.L = c->L; s.R = c->R; s.H = c->H; s.d = c->d; s.Tmax = c->Tmax; s.Bmax = c->Bmax;
    s.Wcap = c->Wcap; s.W = c->W; s.esize = c->esize;
    return s;
}

// Byte offset of row (layer, seq, head, position) of the deep plane.
__host__ __device__ inline int64_t deep_row(const StoreView& s, int l, int b, int h, int64_t p) {
    return ((((int64_t)l * s.Bmax + b) * s.H + h) * s.Tmax + p) * (int64_t)s.d * s.esize;
}

// The sequence whose deep plane holds position p of sequence b (its fork parent
// below the fork position, else b itself).
__device__ __forceinline__ int deep_owner(const StoreView& s, int b, int64_t p) {
    return p < s.fpos[b] ? s.fbase[b] : b;
}

// Byte offset of ring slot `slot` of plane r (1..R-1).
__host__ __device__ inline int64_t ring_row(const StoreView& s, int l, int b, int h, int r, int slot) {
    return (((((int64_t)l * s.Bmax + b) * s.H + h) * (s.R - 1) + (r - 1)) * s.Wcap + slot) *
           (int64_t)s.d * s.esize;
}

__device__ inline void set_device_error(int32_t* err, int code) { atomicCAS(err, 0, code); }

// One verify branch, decoded from an explicit table or the implicit all-depths form.
struct BranchArgs {
    const ripe_branch_t* table;  // NULL: implicit all-depths branches
    const int32_t* seq_ids;      // implicit form: nseq sequence ids
    int nbranch, nrows, k;       // k: tokens per branch in the implicit form
    int max_ntok;                // tokens per branch the launch grid covers
    int sliding;                 // per-query sliding window (implicit form, persistent kernel)
};

struct Branch {
    int seq, depth, ntok, row0, stride;
    bool ok;
};

__device__ inline Branch load_branch(const BranchArgs& ba, int R, int Bmax, int i) {
    Branch b;
    if (ba.table) {
        const ripe_branch_t t = ba.table[i];
        b.seq = t.seq; b.depth = t.depth; b.ntok = t.ntok; b.row0 = t.row0; b.stride = t.row_stride;
    } else {
        int s = i / R;
        b.depth = i % R + 1;
        b.seq = ba.seq_ids[s];
        b.ntok = ba.k;
        b.row0 = s * ba.k * R + b.depth - 1;
        b.stride = R;
    }
    int64_t last = (int64_t)b.row0 + (int64_t)(b.ntok > 0 ? b.ntok - 1 : 0) * b.stride;
    b.ok = b.seq >= 0 && b.seq < Bmax && b.depth >= 1 && b.depth <= R && b.ntok >= 0 &&
           b.ntok <= ba.max_ntok && b.row0 >= 0 && last < ba.nrows && last >= 0;
    return b;
}

// Committed length a verify attends to: len[b], or ctx_len[b] clamped to it.
__device__ inline int context_length(const int32_t* len, const int32_t* ctx, int32_t* err, int b,
                                     bool report) {
    int T = len[b];
    if (ctx) {
        int c = ctx[b];
        if (c > T) {
            if (report) set_device_error(err, RIPE_DEVERR_CTX);
        } else {
            T = c < 0 ? 0 : c;
        }
    }
    return T;
}

// ---------------------------------------------------------------------------
// Counter-based generator for synthetic stores (same definition as the
// documented Python generator: SplitMix64 output function, Irwin-Hall n=4).
// ---------------------------------------------------------------------------
__host__ __device__ inline uint64_t splitmix64_out(uint64_t x) {
    uint64_t z = x + 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

__device__ inline float synth_normal(uint64_t key, uint64_t idx) {
    uint64_t w = splitmix64_out(key + idx);
    int64_t s = (int64_t)((w & 0xFFFFull) + ((w >> 16) & 0xFFFFull) + ((w >> 32) & 0xFFFFull) + (w >> 48)) -
                131070;
    return __fmul_rn((float)s, __uint_as_float(0x37DDB3D7u));  // fl32(1/sqrt((2^32-1)/3))
}

__host__ __device__ inline uint64_t synth_index(int layer, int plane, int seq, int head, int64_t pos,
                                                 int chan) {
    return ((uint64_t)layer << 54) | ((uint64_t)plane << 48) | ((uint64_t)seq << 38) |
           ((uint64_t)head << 30) | ((uint64_t)pos << 10) | (uint64_t)chan;
}

// Kernel launch bookkeeping (counted on the host for every launch issued).
void ripe_count_launch(int n = 1);

// Per-device one-time set-up (kernel attributes such as the dynamic shared-memory
// limit belong to a device): `fn` runs once for each device it is reached on,
// with that device current; concurrent callers wait for the first.  A failed
// set-up is retried on the next call.
struct PerDeviceOnce {
    std::atomic<uint64_t> done{0};  // one bit per device ordinal < 64
    std::mutex mu;
};

template <typename F>
inline cudaError_t per_device_once(PerDeviceOnce& once, F&& fn) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    const uint64_t bit = 1ull << dev;
    if (once.done.load(std::memory_order_acquire) & bit) return cudaSuccess;
    std::lock_guard<std::mutex> lock(once.mu);
    if (once.done.load(std::memory_order_relaxed) & bit) return cudaSuccess;
    e = fn();
    if (e == cudaSuccess) once.done.fetch_or(bit, std::memory_order_release);
    return e;
}
