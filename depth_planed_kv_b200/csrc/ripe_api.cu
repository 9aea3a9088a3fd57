// ripe_api.cu -- the C ABI of libripe (include/ripe.h): argument checks, the
// store allocation, scratch management and kernel sequencing.  Every compute
// step runs in the kernels of ripe_store.cu, ripe_verify.cu and
// ripe_deep_sm100.cu; this file only validates and launches.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <new>
#include <string>

#include "ripe_internal.cuh"
#include "ripe_launch.h"

namespace {

thread_local std::string g_last_error;
std::atomic<uint64_t> g_launches{0};

int fail(int status, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return status;
}

int cuda_fail(cudaError_t e, const char* what) {
    return fail(RIPE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace

bool stream_capturing(cudaStream_t st) {
    if (!st) return false;  // the legacy default stream is never captured
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return cs != cudaStreamCaptureStatusNone;
}

namespace {

struct Layout {
    size_t kdeep, vdeep, kwin, vwin, len, ws, rfloor, base, fpos, err, total;
};

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

int check_dims(int layers, int R, int H, int d, int W, int Tmax, int max_seqs, int kmax, int dtype) {
    if (layers < 1 || layers > 64) return fail(RIPE_ERR_INVALID_ARG, "layers=%d outside [1,64]", layers);
    if (R < 1 || R > 64) return fail(RIPE_ERR_INVALID_ARG, "R=%d outside [1,64]", R);
    if (H < 1 || H > 256) return fail(RIPE_ERR_INVALID_ARG, "H=%d outside [1,256]", H);
    if (dtype != RIPE_BF16 && dtype != RIPE_F32) return fail(RIPE_ERR_INVALID_ARG, "dtype=%d", dtype);
    if (d < 8 || d > 128) return fail(RIPE_ERR_UNSUPPORTED, "d=%d outside [8,128]", d);
    const int es = dtype == RIPE_BF16 ? 2 : 4;
    if ((d * es) % 16) return fail(RIPE_ERR_UNALIGNED, "d*sizeof(element)=%d not a multiple of 16", d * es);
    if (W < 0) return fail(RIPE_ERR_INVALID_ARG, "W=%d < 0", W);
    if (Tmax < 1 || Tmax > (1 << 24)) return fail(RIPE_ERR_INVALID_ARG, "Tmax=%d outside [1,2^24]", Tmax);
    if (max_seqs < 1 || max_seqs > 1024) return fail(RIPE_ERR_INVALID_ARG, "max_seqs=%d outside [1,1024]", max_seqs);
    if (kmax < 1 || kmax > 4096) return fail(RIPE_ERR_INVALID_ARG, "kmax=%d outside [1,4096]", kmax);
    if ((int64_t)W + kmax > (1 << 24)) return fail(RIPE_ERR_INVALID_ARG, "W+kmax too large");
    return RIPE_OK;
}

Layout layout_of(int L, int R, int H, int d, int W, int Tmax, int Bmax, int kmax, int dtype) {
    const size_t es = dtype == RIPE_BF16 ? 2 : 4;
    const size_t Wcap = (size_t)W + kmax;
    Layout y;
    y.kdeep = 0;
    const size_t deep = round256((size_t)L * Bmax * H * Tmax * d * es);
    const size_t ring = round256((size_t)L * Bmax * H * (R - 1) * Wcap * d * es);
    y.vdeep = y.kdeep + deep;
    y.kwin = y.vdeep + deep;
    y.vwin = y.kwin + ring;
    y.len = y.vwin + ring;
    y.ws = y.len + round256(sizeof(int32_t) * Bmax);
    y.rfloor = y.ws + round256(sizeof(int32_t) * Bmax);
    y.base = y.rfloor + round256(sizeof(int32_t) * Bmax);
    y.fpos = y.base + round256(sizeof(int32_t) * Bmax);
    y.err = y.fpos + round256(sizeof(int32_t) * Bmax);
    y.total = y.err + 256;
    return y;
}

cudaStream_t as_stream(ripe_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

// A cache's store and scratch live on the device it was created on; every call
// that enqueues work must find that device current.
int check_cache(ripe_cache_t c) {
    if (!c) return fail(RIPE_ERR_INVALID_ARG, "cache is NULL");
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != c->device)
        return fail(RIPE_ERR_INVALID_ARG, "the current device (%d) is not the cache's device (%d)", dev, c->device);
    return RIPE_OK;
}

int ensure_workspace(ripe_cache_s* c, size_t need, cudaStream_t st) {
    if (need <= c->work_bytes) return RIPE_OK;
    if (st) {
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        cudaError_t e = cudaStreamIsCapturing(st, &cs);
        if (e != cudaSuccess) return cuda_fail(e, "cudaStreamIsCapturing");
        if (cs != cudaStreamCaptureStatusNone)
            return fail(RIPE_ERR_CAPTURING, "verify scratch must grow to %zu bytes during capture; "
                        "call ripe_reserve_workspace first", need);
    }
    if (c->work) {
        cudaError_t e = cudaDeviceSynchronize();
        if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
        cudaFree(c->work);
        c->work = nullptr;
        c->work_bytes = 0;
    }
    size_t sz = need + need / 4;
    void* p = nullptr;
    if (cudaMalloc(&p, sz) != cudaSuccess) {
        cudaGetLastError();
        return fail(RIPE_ERR_OOM, "cudaMalloc(%zu) for verify scratch failed", sz);
    }
    // Zeroed once, so that no partial a kernel skips reads as NaN.
    cudaError_t e = cudaMemset(p, 0, sz);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
        cudaFree(p);
        return cuda_fail(e, "zeroing the verify scratch");
    }
    c->work = p;
    c->work_bytes = sz;
    return RIPE_OK;
}

int verify_common(ripe_cache_s* c, int layer, const BranchArgs& ba, const void* Q, const void* Kb,
                  const void* Vb, const int32_t* ctx, float scale, void* O, float* lse, cudaStream_t st) {
    if (layer < 0 || layer >= c->L) return fail(RIPE_ERR_INVALID_ARG, "layer=%d outside [0,%d)", layer, c->L);
    if (ba.nbranch < 0 || ba.nrows < 0) return fail(RIPE_ERR_INVALID_ARG, "negative branch or row count");
    if (ba.nbranch == 0 || ba.nrows == 0) return RIPE_OK;
    if (!Q || !Kb || !Vb || !O) return fail(RIPE_ERR_INVALID_ARG, "Q, Kblk, Vblk and O must be non-NULL");
    if (!aligned16(Q) || !aligned16(Kb) || !aligned16(Vb) || !aligned16(O))
        return fail(RIPE_ERR_UNALIGNED, "Q, Kblk, Vblk and O must be 16-byte aligned");
    if (lse && ((uintptr_t)lse & 3u)) return fail(RIPE_ERR_UNALIGNED, "lse must be 4-byte aligned");
    if (!(scale == scale) || isinf(scale)) return fail(RIPE_ERR_INVALID_ARG, "scale is not finite");
    if (scale == 0.f) scale = 1.0f / sqrtf((float)c->d);
    // A captured launch replays while the sequences grow: its plan covers Tmax.
    const VerifyPlan plan = plan_verify(c, ba.nbranch, ba.nrows, ba.max_ntok, ba.table == nullptr,
                                        stream_capturing(st), ba.sliding != 0);
    if (ba.sliding && !plan.persist)
        return fail(RIPE_ERR_UNSUPPORTED, "the sliding window needs the persistent sm_100a kernel (bf16, d in "
                    "{64,96,128}, k*R <= 256)");
    int rc = ensure_workspace(c, plan.work_bytes, st);
    if (rc != RIPE_OK) return rc;
    cudaError_t e = launch_verify(c, plan, layer, ba, Q, Kb, Vb, ctx, scale, O, lse, c->work, st);
    if (e != cudaSuccess) return cuda_fail(e, "verify launch");
    return RIPE_OK;
}

}  // namespace

void ripe_count_launch(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

int ripe_fail(int status, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return status;
}

extern "C" {

const char* ripe_error_string(int status) {
    switch (status) {
        case RIPE_OK: return "ok";
        case RIPE_ERR_INVALID_ARG: return "invalid argument";
        case RIPE_ERR_CAPACITY: return "capacity exceeded";
        case RIPE_ERR_UNALIGNED: return "unaligned pointer or row size";
        case RIPE_ERR_OOM: return "device allocation failed";
        case RIPE_ERR_CUDA: return "CUDA runtime error";
        case RIPE_ERR_DEVICE: return "device-side check failed";
        case RIPE_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case RIPE_ERR_CAPTURING: return "allocation needed during stream capture";
        default: return "unknown status";
    }
}

const char* ripe_last_error(void) { return g_last_error.c_str(); }

uint64_t ripe_launch_count(void) { return g_launches.load(); }

int ripe_cache_bytes(int layers, int R, int H, int d, int W, int Tmax, int max_seqs, int kmax, int dtype,
                     size_t* bytes) {
    int rc = check_dims(layers, R, H, d, W, Tmax, max_seqs, kmax, dtype);
    if (rc != RIPE_OK) return rc;
    if (!bytes) return fail(RIPE_ERR_INVALID_ARG, "bytes is NULL");
    *bytes = layout_of(layers, R, H, d, W, Tmax, max_seqs, kmax, dtype).total;
    return RIPE_OK;
}

int ripe_cache_create(int layers, int R, int H, int d, int W, int Tmax, int max_seqs, int kmax, int dtype,
                      void* dev_mem, ripe_cache_t* out) {
    if (!out) return fail(RIPE_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    int rc = check_dims(layers, R, H, d, W, Tmax, max_seqs, kmax, dtype);
    if (rc != RIPE_OK) return rc;
    if (dev_mem && ((uintptr_t)dev_mem & 255u)) return fail(RIPE_ERR_UNALIGNED, "dev_mem must be 256-byte aligned");
    const Layout y = layout_of(layers, R, H, d, W, Tmax, max_seqs, kmax, dtype);
    ripe_cache_s* c = new (std::nothrow) ripe_cache_s();
    if (!c) return fail(RIPE_ERR_OOM, "host allocation failed");
    c->L = layers; c->R = R; c->H = H; c->d = d; c->W = W; c->Tmax = Tmax; c->Bmax = max_seqs;
    c->kmax = kmax; c->dtype = dtype; c->Wcap = W + kmax; c->esize = dtype == RIPE_BF16 ? 2 : 4;
    c->bytes = y.total;
    cudaGetDevice(&c->device);
    if (dev_mem) {
        c->base = (char*)dev_mem;
        c->owns = false;
    } else {
        void* p = nullptr;
        if (cudaMalloc(&p, y.total) != cudaSuccess) {
            cudaGetLastError();
            delete c;
            return fail(RIPE_ERR_OOM, "cudaMalloc(%zu) for the store failed", y.total);
        }
        c->base = (char*)p;
        c->owns = true;
    }
    c->kdeep = c->base + y.kdeep; c->vdeep = c->base + y.vdeep;
    c->kwin = c->base + y.kwin; c->vwin = c->base + y.vwin;
    c->len = (int32_t*)(c->base + y.len); c->ws = (int32_t*)(c->base + y.ws);
    c->rfloor = (int32_t*)(c->base + y.rfloor);
    c->fbase = (int32_t*)(c->base + y.base);
    c->fpos = (int32_t*)(c->base + y.fpos);
    c->err = (int32_t*)(c->base + y.err);
    c->tc_ready = false;
    if (fused_supported(dtype, d)) {
        const int tm = make_tensor_maps(c);
        c->tc_ready = tm == 0;
        if (!c->tc_ready)
            fail(RIPE_OK, "tensor maps of this store cannot be built (code %d); verify uses the CUDA-core "
                 "kernels (ripe_cache_verify_path reports 0)", tm);
    }
    // Zeroed store: key tiles that overrun a region read finite values.  Every
    // sequence starts as the owner of its own deep plane (not a fork).
    cudaError_t e = cudaMemset(c->base, 0, y.total);
    if (e == cudaSuccess) e = launch_init_meta(c, nullptr);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
        if (c->owns) cudaFree(c->base);
        delete c;
        return cuda_fail(e, "zeroing the store");
    }
    *out = c;
    return RIPE_OK;
}

int ripe_cache_destroy(ripe_cache_t c) {
    if (!c) return fail(RIPE_ERR_INVALID_ARG, "cache is NULL");
    cudaDeviceSynchronize();
    if (c->work) cudaFree(c->work);
    if (c->owns) cudaFree(c->base);
    delete c;
    return RIPE_OK;
}

int ripe_cache_reset(ripe_cache_t c, const int32_t* seq_ids, int nseq, ripe_stream_t stream) {
    int rc = check_cache(c);
    if (rc != RIPE_OK) return rc;
    if (nseq < 0 || nseq > c->Bmax) return fail(RIPE_ERR_INVALID_ARG, "nseq=%d outside [0,%d]", nseq, c->Bmax);
    if (nseq == 0) return RIPE_OK;
    if (!seq_ids) return fail(RIPE_ERR_INVALID_ARG, "seq_ids is NULL");
    cudaError_t e = launch_reset(c, seq_ids, nseq, as_stream(stream));
    return e == cudaSuccess ? RIPE_OK : cuda_fail(e, "reset launch");
}

int ripe_append(ripe_cache_t c, const int32_t* seq_ids, const int32_t* n_acc, int nseq, const void* K,
                const void* V, int kmax_in, ripe_stream_t stream) {
    int rc = check_cache(c);
    if (rc != RIPE_OK) return rc;
    if (nseq < 0 || nseq > c->Bmax) return fail(RIPE_ERR_INVALID_ARG, "nseq=%d outside [0,%d]", nseq, c->Bmax);
    if (kmax_in < 1) return fail(RIPE_ERR_INVALID_ARG, "kmax_in=%d < 1", kmax_in);
    if (kmax_in > c->Tmax) return fail(RIPE_ERR_CAPACITY, "kmax_in=%d > Tmax=%d", kmax_in, c->Tmax);
    if (nseq == 0) return RIPE_OK;
    if (!seq_ids || !n_acc || !K || !V) return fail(RIPE_ERR_INVALID_ARG, "NULL pointer argument");
    if (!aligned16(K) || !aligned16(V)) return fail(RIPE_ERR_UNALIGNED, "K and V must be 16-byte aligned");
    const cudaStream_t st = as_stream(stream);
    cudaError_t e = launch_append(c, seq_ids, n_acc, nseq, K, V, kmax_in, st);
    if (e != cudaSuccess) return cuda_fail(e, "append launch");
    // The host's bound on the lengths; a captured append may replay any number of times.
    const int64_t ub = (int64_t)c->len_ub + kmax_in;
    c->len_ub = stream_capturing(st) ? c->Tmax : (int)(ub < c->Tmax ? ub : c->Tmax);
    return RIPE_OK;
}

int ripe_evict(ripe_cache_t c, const int32_t* seq_ids, int nseq, ripe_stream_t stream) {
    int rc = check_cache(c);
    if (rc != RIPE_OK) return rc;
    if (nseq < 0 || nseq > c->Bmax) return fail(RIPE_ERR_INVALID_ARG, "nseq=%d outside [0,%d]", nseq, c->Bmax);
    if (nseq == 0) return RIPE_OK;
    if (!seq_ids) return fail(RIPE_ERR_INVALID_ARG, "seq_ids is NULL");
    cudaError_t e = launch_evict(c, seq_ids, nseq, as_stream(stream));
    return e == cudaSuccess ? RIPE_OK : cuda_fail(e, "evict launch");
}

int ripe_fork(ripe_cache_t c, const int32_t* parent_ids, const int32_t* child_ids, int nseq, ripe_stream_t stream) {
    int rc = check_cache(c);
    if (rc != RIPE_OK) return rc;
    if (nseq < 0 || nseq > c->Bmax) return fail(RIPE_ERR_INVALID_ARG, "nseq=%d outside [0,%d]", nseq, c->Bmax);
    if (nseq == 0) return RIPE_OK;
    if (!parent_ids || !child_ids) return fail(RIPE_ERR_INVALID_ARG, "NULL pointer argument");
    cudaError_t e = launch_fork(c, parent_ids, child_ids, nseq, as_stream(stream));
    return e == cudaSuccess ? RIPE_OK : cuda_fail(e, "fork launch");
}

int ripe_truncate(ripe_cache_t c, const int32_t* seq_ids, const int32_t* new_len, int nseq,
                  ripe_stream_t stream) {
    int rc = check_cache(c);
    if (rc != RIPE_OK) return rc;
    if (nseq < 0 || nseq > c->Bmax) return fail(RIPE_ERR_INVALID_ARG, "nseq=%d outside [0,%d]", nseq, c->Bmax);
    if (nseq == 0) return RIPE_OK;
    if (!seq_ids || !new_len) return fail(RIPE_ERR_INVALID_ARG, "NULL pointer argument");
    cudaError_t e = launch_truncate(c, seq_ids, new_len, nseq, as_stream(stream));
    return e == cudaSuccess ? RIPE_OK : cuda_fail(e, "truncate launch");
}

int ripe_verify_attn(ripe_cache_t c, int layer, const ripe_branch_t* branches, int nbranch, int nrows,
                     const void* Q, const void* Kb, const void* Vb, const int32_t* ctx, float scale, void* O,
                     float* lse, ripe_stream_t stream) {
    int rc = check_cache(c);
    if (rc != RIPE_OK) return rc;
    if (nbranch > 0 && !branches) return fail(RIPE_ERR_INVALID_ARG, "branches is NULL");
    if (branches && !aligned16(branches)) return fail(RIPE_ERR_UNALIGNED, "branches must be 16-byte aligned");
    BranchArgs ba{};
    ba.table = branches;
    ba.nbranch = nbranch;
    ba.nrows = nrows;
    ba.max_ntok = c->kmax;
    return verify_common(c, layer, ba, Q, Kb, Vb, ctx, scale, O, lse, as_stream(stream));
}

int ripe_verify_attn_all_depths(ripe_cache_t c, int layer, const int32_t* seq_ids, int nseq, int k,
                                const void* Q, const void* Kb, const void* Vb, const int32_t* ctx, float scale,
                                void* O, float* lse, ripe_stream_t stream) {
    int rc = check_cache(c);
    if (rc != RIPE_OK) return rc;
    if (nseq < 0 || nseq > c->Bmax) return fail(RIPE_ERR_INVALID_ARG, "nseq=%d outside [0,%d]", nseq, c->Bmax);
    if (k < 1 || k > 4096) return fail(RIPE_ERR_INVALID_ARG, "k=%d outside [1,4096]", k);
    if (nseq > 0 && !seq_ids) return fail(RIPE_ERR_INVALID_ARG, "seq_ids is NULL");
    const int64_t nrows = (int64_t)nseq * k * c->R;
    if (nrows > (1 << 30)) return fail(RIPE_ERR_INVALID_ARG, "too many rows");
    BranchArgs ba{};
    ba.table = nullptr;
    ba.seq_ids = seq_ids;
    ba.nbranch = nseq * c->R;
    ba.nrows = (int)nrows;
    ba.k = k;
    ba.max_ntok = k;
    return verify_common(c, layer, ba, Q, Kb, Vb, ctx, scale, O, lse, as_stream(stream));
}

int ripe_verify_attn_all_depths_sliding(ripe_cache_t c, int layer, const int32_t* seq_ids, int nseq, int k,
                                        const void* Q, const void* Kb, const void* Vb, const int32_t* ctx,
                                        float scale, void* O, float* lse, ripe_stream_t stream) {
    int rc = check_cache(c);
    if (rc != RIPE_OK) return rc;
    if (nseq < 0 || nseq > c->Bmax) return fail(RIPE_ERR_INVALID_ARG, "nseq=%d outside [0,%d]", nseq, c->Bmax);
    if (k < 1 || k > 4096) return fail(RIPE_ERR_INVALID_ARG, "k=%d outside [1,4096]", k);
    if (nseq > 0 && !seq_ids) return fail(RIPE_ERR_INVALID_ARG, "seq_ids is NULL");
    BranchArgs ba{};
    ba.table = nullptr;
    ba.seq_ids = seq_ids;
    ba.nbranch = nseq * c->R;
    ba.nrows = nseq * k * c->R;
    ba.k = k;
    ba.max_ntok = k;
    ba.sliding = 1;
    return verify_common(c, layer, ba, Q, Kb, Vb, ctx, scale, O, lse, as_stream(stream));
}

int ripe_reserve_workspace(ripe_cache_t c, int max_rows) {
    int rc = check_cache(c);
    if (rc != RIPE_OK) return rc;
    if (max_rows < 0) return fail(RIPE_ERR_INVALID_ARG, "max_rows < 0");
    // The most scratch a call of up to max_rows rows can take under capture: the
    // fewest branches and tokens per branch give the most splits, and captured
    // calls plan for Tmax.
    const VerifyPlan plan = plan_verify(c, 1, max_rows, 1, false, true);
    return ensure_workspace(c, plan.work_bytes, nullptr);
}

int ripe_synth_fill(ripe_cache_t c, const int32_t* seq_ids, const int32_t* T, int nseq, uint64_t seed,
                    const float* coef, ripe_stream_t stream) {
    int rc = check_cache(c);
    if (rc != RIPE_OK) return rc;
    if (nseq < 0 || nseq > c->Bmax) return fail(RIPE_ERR_INVALID_ARG, "nseq=%d outside [0,%d]", nseq, c->Bmax);
    if (nseq > 0 && (!seq_ids || !T || !coef)) return fail(RIPE_ERR_INVALID_ARG, "NULL pointer argument");
    if (seed >= (1ull << 47)) return fail(RIPE_ERR_INVALID_ARG, "seed must be < 2^47");
    for (int i = 0; i < nseq; ++i) {
        if (seq_ids[i] < 0 || seq_ids[i] >= c->Bmax) return fail(RIPE_ERR_INVALID_ARG, "seq id %d", seq_ids[i]);
        if (T[i] < 0 || T[i] > c->Tmax) return fail(RIPE_ERR_CAPACITY, "T=%d outside [0,Tmax]", T[i]);
        if (T[i] >= (1 << 19)) return fail(RIPE_ERR_INVALID_ARG, "synthetic positions must be < 2^19");
    }
    if (c->H > 256 || c->L > 64 || c->Bmax > 1024) return fail(RIPE_ERR_UNSUPPORTED, "generator index range");
    for (int i = 0; i < nseq; ++i) {
        cudaError_t e = launch_synth_fill(c, seq_ids[i], T[i], seed, coef, as_stream(stream));
        if (e != cudaSuccess) return cuda_fail(e, "synthetic fill launch");
        if (T[i] > c->len_ub) c->len_ub = T[i];
    }
    return RIPE_OK;
}

int ripe_accept(int nseq, int k, int V, const float* zp, const float* zq, const float* zf, const int32_t* x1,
                const int32_t* x2, const float* u, float temperature, int32_t* n_accepted, int32_t* token,
                int32_t* path, ripe_stream_t stream) {
    if (nseq < 0 || nseq > (1 << 20)) return fail(RIPE_ERR_INVALID_ARG, "nseq=%d outside [0, 2^20]", nseq);
    if (k < 1 || k > 4096) return fail(RIPE_ERR_INVALID_ARG, "k=%d outside [1, 4096]", k);
    if (V < 1 || V > (1 << 24)) return fail(RIPE_ERR_INVALID_ARG, "V=%d outside [1, 2^24]", V);
    if (!(temperature >= 0.f) || isinf(temperature))
        return fail(RIPE_ERR_INVALID_ARG, "temperature must be finite and >= 0");
    if (nseq == 0) return RIPE_OK;
    if (!zp || !zq || !x1 || !u || !n_accepted || !token || !path || (zf && !x2))
        return fail(RIPE_ERR_INVALID_ARG, "NULL pointer argument (x2 is required with zf)");
    const auto mis = [](const void* p) { return ((uintptr_t)p & 3u) != 0; };
    if (mis(zp) || mis(zq) || (zf && mis(zf)) || mis(x1) || (x2 && mis(x2)) || mis(u) || mis(n_accepted) ||
        mis(token) || mis(path))
        return fail(RIPE_ERR_UNALIGNED, "arrays must be 4-byte aligned");
    cudaError_t e = launch_accept(nseq, k, V, zp, zq, zf, x1, x2, u, temperature, n_accepted, token, path,
                                  as_stream(stream));
    return e == cudaSuccess ? RIPE_OK : cuda_fail(e, "accept launch");
}

int ripe_debug_stall_next_verify(ripe_cache_t c, long long cycles) {
    int rc = check_cache(c);
    if (rc != RIPE_OK) return rc;
    if (cycles < 0 || cycles > (1ll << 31)) return fail(RIPE_ERR_INVALID_ARG, "cycles=%lld outside [0, 2^31]", cycles);
    c->probe_cycles.store(cycles);
    return RIPE_OK;
}

int ripe_cache_set_all_depths_kernel(ripe_cache_t c, int kernel) {
    int rc = check_cache(c);
    if (rc != RIPE_OK) return rc;
    if (kernel != RIPE_ALL_DEPTHS_AUTO && kernel != RIPE_ALL_DEPTHS_PERSISTENT && kernel != RIPE_ALL_DEPTHS_CLUSTER)
        return fail(RIPE_ERR_INVALID_ARG, "kernel=%d is not a RIPE_ALL_DEPTHS_* value", kernel);
    c->all_depths_kernel = kernel;
    return RIPE_OK;
}

int ripe_cache_verify_path(ripe_cache_t c, int* path) {
    int rc = check_cache(c);
    if (rc != RIPE_OK) return rc;
    if (!path) return fail(RIPE_ERR_INVALID_ARG, "path is NULL");
    *path = c->tc_ready ? RIPE_PATH_FUSED_SM100 : RIPE_PATH_CUDA_CORE;
    return RIPE_OK;
}

int ripe_cache_buffers(ripe_cache_t c, void** kdeep, void** vdeep, void** kwin, void** vwin, int32_t** len,
                       int32_t** ws, int32_t** rfloor) {
    int rc = check_cache(c);
    if (rc != RIPE_OK) return rc;
    if (kdeep) *kdeep = c->kdeep;
    if (vdeep) *vdeep = c->vdeep;
    if (kwin) *kwin = c->kwin;
    if (vwin) *vwin = c->vwin;
    if (len) *len = c->len;
    if (ws) *ws = c->ws;
    if (rfloor) *rfloor = c->rfloor;
    return RIPE_OK;
}

int ripe_read_forks(ripe_cache_t c, int32_t* fbase_host, int32_t* fpos_host, ripe_stream_t stream) {
    int rc = check_cache(c);
    if (rc != RIPE_OK) return rc;
    cudaStream_t st = as_stream(stream);
    cudaError_t e = cudaSuccess;
    if (fbase_host)
        e = cudaMemcpyAsync(fbase_host, c->fbase, sizeof(int32_t) * c->Bmax, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess && fpos_host)
        e = cudaMemcpyAsync(fpos_host, c->fpos, sizeof(int32_t) * c->Bmax, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    return e == cudaSuccess ? RIPE_OK : cuda_fail(e, "read_forks");
}

int ripe_read_meta(ripe_cache_t c, int32_t* len_host, int32_t* ws_host, int32_t* rfloor_host,
                   ripe_stream_t stream) {
    int rc = check_cache(c);
    if (rc != RIPE_OK) return rc;
    cudaStream_t st = as_stream(stream);
    cudaError_t e = cudaSuccess;
    if (len_host) e = cudaMemcpyAsync(len_host, c->len, sizeof(int32_t) * c->Bmax, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess && ws_host)
        e = cudaMemcpyAsync(ws_host, c->ws, sizeof(int32_t) * c->Bmax, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess && rfloor_host)
        e = cudaMemcpyAsync(rfloor_host, c->rfloor, sizeof(int32_t) * c->Bmax, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    return e == cudaSuccess ? RIPE_OK : cuda_fail(e, "read_meta");
}

int ripe_get_device_error(ripe_cache_t c, int32_t* code_host, ripe_stream_t stream) {
    int rc = check_cache(c);
    if (rc != RIPE_OK) return rc;
    if (!code_host) return fail(RIPE_ERR_INVALID_ARG, "code_host is NULL");
    cudaStream_t st = as_stream(stream);
    cudaError_t e = cudaMemcpyAsync(code_host, c->err, sizeof(int32_t), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(c->err, 0, sizeof(int32_t), st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    return e == cudaSuccess ? RIPE_OK : cuda_fail(e, "get_device_error");
}

}  // extern "C"
