// ripe_noalloc.cu -- ripe_verify_attn_noalloc: the branch-list verify for callers
// that must not allocate device memory.
//
// Who needs it: an inference server that has handed almost all of HBM to its own
// pool (KV pages, activations) and forbids out-of-band cudaMalloc; code that
// enqueues work from inside a stream capture, where cudaMalloc breaks the
// capture; and latency-critical paths where cudaMalloc's implicit device
// synchronisation cannot be paid.  For them the per-split partial results live
// in one fixed device array that this file owns, instead of the cache's
// grow-on-demand scratch.
//
// The array is a file-scope __device__ variable, so every GPU on which this
// library's device code is loaded holds it (kStaticScratchBytes) until the
// process exits.  Host code cannot use the array's name as a device address;
// the address is fetched once per device with cudaGetSymbolAddress, with that
// device current, on the first call made on that device.
#include <math.h>

#include <mutex>

#include "ripe_internal.cuh"
#include "ripe_launch.h"
#include "ripe_verify.cuh"

namespace {

constexpr size_t kStaticScratchBytes = RIPE_NOALLOC_SCRATCH_BYTES;  // 32 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_verify_scratch[kStaticScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices];

// Device address of g_verify_scratch on the current device (looked up once per device).
cudaError_t static_scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_verify_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" int ripe_verify_attn_noalloc(ripe_cache_t c, int layer, const ripe_branch_t* branches, int nbranch,
                                        int nrows, const void* Q, const void* Kb, const void* Vb,
                                        const int32_t* ctx, float scale, void* O, float* lse,
                                        ripe_stream_t stream, size_t* scratch_needed) {
    if (scratch_needed) *scratch_needed = 0;
    if (!c) return ripe_fail(RIPE_ERR_INVALID_ARG, "cache is NULL");
    // The static array's address is per device: the call must run on the cache's device.
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess || cur != c->device)
        return ripe_fail(RIPE_ERR_INVALID_ARG, "the current device (%d) is not the cache's device (%d)", cur,
                         c->device);
    if (layer < 0 || layer >= c->L || nbranch < 0 || nrows < 0)
        return ripe_fail(RIPE_ERR_INVALID_ARG, "layer, branch or row count out of range");
    if (nbranch == 0 || nrows == 0) return RIPE_OK;
    if (!branches || !Q || !Kb || !Vb || !O) return ripe_fail(RIPE_ERR_INVALID_ARG, "NULL pointer argument");
    const auto mis = [](const void* p) { return ((uintptr_t)p & 15u) != 0; };
    if (mis(branches) || mis(Q) || mis(Kb) || mis(Vb) || mis(O) || (lse && ((uintptr_t)lse & 3u)))
        return ripe_fail(RIPE_ERR_UNALIGNED, "device pointers must be 16-byte aligned (lse 4-byte)");
    if (!(scale == scale) || isinf(scale)) return ripe_fail(RIPE_ERR_INVALID_ARG, "scale is not finite");
    if (scale == 0.f) scale = 1.0f / sqrtf((float)c->d);

    BranchArgs ba{};
    ba.table = branches;
    ba.nbranch = nbranch;
    ba.nrows = nrows;
    ba.max_ntok = c->kmax;
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    VerifyPlan plan = plan_verify(c, nbranch, nrows, c->kmax, false, stream_capturing(st));
    // A branch list never takes the persistent all-depths kernel.  Fewer, longer
    // deep splits until the partial results fit the fixed array.
    while (plan.part_bytes > kStaticScratchBytes && plan.nsplit > 1) plan_set_splits(plan, c, nrows, plan.nsplit / 2);
    if (scratch_needed) *scratch_needed = plan.part_bytes;
    if (plan.persist || plan.part_bytes > kStaticScratchBytes)
        return ripe_fail(RIPE_ERR_CAPACITY, "this call needs %zu bytes of scratch; the static scratch holds %zu",
                         plan.part_bytes, kStaticScratchBytes);
    void* work = nullptr;
    cudaError_t e = static_scratch_address(&work);
    if (e != cudaSuccess)
        return ripe_fail(RIPE_ERR_CUDA, "cudaGetSymbolAddress of the static scratch: %s", cudaGetErrorString(e));
    e = launch_verify(c, plan, layer, ba, Q, Kb, Vb, ctx, scale, O, lse, work, st);
    if (e != cudaSuccess) return ripe_fail(RIPE_ERR_CUDA, "verify launch: %s", cudaGetErrorString(e));
    return RIPE_OK;
}
