// ripe_launch.h -- host-side launchers of the libripe kernels (internal).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

struct ripe_cache_s;
struct BranchArgs;

cudaError_t launch_append(const ripe_cache_s* c, const int32_t* seq_ids, const int32_t* n_acc, int nseq,
                          const void* K, const void* V, int kmax_in, cudaStream_t st);
cudaError_t launch_evict(const ripe_cache_s* c, const int32_t* seq_ids, int nseq, cudaStream_t st);
cudaError_t launch_reset(const ripe_cache_s* c, const int32_t* seq_ids, int nseq, cudaStream_t st);
cudaError_t launch_truncate(const ripe_cache_s* c, const int32_t* seq_ids, const int32_t* new_len, int nseq,
                            cudaStream_t st);
cudaError_t launch_init_meta(const ripe_cache_s* c, cudaStream_t st);
cudaError_t launch_fork(const ripe_cache_s* c, const int32_t* parents, const int32_t* children, int nseq,
                        cudaStream_t st);
cudaError_t launch_synth_fill(const ripe_cache_s* c, int b, int T, uint64_t seed, const float* coef,
                              cudaStream_t st);

// Verify plan: how the deep region is split and how much scratch the call needs.
struct VerifyPlan {
    int nsplit;        // deep-region splits (partials 0..nsplit-1); the window+block partial is nsplit
    int chunk;         // keys per deep split
    int nrowchunks;    // row chunks per branch (CUDA-core kernel)
    int max_ntok;      // host bound on tokens per branch
    bool fused;        // the whole call in an sm_100a kernel (tcgen05 deep region)
    bool persist;      // ... the persistent all-depths kernel (else the cluster kernel)
    int mt;            // M tiles (of 128 rows) per fused CTA
    int gslots;        // fused CTAs along the sequence-group axis
    int a_ub;          // bound on the deep region's length the splits cover
    int win_ub;        // bound on a branch's window + block keys (CUDA-core kernel)
    // persistent kernel: CTAs, CTAs with deep items, window units per deep / other CTA
    int grid, pd, n_lo, n_hi, ndeep, nunits;
    size_t part_bytes; // per-split partial results
    size_t work_bytes; // scratch needed (the partials)
};

// `capacity`: plan for every length the store can hold (Tmax), not for the host's
// bound on the current lengths -- for launches captured into a CUDA graph, which
// replay while the sequences grow.
VerifyPlan plan_verify(const ripe_cache_s* c, int nbranch, int nrows, int max_ntok, bool all_depths,
                       bool capacity, bool sliding = false);
// True while `st` is being captured into a CUDA graph.
bool stream_capturing(cudaStream_t st);
// Re-plan with `nsplit` deep splits (chunk and scratch size follow).
void plan_set_splits(VerifyPlan& p, const ripe_cache_s* c, int nrows, int nsplit);

struct VerifyArgs;
bool fused_supported(int dtype, int d);
cudaError_t launch_fused(const void* tmaps, const VerifyArgs& a, int gslots, int mt, bool pdl, cudaStream_t st);
// The persistent kernel, then the kernel that merges its partials.
cudaError_t launch_persist(const void* tmaps, const VerifyArgs& a, int pd, int n_lo, int n_hi,
                           int ndeep, int nunits, int grid, int mt, long long probe_cycles, int sliding,
                           int full_box, cudaStream_t st);
// Window warps of a deep CTA and of another CTA of the persistent kernel (0: no kernel).
void persist_shape(int d, int mt, int* nww_deep, int* nww_other);
// The persistent kernel's window units go through its stage ring (producer warps).
bool persist_ring_ok(int d, int mt, int Wcap, int k, int sliding, int full_box);
// The fourteen tensor maps of the sm_100a kernels (0 on success).
int make_tensor_maps(ripe_cache_s* c);
// A tensor map of this call's Q as [rows][H][d], 128-row boxes of one head (false: none).
struct CUtensorMap_st;
bool make_q_map(void* tmap, const VerifyArgs& a);
// SMs of the current device (cached per device).
int device_sm_count();

cudaError_t launch_accept(int nseq, int k, int V, const float* zp, const float* zq, const float* zf, const int32_t* x1,
                          const int32_t* x2, const float* u, float temperature, int32_t* n_acc, int32_t* token,
                          int32_t* path, cudaStream_t st);

// `part`: scratch for the partial results (plan.part_bytes).
cudaError_t launch_verify(const ripe_cache_s* c, const VerifyPlan& plan, int layer, const BranchArgs& ba,
                          const void* Q, const void* Kb, const void* Vb, const int32_t* ctx, float scale,
                          void* O, float* lse, void* part, cudaStream_t st);

// Record a one-line message for ripe_last_error() and return `status`.
int ripe_fail(int status, const char* fmt, ...);
