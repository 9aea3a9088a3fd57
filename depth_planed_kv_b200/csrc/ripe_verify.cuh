// ripe_verify.cuh -- argument block shared by the verify kernels.
#pragma once

#include "ripe_internal.cuh"

struct VerifyArgs {
    StoreView s;
    BranchArgs ba;
    int layer;
    const char *Q, *Kb, *Vb;  // [nrows][H][d], cache dtype
    char* O;                  // [nrows][H][d], cache dtype
    float* lse;               // [nrows][H] or NULL
    const int32_t* ctx;       // per-sequence context length or NULL
    float scale_log2;         // softmax scale * log2(e)
    int nsplit, chunk, nseg;  // deep splits, keys per split, nsplit + 1
    int nrowchunks;           // row chunks per branch in the CUDA-core kernel
    float2* part_ml;          // [nrows][H][nseg] (m in log2 units, l)
    float* part_o;            // [nrows][H][nseg][d]
    int q_tma;                // fused kernel: a tensor map of Q came with the launch
    int32_t* gE;              // persistent kernel: per sequence group, its segment count (0: invalid group)
};

// Deep splits that hold keys for a sequence whose deep region has A keys.
__host__ __device__ inline int deep_splits_used(int A, int chunk, int nsplit) {
    const int n = (A + chunk - 1) / chunk;
    return n < nsplit ? n : nsplit;
}

// Scratch layout: the (m, l) pairs, padded to 256 bytes, then the o vectors.
inline size_t verify_ml_bytes(int nrows, int H, int nseg) {
    return ((size_t)nrows * H * nseg * sizeof(float2) + 255) / 256 * 256;
}
inline size_t verify_work_bytes(int nrows, int H, int d, int nseg) {
    return verify_ml_bytes(nrows, H, nseg) + (size_t)nrows * H * nseg * d * sizeof(float);
}
// The persistent kernel's scratch: the partials, then one segment count per group.
inline size_t persist_work_bytes(int nrows, int H, int d, int nseg, int ngroups) {
    return verify_work_bytes(nrows, H, d, nseg) + ((size_t)ngroups * sizeof(int32_t) + 255) / 256 * 256;
}
