// ripe_accept.cu -- the acceptance step of self-speculative decoding in a looped
// model, LoopSpec order (LoopSpec article, rit.work: sections on the second
// branch and on the final check): for each draft position, first try the early
// draft x1 against the final distribution p, then the fallback x2 prepared from a
// deeper state, and only after both are rejected restart with a draw from what p
// still has to give.
//
// For position j of a sequence, with p, q1, qf the softmaxes of the final, draft
// and deeper logits at the temperature:
//   accept x1        if u0 * q1(x1) < p(x1);
//   else p1 = norm((p - q1)+) (p itself if that has no mass);
//   fallback present if qf(x1) < q1(x1) at temperature 1 (the deeper state lowered
//                    its confidence in x1) and q2 = norm((qf - q1)+) has mass;
//   accept x2        if u1 * q2(x2) < p1(x2);
//   else restart     with the smallest v whose running sum of w = norm((p1 - q2)+)
//                    (p1 without a fallback; p1 if w has no mass) exceeds u2 * sum(w).
// Temperature 0 is greedy: accept x1 iff it is the argmax of the final logits
// (lowest index on ties), then x2 likewise when the fallback is present, else emit
// that argmax.  The block of k positions stops at the first rejected x1.
//
// One CTA per sequence, positions in order; every quantity is a block-wide
// reduction over the vocabulary (fp32, expf), the logits re-read from L2.
#include <math.h>

#include "ripe_internal.cuh"
#include "ripe_launch.h"

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;

struct Red {
    float* f;  // [kWarps] scratch
    int* i;    // [kWarps] scratch
};

__device__ float block_sum(float v, Red r) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int w = threadIdx.x / 32, l = threadIdx.x % 32;
    __syncthreads();
    if (l == 0) r.f[w] = v;
    __syncthreads();
    float t = 0.f;
    for (int k = 0; k < kWarps; ++k) t += r.f[k];  // same order in every thread
    return t;
}

__device__ float block_max(float v, Red r) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int w = threadIdx.x / 32, l = threadIdx.x % 32;
    __syncthreads();
    if (l == 0) r.f[w] = v;
    __syncthreads();
    float t = -INFINITY;
    for (int k = 0; k < kWarps; ++k) t = fmaxf(t, r.f[k]);
    return t;
}

// Index of the largest value, lowest index on ties (-1 if every value is -inf/NaN).
__device__ int block_argmax(const float* z, int V, Red r) {
    float best = -INFINITY;
    int bi = -1;
    for (int v = threadIdx.x; v < V; v += kThreads) {  // ascending: ties keep the first
        const float x = z[v];
        if (bi < 0 || x > best) {
            best = x;
            bi = v;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, best, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (oi >= 0 && (bi < 0 || ob > best || (ob == best && oi < bi))) {
            best = ob;
            bi = oi;
        }
    }
    const int w = threadIdx.x / 32, l = threadIdx.x % 32;
    __syncthreads();
    if (l == 0) {
        r.f[w] = best;
        r.i[w] = bi;
    }
    __syncthreads();
    float tb = -INFINITY;
    int ti = -1;
    for (int k = 0; k < kWarps; ++k) {
        const int oi = r.i[k];
        const float ob = r.f[k];
        if (oi >= 0 && (ti < 0 || ob > tb || (ob == tb && oi < ti))) {
            tb = ob;
            ti = oi;
        }
    }
    return ti;
}

// Softmax statistics of z at inverse temperature it: max of z*it and sum of exp.
struct Sm {
    float m, s, it;
    __device__ float prob(float z) const { return expf(z * it - m) / s; }
};

__device__ Sm softmax_stats(const float* z, int V, float it, Red r) {
    float mx = -INFINITY;
    for (int v = threadIdx.x; v < V; v += kThreads) mx = fmaxf(mx, z[v] * it);
    Sm sm;
    sm.it = it;
    sm.m = block_max(mx, r);
    float s = 0.f;
    for (int v = threadIdx.x; v < V; v += kThreads) s += expf(z[v] * it - sm.m);
    sm.s = block_sum(s, r);
    return sm;
}

// Inverse-CDF draw from the non-negative weights w(v) (a functor): the smallest v
// whose running sum exceeds u * total.  Each thread owns a contiguous slice of the
// vocabulary; slice sums are scanned in thread order.
template <typename W>
__device__ int block_draw(W w, int V, float u, Red r, float* scan) {
    const int per = (V + kThreads - 1) / kThreads;
    const int v0 = threadIdx.x * per, v1 = min(V, v0 + per);
    float local = 0.f;
    for (int v = v0; v < v1; ++v) local += w(v);
    __syncthreads();
    scan[threadIdx.x] = local;
    __syncthreads();
    if (threadIdx.x == 0) {  // exclusive prefix over the slices, in order
        float acc = 0.f;
        for (int t = 0; t < kThreads; ++t) {
            const float x = scan[t];
            scan[t] = acc;
            acc += x;
        }
        scan[kThreads] = acc;
    }
    __syncthreads();
    const float total = scan[kThreads];
    const float thr = u * total;
    int found = V;  // none
    float acc = scan[threadIdx.x];
    if (acc <= thr && local > 0.f) {
        for (int v = v0; v < v1; ++v) {
            acc += w(v);
            if (acc > thr) {
                found = v;
                break;
            }
        }
    }
    // the smallest token found; if rounding left none, the last token with weight
    int lastpos = -1;
    for (int v = v0; v < v1; ++v)
        if (w(v) > 0.f) lastpos = v;
    __syncthreads();
    if (threadIdx.x < kWarps) r.i[threadIdx.x] = V;
    __syncthreads();
    atomicMin(&r.i[threadIdx.x / 32], found);
    __syncthreads();
    int best = V;
    for (int k = 0; k < kWarps; ++k) best = min(best, r.i[k]);
    if (best < V) return best;
    __syncthreads();
    if (threadIdx.x < kWarps) r.i[threadIdx.x] = -1;
    __syncthreads();
    atomicMax(&r.i[threadIdx.x / 32], lastpos);
    __syncthreads();
    int last = -1;
    for (int k = 0; k < kWarps; ++k) last = max(last, r.i[k]);
    return last;
}

__global__ void __launch_bounds__(kThreads) accept_kernel(int k, int V, const float* __restrict__ zp_all,
                                                          const float* __restrict__ zq_all,
                                                          const float* __restrict__ zf_all,
                                                          const int32_t* __restrict__ x1_all,
                                                          const int32_t* __restrict__ x2_all,
                                                          const float* __restrict__ u_all, float temperature,
                                                          int32_t* n_acc, int32_t* token, int32_t* path) {
    __shared__ float red_f[kWarps];
    __shared__ int red_i[kWarps];
    __shared__ float scan[kThreads + 1];
    const Red r{red_f, red_i};
    const int b = blockIdx.x;
    int j = 0, tok = -1, pth = 0;
    for (; j < k; ++j) {
        const int64_t off = ((int64_t)b * k + j) * V;
        const float* zp = zp_all + off;
        const float* zq = zq_all + off;
        const float* zf = zf_all ? zf_all + off : nullptr;
        const int x1 = x1_all[(int64_t)b * k + j];
        const int x2 = x2_all ? x2_all[(int64_t)b * k + j] : -1;
        const float* u = u_all + ((int64_t)b * k + j) * 3;
        const bool x1_ok = x1 >= 0 && x1 < V, x2_ok = x2 >= 0 && x2 < V;
        // the gate: the deeper state lowered its confidence in x1 (temperature 1)
        bool gate = false;
        if (zf && x1_ok) {
            const Sm f1 = softmax_stats(zf, V, 1.f, r), q1t = softmax_stats(zq, V, 1.f, r);
            gate = f1.prob(zf[x1]) < q1t.prob(zq[x1]);
        }
        if (temperature == 0.f) {
            const int best = block_argmax(zp, V, r);
            if (x1 == best) continue;
            tok = (gate && x2 == best) ? x2 : best;
            pth = (gate && x2 == best) ? 1 : 2;
            break;
        }
        const float it = 1.f / temperature;
        const Sm P = softmax_stats(zp, V, it, r), Q = softmax_stats(zq, V, it, r);
        if (x1_ok && u[0] * Q.prob(zq[x1]) < P.prob(zp[x1])) continue;
        // what p still has to give after the first proposal
        float z1 = 0.f;
        for (int v = threadIdx.x; v < V; v += kThreads) z1 += fmaxf(P.prob(zp[v]) - Q.prob(zq[v]), 0.f);
        z1 = block_sum(z1, r);
        const bool p1_is_p = !(z1 > 0.f);
        auto p1 = [&](int v) { return p1_is_p ? P.prob(zp[v]) : fmaxf(P.prob(zp[v]) - Q.prob(zq[v]), 0.f) / z1; };
        if (gate) {
            const Sm F = softmax_stats(zf, V, it, r);
            float z2 = 0.f;
            for (int v = threadIdx.x; v < V; v += kThreads) z2 += fmaxf(F.prob(zf[v]) - Q.prob(zq[v]), 0.f);
            z2 = block_sum(z2, r);
            if (z2 > 0.f) {
                auto q2 = [&](int v) { return fmaxf(F.prob(zf[v]) - Q.prob(zq[v]), 0.f) / z2; };
                if (x2_ok && u[1] * q2(x2) < p1(x2)) {
                    tok = x2;
                    pth = 1;
                    break;
                }
                float z3 = 0.f;
                for (int v = threadIdx.x; v < V; v += kThreads) z3 += fmaxf(p1(v) - q2(v), 0.f);
                z3 = block_sum(z3, r);
                if (z3 > 0.f)
                    tok = block_draw([&](int v) { return fmaxf(p1(v) - q2(v), 0.f); }, V, u[2], r, scan);
                else
                    tok = block_draw(p1, V, u[2], r, scan);
                pth = 2;
                break;
            }
        }
        tok = block_draw(p1, V, u[2], r, scan);
        pth = 2;
        break;
    }
    if (threadIdx.x == 0) {
        n_acc[b] = j;
        token[b] = j < k ? tok : -1;
        path[b] = j < k ? pth : 0;
    }
}

}  // namespace

cudaError_t launch_accept(int nseq, int k, int V, const float* zp, const float* zq, const float* zf, const int32_t* x1,
                          const int32_t* x2, const float* u, float temperature, int32_t* n_acc, int32_t* token,
                          int32_t* path, cudaStream_t st) {
    accept_kernel<<<nseq, kThreads, 0, st>>>(k, V, zp, zq, zf, x1, x2, u, temperature, n_acc, token, path);
    ripe_count_launch();
    return cudaGetLastError();
}
