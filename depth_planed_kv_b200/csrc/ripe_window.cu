// ripe_window.cu -- the window planes and the draft block of RIPE verify-attention,
// and the final merge of each row's partial results.
//
// A query at loop depth r reads plane r of the positions still inside the window
// (RIPE abstract, sentence introducing RIPE) and the draft-block tokens of its own
// branch at plane r.  Those keys differ from depth to depth, so nothing can be
// stacked across depths: a unit is one (branch, head, chunk of <= 16 rows) and its
// work is two small dense products, S = Q K^T ([rows x d] . [d x keys]) and
// O = P V.  One warp owns one unit:
//   - K, V and Q rows arrive in the warp's shared-memory slice by 16-byte
//     asynchronous copies (rows at a padded stride: ldmatrix without conflicts);
//   - both products run on warp-level tensor-core MMA tiles (m16n8k16, bf16 in,
//     fp32 accumulate) -- a unit has 4-16 rows, too few for a 64/128-row tcgen05
//     tile, while a CUDA-core formulation needs ~6-10 K instructions per unit;
//   - the online softmax runs on the fp32 fragments with quad-shuffle max/sum,
//     and P goes from the S fragments straight into the A fragments of P V.
//
// Merge: the window warp and the deep CTAs of the same (branch, row chunk, head)
// each write a partial (m, l, o) and then count their arrival; whoever arrives
// last merges -- M = max m, L = sum l 2^(m-M), O = sum o 2^(m-M) / L, deep
// splits in order and this partial last, the same operation order on both sides
// -- and writes O and the LSE.  No one waits for anyone.
#include "ripe_launch.h"
#include "ripe_verify.cuh"
#include "sm100_ptx.cuh"

namespace {

constexpr int kRowChunk = 16;      // rows of a branch per unit (the launch's row chunks)
constexpr int kWarpsPerCta = 2;    // independent units per CTA

template <int D, int KT>
struct MmaWinLayout {
    static constexpr int STR = 2 * D + 16;  // padded row stride (odd number of 16-byte units)
    static constexpr int NVEC = 2 * D / 16;
    static constexpr int WARP_BYTES = (16 + 2 * KT) * STR;  // Q (16 rows), K tile, V tile
    static constexpr int BYTES = kWarpsPerCta * WARP_BYTES;
};

template <int D, int KT>
__global__ void __launch_bounds__(kWarpsPerCta * 32) window_mma_kernel(VerifyArgs a) {
    using namespace sm100;
    using Lay = MmaWinLayout<D, KT>;
    constexpr int STR = Lay::STR, NVEC = Lay::NVEC;
    constexpr int NKS = D / 16;   // k-steps of Q K^T
    constexpr int NNT = D / 8;    // n-tiles of P V (output channels)
    constexpr int SNT = KT / 8;   // n-tiles of S (keys)
    constexpr int PKS = KT / 16;  // k-steps of P V
    static_assert(KT % 16 == 0 && NKS % 2 == 0 && NNT % 2 == 0, "tile shape");

    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    uint8_t* sQ = smem + warp * Lay::WARP_BYTES;
    uint8_t* sK = sQ + 16 * STR;
    uint8_t* sV = sK + KT * STR;
    const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);

    const StoreView& s = a.s;
    const int H = s.H;
    const int64_t nunits = (int64_t)a.ba.nbranch * a.nrowchunks * H;
    const int64_t u = (int64_t)blockIdx.x * kWarpsPerCta + warp;
    bool active = u < nunits;
    int h = 0, rc = 0, bi = 0;
    Branch br;
    br.ok = false;
    if (active) {
        h = (int)(u % H);
        const int64_t u2 = u / H;
        rc = (int)(u2 % a.nrowchunks);
        bi = (int)(u2 / a.nrowchunks);
        br = load_branch(a.ba, s.R, s.Bmax, bi);
        if (!br.ok && lane == 0 && rc == 0 && h == 0) set_device_error(s.err, RIPE_DEVERR_BRANCH);
        active = br.ok && rc * kRowChunk < br.ntok;
    }

    if (active) {
        const int j0 = rc * kRowChunk;
        const int nr = min(kRowChunk, br.ntok - j0);
        const int b = br.seq, r = br.depth;
        const int T = context_length(s.len, a.ctx, s.err, b, h == 0 && rc == 0 && lane == 0);
        const int A = min(s.ws[b], T);
        const int nwin = T - A;
        const int nk = nwin + j0 + nr;  // block tokens 0..j0+nr-1 are visible to some row here
        const bool ring = r < s.R;
        const int slot0 = A % s.Wcap;
        const char* kbase = ring ? s.kwin + ring_row(s, a.layer, b, h, r, 0) : s.kdeep + deep_row(s, a.layer, b, h, A);
        const char* vbase = ring ? s.vwin + ring_row(s, a.layer, b, h, r, 0) : s.vdeep + deep_row(s, a.layer, b, h, A);
        const int row_lo = lane / 4, row_hi = lane / 4 + 8;  // fragment rows of this lane

        // Q rows of the unit (rows past nr are zero).
        for (int e = lane; e < 16 * NVEC; e += 32) {
            const int rr = e / NVEC, v = e - rr * NVEC;
            uint8_t* dst = sQ + rr * STR + 16 * v;
            if (rr < nr) {
                const int64_t row = br.row0 + (int64_t)(j0 + rr) * br.stride;
                cp_async16(dst, a.Q + (row * H + h) * (2 * D) + 16 * v);
            } else {
                *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
            }
        }

        float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.f, l_hi = 0.f;
        float o[NNT][4];
#pragma unroll
        for (int nt = 0; nt < NNT; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
        uint32_t qa[NKS][4];

        const int ntile = (nk + KT - 1) / KT;
        for (int t = 0; t < ntile; ++t) {
            const int k0 = t * KT, nkt = min(nk - k0, KT);
            // ---- K and V rows of this tile (zero rows past the keys: P V reads them)
            for (int e = lane; e < KT * NVEC; e += 32) {
                const int kk = e / NVEC, v = e - kk * NVEC;
                uint8_t* dk = sK + kk * STR + 16 * v;
                uint8_t* dv = sV + kk * STR + 16 * v;
                if (kk < nkt) {
                    const int key = k0 + kk;
                    const char *kp, *vp;
                    if (key < nwin) {
                        int pos = key;
                        if (ring) {
                            pos = slot0 + key;
                            if (pos >= s.Wcap) pos -= s.Wcap;
                        }
                        kp = kbase + (int64_t)pos * (2 * D);
                        vp = vbase + (int64_t)pos * (2 * D);
                    } else {
                        const int64_t row = br.row0 + (int64_t)(key - nwin) * br.stride;
                        kp = a.Kb + (row * H + h) * (2 * D);
                        vp = a.Vb + (row * H + h) * (2 * D);
                    }
                    cp_async16(dk, kp + 16 * v);
                    cp_async16(dv, vp + 16 * v);
                } else {
                    *reinterpret_cast<uint4*>(dk) = make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4*>(dv) = make_uint4(0, 0, 0, 0);
                }
            }
            cp_async_commit();
            cp_async_wait_all();
            __syncwarp();
            if (t == 0) {
                // Q fragments (A operand), all k-steps, kept in registers.
#pragma unroll
                for (int ks = 0; ks < NKS; ++ks) {
                    const int qr = (lane & 7) + 8 * ((lane >> 3) & 1);
                    const int qc = 16 * ks + 8 * (lane >> 4);
                    ldsm_x4(aQ + qr * STR + 2 * qc, qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3]);
                }
            }
            // ---- S = Q K^T on m16n8k16 tiles
            float sc[SNT][4];
#pragma unroll
            for (int nt = 0; nt < SNT; ++nt) {
                sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
                const int kr = 8 * nt + (lane & 7);
#pragma unroll
                for (int ks = 0; ks < NKS; ks += 2) {
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(aK + kr * STR + 2 * (16 * ks + 8 * (lane >> 3)), b0, b1, b2, b3);
                    mma_16816(sc[nt], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b0, b1);
                    mma_16816(sc[nt], qa[ks + 1][0], qa[ks + 1][1], qa[ks + 1][2], qa[ks + 1][3], b2, b3);
                }
            }
            // ---- masking, scale to log2 units, row max over the quad
            float mx_lo = -INFINITY, mx_hi = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < SNT; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int kk = 8 * nt + 2 * (lane & 3) + (e & 1);
                    const int key = k0 + kk;
                    const int row = e < 2 ? row_lo : row_hi;
                    const bool ok = kk < nkt && row < nr && (key < nwin || key - nwin <= j0 + row);
                    sc[nt][e] = ok ? sc[nt][e] * a.scale_log2 : -INFINITY;
                }
                mx_lo = fmaxf(mx_lo, fmaxf(sc[nt][0], sc[nt][1]));
                mx_hi = fmaxf(mx_hi, fmaxf(sc[nt][2], sc[nt][3]));
            }
            mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 1));
            mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 2));
            mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 1));
            mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 2));
            const float mn_lo = fmaxf(m_lo, mx_lo), mn_hi = fmaxf(m_hi, mx_hi);
            const float al_lo = mn_lo == -INFINITY ? 1.f : ex2(m_lo - mn_lo);
            const float al_hi = mn_hi == -INFINITY ? 1.f : ex2(m_hi - mn_hi);
            float sum_lo = 0.f, sum_hi = 0.f;
#pragma unroll
            for (int nt = 0; nt < SNT; ++nt) {
                sc[nt][0] = mn_lo == -INFINITY ? 0.f : ex2(sc[nt][0] - mn_lo);
                sc[nt][1] = mn_lo == -INFINITY ? 0.f : ex2(sc[nt][1] - mn_lo);
                sc[nt][2] = mn_hi == -INFINITY ? 0.f : ex2(sc[nt][2] - mn_hi);
                sc[nt][3] = mn_hi == -INFINITY ? 0.f : ex2(sc[nt][3] - mn_hi);
                sum_lo += sc[nt][0] + sc[nt][1];
                sum_hi += sc[nt][2] + sc[nt][3];
            }
            sum_lo += __shfl_xor_sync(0xffffffffu, sum_lo, 1);
            sum_lo += __shfl_xor_sync(0xffffffffu, sum_lo, 2);
            sum_hi += __shfl_xor_sync(0xffffffffu, sum_hi, 1);
            sum_hi += __shfl_xor_sync(0xffffffffu, sum_hi, 2);
            l_lo = l_lo * al_lo + sum_lo;
            l_hi = l_hi * al_hi + sum_hi;
            m_lo = mn_lo;
            m_hi = mn_hi;
#pragma unroll
            for (int nt = 0; nt < NNT; ++nt) {
                o[nt][0] *= al_lo; o[nt][1] *= al_lo;
                o[nt][2] *= al_hi; o[nt][3] *= al_hi;
            }
            // ---- O += P V: P from the S fragments, V^T fragments by ldmatrix.trans
#pragma unroll
            for (int ks = 0; ks < PKS; ++ks) {
                const uint32_t p0 = pack_bf16(sc[2 * ks][0], sc[2 * ks][1]);
                const uint32_t p1 = pack_bf16(sc[2 * ks][2], sc[2 * ks][3]);
                const uint32_t p2 = pack_bf16(sc[2 * ks + 1][0], sc[2 * ks + 1][1]);
                const uint32_t p3 = pack_bf16(sc[2 * ks + 1][2], sc[2 * ks + 1][3]);
                const int vr = 16 * ks + (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
                for (int nt = 0; nt < NNT; nt += 2) {
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(aV + vr * STR + 2 * (8 * nt + 8 * (lane >> 4)), b0, b1, b2, b3);
                    mma_16816(o[nt], p0, p1, p2, p3, b0, b1);
                    mma_16816(o[nt + 1], p0, p1, p2, p3, b2, b3);
                }
            }
            __syncwarp();
        }

        // ---- partial of this split (window + block), then count the arrival
        const int seg = a.nsplit;
        const int64_t row_g_lo = br.row0 + (int64_t)(j0 + row_lo) * br.stride;
        const int64_t row_g_hi = br.row0 + (int64_t)(j0 + row_hi) * br.stride;
        const int64_t pi_lo = (row_g_lo * H + h) * a.nseg + seg, pi_hi = (row_g_hi * H + h) * a.nseg + seg;
#pragma unroll
        for (int nt = 0; nt < NNT; ++nt) {
            const int c = 8 * nt + 2 * (lane & 3);
            if (row_lo < nr) *reinterpret_cast<float2*>(a.part_o + pi_lo * D + c) = make_float2(o[nt][0], o[nt][1]);
            if (row_hi < nr) *reinterpret_cast<float2*>(a.part_o + pi_hi * D + c) = make_float2(o[nt][2], o[nt][3]);
        }
        if ((lane & 3) == 0) {
            if (row_lo < nr) a.part_ml[pi_lo] = make_float2(m_lo, l_lo);
            if (row_hi < nr) a.part_ml[pi_hi] = make_float2(m_hi, l_hi);
        }
        __syncwarp();
        const int ndeep = deep_splits_used(A, a.chunk, a.nsplit);
        int last = 0;
        if (lane == 0) {
            int* cnt = a.cnt + ((int64_t)bi * a.nrowchunks + rc) * H + h;
            __threadfence();  // releases the warp's partial (ordered before by __syncwarp)
            last = atomicAdd(cnt, 1) == ndeep;
            if (last) *cnt = 0;
            __threadfence();
        }
        last = __shfl_sync(0xffffffffu, last, 0);
        if (last) {
            // Merge rows row_lo and row_hi for this lane's columns.
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int row = half ? row_hi : row_lo;
                if (row >= nr) continue;
                const int64_t rg = half ? row_g_hi : row_g_lo;
                const int64_t base = (rg * H + h) * a.nseg;
                const float mw = half ? m_hi : m_lo, lw = half ? l_hi : l_lo;
                float M = mw;
                for (int sg = 0; sg < ndeep; ++sg) M = fmaxf(M, __ldcg(a.part_ml + base + sg).x);
                float L = 0.f, acc[NNT][2];
#pragma unroll
                for (int nt = 0; nt < NNT; ++nt) acc[nt][0] = acc[nt][1] = 0.f;
                for (int sg = 0; sg < ndeep; ++sg) {
                    const float2 ml = __ldcg(a.part_ml + base + sg);
                    const float f = ex2(ml.x - M);
                    L = fmaf(ml.y, f, L);
#pragma unroll
                    for (int nt = 0; nt < NNT; ++nt) {
                        const float2 x = __ldcg(reinterpret_cast<const float2*>(a.part_o + (base + sg) * D +
                                                                                8 * nt + 2 * (lane & 3)));
                        acc[nt][0] = fmaf(x.x, f, acc[nt][0]);
                        acc[nt][1] = fmaf(x.y, f, acc[nt][1]);
                    }
                }
                const float fo = ex2(mw - M);
                L = fmaf(lw, fo, L);
                __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.O) + (rg * H + h) * D;
#pragma unroll
                for (int nt = 0; nt < NNT; ++nt) {
                    const float x0 = fmaf(half ? o[nt][2] : o[nt][0], fo, acc[nt][0]);
                    const float x1 = fmaf(half ? o[nt][3] : o[nt][1], fo, acc[nt][1]);
                    *reinterpret_cast<__nv_bfloat162*>(orow + 8 * nt + 2 * (lane & 3)) =
                        __floats2bfloat162_rn(x0 / L, x1 / L);
                }
                if ((lane & 3) == 0 && a.lse) a.lse[rg * H + h] = (M + log2f(L)) * 0.69314718055994531f;
            }
        }
    }

    // Completion: the last CTA of this grid waits for the deep-plane grid it may run
    // beside (programmatic dependent launch), so that this grid ending implies both ended.
    __syncthreads();
    if (threadIdx.x == 0) {
        const int n = atomicAdd(a.done, 1);
        if (n == (int)gridDim.x - 1) {
            *a.done = 0;
            grid_dependency_wait();
        }
    }
    grid_launch_dependents();
}

template <int D, int KT>
cudaError_t launch_mma_t(cudaLaunchConfig_t cfg, const VerifyArgs& a, int64_t units) {
    using Lay = MmaWinLayout<D, KT>;
    static bool set = false;
    if (!set) {
        cudaFuncSetAttribute(window_mma_kernel<D, KT>, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::BYTES);
        cudaFuncSetAttribute(window_mma_kernel<D, KT>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
        set = true;
    }
    const int64_t grid = (units + kWarpsPerCta - 1) / kWarpsPerCta;
    if (grid > 0x7fffffff) return cudaErrorInvalidConfiguration;
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kWarpsPerCta * 32);
    cfg.dynamicSmemBytes = Lay::BYTES;
    return cudaLaunchKernelEx(&cfg, window_mma_kernel<D, KT>, a);
}

template <int D>
cudaError_t launch_mma_d(cudaLaunchConfig_t cfg, const VerifyArgs& a, int64_t units, int keys_ub) {
    if (keys_ub <= 32) return launch_mma_t<D, 32>(cfg, a, units);
    if (keys_ub <= 80) return launch_mma_t<D, 80>(cfg, a, units);
    return launch_mma_t<D, 144>(cfg, a, units);
}

}  // namespace

bool window_supported(int dtype, int d) { return dtype == RIPE_BF16 && (d == 64 || d == 96 || d == 128); }

cudaError_t launch_window(const VerifyArgs& a, int nbranch, int keys_ub, bool pdl, cudaStream_t st) {
    const int64_t units = (int64_t)nbranch * a.nrowchunks * a.s.H;
    if (units == 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    cudaError_t e = cudaErrorInvalidValue;
    switch (a.s.d) {
        case 64: e = launch_mma_d<64>(cfg, a, units, keys_ub); break;
        case 96: e = launch_mma_d<96>(cfg, a, units, keys_ub); break;
        case 128: e = launch_mma_d<128>(cfg, a, units, keys_ub); break;
    }
    ripe_count_launch();
    return e;
}
