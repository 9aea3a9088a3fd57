/*
 * ripe.h -- C ABI of libripe: RIPE verify-attention over a depth-planed KV cache
 * on NVIDIA B200 (sm_100a).
 *
 * The operation.  A looped (recurrent-depth) language model runs one block of
 * layers R times per token, so each recurrent layer has R key/value planes per
 * position, one per loop; self-speculative decoding drafts with a few loops and
 * verifies with all R, reading all planes (RIPE abstract, zhuanzhiai.com
 * mirror, first sentence).  RIPE stores the deepest plane R for every position
 * and all R planes only for a window of the W most recent positions (same
 * abstract, sentence introducing RIPE).  A verify query at loop depth r reads
 * plane r inside the window and plane R outside it, plus the draft-block tokens
 * of its own branch at plane r, causally.  Branches at different recurrent
 * depths (LoopSpec's main, early-draft and fallback branches) are verified in
 * one batched call (LoopSpec article, rit.work, section on the early draft).
 *
 * Conventions shared by every entry point:
 *   - Every function returns a ripe_status; RIPE_OK is 0.  Argument errors are
 *     detected on the host and returned before anything is enqueued;
 *     ripe_last_error() then holds a one-line message for the calling thread.
 *   - Device work is asynchronous on the given stream (a cudaStream_t passed as
 *     void*; NULL is the legacy default stream).  Conditions only the device
 *     can see (a sequence id out of range, an append past capacity, a context
 *     length above the committed length) skip the offending item and set the
 *     cache's device error word instead of trapping; read it with
 *     ripe_get_device_error().
 *   - Every call that takes a cache must be made with the cache's device current
 *     (the device that was current at ripe_cache_create); RIPE_ERR_INVALID_ARG
 *     otherwise.  ripe_cache_destroy may be called from any device.
 *   - Pointers named *_dev are device pointers; *_host are host pointers.  The
 *     caller owns every buffer it passes; the library keeps no reference to
 *     them after the call's device work has run.
 *   - bf16 is IEEE-style bfloat16 (1-8-7); f32 is IEEE binary32.
 *   - Device data pointers must be 16-byte aligned, and d * sizeof(element)
 *     must be a multiple of 16 (RIPE_ERR_UNALIGNED otherwise).
 */
#ifndef RIPE_H_
#define RIPE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct ripe_cache_s* ripe_cache_t;
typedef void* ripe_stream_t; /* a cudaStream_t */

typedef enum {
    RIPE_OK = 0,
    RIPE_ERR_INVALID_ARG = 1, /* a size, id or pointer is out of its documented range */
    RIPE_ERR_CAPACITY = 2,    /* a host-known size exceeds the cache's capacity */
    RIPE_ERR_UNALIGNED = 3,   /* a device pointer or row is not 16-byte aligned */
    RIPE_ERR_OOM = 4,         /* device allocation failed */
    RIPE_ERR_CUDA = 5,        /* a CUDA runtime call failed */
    RIPE_ERR_DEVICE = 6,      /* the device error word was set (see ripe_get_device_error) */
    RIPE_ERR_UNSUPPORTED = 7, /* shape or dtype the library has no kernel for */
    RIPE_ERR_CAPTURING = 8    /* the call would allocate while the stream is being captured */
} ripe_status;

typedef enum { RIPE_BF16 = 0, RIPE_F32 = 1 } ripe_dtype;

/* Device error word values (first error wins until cleared). */
enum {
    RIPE_DEVERR_NONE = 0,
    RIPE_DEVERR_SEQ_RANGE = 1,   /* a sequence id outside [0, max_seqs) */
    RIPE_DEVERR_CAPACITY = 2,    /* append would pass Tmax; that sequence was skipped */
    RIPE_DEVERR_COUNT = 3,       /* an accepted count outside [0, kmax_in] */
    RIPE_DEVERR_CTX = 4,         /* ctx_len above the committed length; clamped to it */
    RIPE_DEVERR_BRANCH = 5,      /* a branch with depth outside [1,R], rows out of range, more tokens
                                    than the cache's kmax, or a sequence's branches not adjacent */
    RIPE_DEVERR_TIMEOUT = 6,     /* a kernel's bounded wait expired; its outputs are incomplete */
    RIPE_DEVERR_FORK = 7         /* a fork pair with an id out of range, parent == child, or a parent
                                    that is itself a fork; that pair was skipped */
};

/*
 * One verify branch: ntok draft tokens of sequence `seq` at loop depth `depth`
 * (1..R; R = deepest).  Token j's query, block key and block value are row
 * row0 + j*row_stride of Q / Kblk / Vblk, and its output goes to the same row
 * of O.  Token j attends to the sequence's committed positions (RIPE read rule)
 * and to tokens 0..j of the same branch.  Branches of one sequence must be
 * adjacent in the list (the deepest plane is then read once for all of them).
 */
typedef struct {
    int32_t seq;
    int32_t depth;
    int32_t ntok;
    int32_t row0;
    int32_t row_stride;
    int32_t reserved[3]; /* must be 0 */
} ripe_branch_t;

/*
 * Store layout (all in one device allocation, each part 256-byte aligned):
 *   Kdeep, Vdeep  [layers][max_seqs][H][Tmax][d]       plane R of every position
 *   Kwin,  Vwin   [layers][max_seqs][H][R-1][Wcap][d]  planes 1..R-1, ring buffer:
 *                 position p lives in slot p mod Wcap, Wcap = W + kmax
 *   len[max_seqs], ws[max_seqs] (int32)                committed length T_b and
 *                 window start ws_b; positions ws_b <= p < T_b are live in the ring
 *   rfloor[max_seqs] (int32)                           ring floor: the lowest position
 *                 whose ring slots still hold its own planes (rfloor_b <= ws_b);
 *                 append raises it like ws, evict does not
 *   fbase[max_seqs], fpos[max_seqs] (int32)            forks: sequence b reads its deep
 *                 positions below fpos_b from sequence fbase_b (b and 0 when b is not
 *                 a fork)
 * Memory per layer, sequence and head grows as T + W*(R-1) planes instead of R*T
 * (RIPE abstract, sentence on the 64-position window and 11.9% of the full
 * cache's memory).
 */

/* Bytes ripe_cache_create needs for these sizes (store + metadata). */
int ripe_cache_bytes(int layers, int R, int H, int d, int W, int Tmax, int max_seqs, int kmax,
                     int dtype, size_t* bytes);

/*
 * Create a cache on the current CUDA device.  layers >= 1; 1 <= R <= 64;
 * 1 <= H <= 256; d in [8, 128] with d*sizeof(element) a multiple of 16;
 * W >= 0; Tmax >= 1; 1 <= max_seqs <= 1024; kmax >= 1 (largest append per call,
 * and largest draft block).  dev_mem: NULL to let the library cudaMalloc the
 * store (freed by ripe_cache_destroy), else a caller-owned device buffer of at
 * least ripe_cache_bytes bytes, 256-byte aligned, that outlives the cache.  All
 * lengths start at 0.  Returns RIPE_ERR_OOM if the allocation fails.
 */
int ripe_cache_create(int layers, int R, int H, int d, int W, int Tmax, int max_seqs, int kmax,
                      int dtype, void* dev_mem, ripe_cache_t* out);

/* Free the cache (and its store if the library allocated it).  Synchronises the device. */
int ripe_cache_destroy(ripe_cache_t cache);

/* Set len = ws = rfloor = 0 for the listed sequences (device ids, nseq of them); a
 * fork among them is released (it no longer reads its parent). */
int ripe_cache_reset(ripe_cache_t cache, const int32_t* seq_ids_dev, int nseq,
                     ripe_stream_t stream);

/*
 * Commit accepted draft tokens with all their planes (RIPE abstract: new
 * positions enter the window at full depth).  For listed sequence i (id
 * seq_ids_dev[i]) with n = n_acc_dev[i] accepted tokens, 0 <= n <= kmax_in:
 * positions T..T+n-1 (T = len before the call) receive plane R in Kdeep/Vdeep
 * and planes 1..R-1 in the ring (only the last min(n, Wcap) positions, the
 * earlier ones would be overwritten), then len += n and, if more than Wcap
 * positions would be live, ws = len - Wcap.
 *   K, V: device, [layers][nseq][kmax_in][R][H][d] in the cache dtype; plane
 *         index r-1 on the fourth axis (index R-1 is the deepest plane).
 *   kmax_in >= 1 (a prefill may exceed the cache's kmax: only the last Wcap
 *   positions then keep planes 1..R-1).  Sequence ids in one call must be distinct.
 * A sequence whose append would pass Tmax is skipped (RIPE_DEVERR_CAPACITY).
 * The library keeps a host-side bound on the lengths (it plans verify launches
 * from it); an append enqueued while the stream is captured into a CUDA graph
 * may replay any number of times, so it raises that bound to Tmax.
 */
int ripe_append(ripe_cache_t cache, const int32_t* seq_ids_dev, const int32_t* n_acc_dev, int nseq,
                const void* K, const void* V, int kmax_in, ripe_stream_t stream);

/*
 * Positions leaving the window collapse to the deepest plane (RIPE abstract,
 * sentence introducing RIPE): ws = max(ws, len - W) for each listed sequence.
 * No data moves: plane R of every position is already in Kdeep/Vdeep, and the
 * ring slots below ws become free.
 */
int ripe_evict(ripe_cache_t cache, const int32_t* seq_ids_dev, int nseq, ripe_stream_t stream);

/*
 * Branch forks (LoopSpec article, deployment section: the server keeps a KV cache
 * per branch and deletes rejected continuations).  For each i, sequence
 * child_ids_dev[i] becomes a fork of parent_ids_dev[i] at the parent's current
 * length T: it reads the parent's deep plane below its fork position
 * f = floor(T / 64) * 64 (no copy), owns copies of the parent's deep rows f..T-1
 * and of the parent's whole ring (Wcap = W + kmax positions x (R-1) planes per
 * layer and head), and takes the parent's len, ws and rfloor.  Appends, evicts
 * and verifies of the child then act on the child alone; a verify reads the
 * parent's prefix and then the child's own positions.  ripe_cache_reset releases
 * a fork.  While a fork lives its parent must keep its deep rows below f (no
 * truncate below f) and must not be reset; a fork cannot be truncated below f
 * (RIPE_DEVERR_COUNT, skipped).  A pair whose parent is itself a fork, whose ids
 * are out of range or equal, is skipped and sets RIPE_DEVERR_FORK.  Child ids of
 * one call must be distinct and must not be parents in the same call.
 */
int ripe_fork(ripe_cache_t cache, const int32_t* parent_ids_dev, const int32_t* child_ids_dev, int nseq,
              ripe_stream_t stream);

/*
 * Roll the listed sequences back to a confirmed prefix (LoopSpec article,
 * section on the second branch: a rejected early draft discards the dependent
 * branch's work and decoding returns to the confirmed prefix).  With
 * T' = new_len_dev[i] >= 0 (device int32; a negative value skips the sequence
 * and sets RIPE_DEVERR_COUNT):
 *   len = min(len, T'),  rfloor = min(rfloor, len),  ws = min(ws, max(len - W, rfloor)).
 * That is the state an evict at the confirmed length leaves: positions pushed out
 * of the window only by the rejected tokens come back (their ring slots still
 * hold every plane), as long as at most kmax positions are rolled back
 * (Wcap = W + kmax).  Positions whose ring slots the rejected tokens overwrote
 * stay at the deepest plane.  T' >= len changes nothing.
 */
int ripe_truncate(ripe_cache_t cache, const int32_t* seq_ids_dev, const int32_t* new_len_dev,
                  int nseq, ripe_stream_t stream);

/*
 * Batched verify-attention for one layer over a branch list.
 *   branches_dev: device array of nbranch ripe_branch_t (see above).
 *   Q, Kblk, Vblk: device, [nrows][H][d]; Q in the cache dtype, Kblk/Vblk are the
 *         draft tokens' keys/values at their branch's depth, in the cache dtype.
 *   ctx_len_dev: NULL to attend to each sequence's committed length len, else a
 *         device int32 array indexed by sequence id giving T_b <= len (larger
 *         values are clamped and flag RIPE_DEVERR_CTX).
 *   scale: softmax scale; 0 means 1/sqrt(d).
 *   O: device, [nrows][H][d] in the cache dtype; rows not covered by a branch
 *         are left untouched.
 *   lse: device float [nrows][H] (natural-log sum of exp of the scaled scores),
 *         or NULL.
 * For branch (b, depth r) token j and head h the keys are: positions
 * p in [0, min(ws_b, T_b)) at plane R; positions p in [min(ws_b,T_b), T_b) at
 * plane r; block tokens 0..j of the branch at plane r.  s = scale*<q,k>,
 * O = softmax(s) V, accumulated in fp32.
 * Work space: the cache holds a scratch buffer for per-split partial results;
 * a call that needs more than it holds grows it (a cudaMalloc), which returns
 * RIPE_ERR_CAPTURING if the stream is being captured -- call
 * ripe_reserve_workspace first in that case.
 * CUDA graphs: a call enqueued while the stream is being captured is planned
 * for every length the cache can hold (its deep-region splits cover Tmax), so
 * the captured launch stays exact when replayed after the sequences have grown.
 */
int ripe_verify_attn(ripe_cache_t cache, int layer, const ripe_branch_t* branches_dev, int nbranch,
                     int nrows, const void* Q, const void* Kblk, const void* Vblk,
                     const int32_t* ctx_len_dev, float scale, void* O, float* lse,
                     ripe_stream_t stream);

/*
 * All k draft tokens verified at all R depths in one launch (RIPE abstract:
 * draft with a few loops, verify with all R).  Equivalent to ripe_verify_attn
 * with the R*nseq branches (s, r): seq = seq_ids_dev[s], depth r, ntok k,
 * row0 = s*k*R + r-1, row_stride R.
 *   Q, Kblk, Vblk, O: device, [nseq][k][R][H][d]; lse: [nseq][k][R][H] or NULL.
 */
int ripe_verify_attn_all_depths(ripe_cache_t cache, int layer, const int32_t* seq_ids_dev, int nseq,
                                int k, const void* Q, const void* Kblk, const void* Vblk,
                                const int32_t* ctx_len_dev, float scale, void* O, float* lse,
                                ripe_stream_t stream);

/*
 * ripe_verify_attn_all_depths under the per-query sliding-window reading (the
 * RIPE abstract's fifth sentence read per query): draft token j, at position
 * T + j, reads the W most recent positions T+j-W+1 .. T+j at its own depth r --
 * a committed one only while the store still holds its planes (p >= ws) -- and
 * every older position at the deepest plane R; an older draft token j' < j-W+1 is
 * read at plane R, which is its depth-R row in the same call.  With W >= k no
 * draft token is read at plane R (batched verification is then block-independent).
 * Same arguments and layouts as ripe_verify_attn_all_depths.  Served by the
 * persistent sm_100a kernel only (bf16, d in {64, 96, 128}, k*R <= 256);
 * RIPE_ERR_UNSUPPORTED otherwise.
 */
int ripe_verify_attn_all_depths_sliding(ripe_cache_t cache, int layer, const int32_t* seq_ids_dev, int nseq,
                                        int k, const void* Q, const void* Kblk, const void* Vblk,
                                        const int32_t* ctx_len_dev, float scale, void* O, float* lse,
                                        ripe_stream_t stream);

/*
 * ripe_verify_attn for callers that cannot allocate device memory.  The pages
 * have no counterpart: this is a deployment variant, not part of the method.
 *
 * Some callers cannot call cudaMalloc: a serving stack that has reserved nearly
 * all of HBM for its own pools and forbids other allocations, code that enqueues
 * work while a stream is being captured into a CUDA graph, or a latency-bound
 * path that cannot afford cudaMalloc's implicit device synchronisation.  This
 * entry point takes the same arguments and computes the same result as
 * ripe_verify_attn, but never allocates: its per-split partial results go to a
 * fixed device array of RIPE_NOALLOC_SCRATCH_BYTES owned by the library, which
 * every GPU that loads the library's device code holds until the process exits.
 *   - The cache's device must be current (RIPE_ERR_INVALID_ARG otherwise), as for
 *     every entry point that takes a cache.
 *   - The first call on each device looks up that array's device address
 *     (cudaGetSymbolAddress, with the device current); make that first call
 *     before any stream capture on the device.
 *   - A call whose partial results would not fit even with the deep region in
 *     one split returns RIPE_ERR_CAPACITY (ripe_last_error gives the bytes
 *     needed); *scratch_needed (if not NULL) receives the bytes the call uses or
 *     would need.
 *   - All calls share the one array and it keeps the last call's contents.
 *     Nothing in it has to start at zero: each call writes every partial it
 *     later reads.  Calls that may overlap on the GPU (different streams without
 *     ordering between them) race on the array: serialise them.
 */
#define RIPE_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
int ripe_verify_attn_noalloc(ripe_cache_t cache, int layer, const ripe_branch_t* branches_dev, int nbranch,
                             int nrows, const void* Q, const void* Kblk, const void* Vblk,
                             const int32_t* ctx_len_dev, float scale, void* O, float* lse,
                             ripe_stream_t stream, size_t* scratch_needed);

/* Pre-size the verify scratch for any call of up to max_rows rows enqueued under
 * stream capture (the largest split count such a call can get), before capture. */
int ripe_reserve_workspace(ripe_cache_t cache, int max_rows);

/*
 * Synthetic store fill for benchmarks and tests: writes the same store state as
 * one ripe_append of T_host[i] positions to each listed sequence, with values
 * from the counter-based generator documented in depth_planed_kv_b200/synth.py
 * (SplitMix64 words, four 16-bit fields summed, centred and scaled to unit
 * variance; plane r < R = deepest + coef[r-1] * noise, rounded to the cache dtype).
 *   seq_ids_host, T_host: host arrays of nseq entries (T <= Tmax).
 *   coef_host: host float[R] (coef[r-1] = decay^(R-r)).
 */
int ripe_synth_fill(ripe_cache_t cache, const int32_t* seq_ids_host, const int32_t* T_host, int nseq,
                    uint64_t seed, const float* coef_host, ripe_stream_t stream);

/*
 * Which kernels serve ripe_verify_attn* for this cache:
 *   RIPE_PATH_FUSED_SM100 (1): the fused sm_100a kernel (tcgen05/TMEM deep plane,
 *     TMA-fed, in-cluster merge) -- bf16 with d in {64, 96, 128};
 *   RIPE_PATH_CUDA_CORE (0): the CUDA-core split and merge kernels (fp32, other head
 *     sizes, or a store too large for the tensor maps -- ripe_cache_create then
 *     leaves a note in ripe_last_error).
 */
enum { RIPE_PATH_CUDA_CORE = 0, RIPE_PATH_FUSED_SM100 = 1 };
int ripe_cache_verify_path(ripe_cache_t cache, int* path);

/*
 * Which sm_100a kernel serves ripe_verify_attn_all_depths on this cache (a
 * scheduling choice; both compute the same rows, and the pages have no
 * counterpart):
 *   RIPE_ALL_DEPTHS_AUTO (0, the default): the persistent kernel where the deep
 *     region outweighs the windows (deep length >= R * (Wcap + k)) over at least
 *     as many (sequence, head) pairs as the GPU has SMs, or where the windows
 *     outweigh the deep region (R * Wcap >= deep length) and each window with the
 *     k draft tokens fits one stage of the kernel's ring (Wcap + k <= 80, or 48
 *     for d = 128 with k*R > 128), else the cluster kernel;
 *   RIPE_ALL_DEPTHS_PERSISTENT (1): the persistent kernel whenever it can serve
 *     the call (k*R <= 256);
 *   RIPE_ALL_DEPTHS_CLUSTER (2): the cluster kernel.
 * The sliding form always runs in the persistent kernel.  RIPE_ERR_INVALID_ARG
 * for another value; the setting takes effect from the next call.
 */
enum { RIPE_ALL_DEPTHS_AUTO = 0, RIPE_ALL_DEPTHS_PERSISTENT = 1, RIPE_ALL_DEPTHS_CLUSTER = 2 };
int ripe_cache_set_all_depths_kernel(ripe_cache_t cache, int kernel);

/*
 * The acceptance step of self-speculative decoding, in LoopSpec's order (LoopSpec
 * article, sections on the second branch and on the final check): for each draft
 * position, first the early draft x1 is tested against the final distribution,
 * then the fallback x2 prepared from a deeper state, and only after both are
 * rejected the pipeline restarts from what the final distribution still has to
 * give.  Sampling keeps the final distribution; greedy decoding (temperature 0)
 * keeps the final argmax.
 *   zp, zq, zf: device float [nseq][k][V] logits of the final loop, of the draft's
 *       loop and of the deeper loop the fallback came from (zf NULL: no fallback).
 *   x1, x2: device int32 [nseq][k] the draft and fallback tokens (x2 may be NULL
 *       only without zf).
 *   u: device float [nseq][k][3] uniforms in [0, 1): accept x1, accept x2, restart.
 *   temperature >= 0 (0: greedy).
 * With p, q1, qf the softmaxes at the temperature: x1 is accepted if
 * u0 * q1(x1) < p(x1); the fallback exists if qf(x1) < q1(x1) at temperature 1 and
 * q2 = norm((qf - q1)+) has mass; x2 is accepted if u1 * q2(x2) < p1(x2) with
 * p1 = norm((p - q1)+); else the restart token is the smallest v whose running sum
 * of norm((p1 - q2)+) (p1 without a fallback) exceeds u2 times its total.  A
 * remainder without mass is replaced by the distribution it came from.  Positions
 * are checked in order and the first rejected x1 ends the block.
 * Outputs (device int32 [nseq]): n_accepted (drafts accepted, 0..k), token (the
 * fallback or restart token emitted at position n_accepted, -1 when all k were
 * accepted) and path (0 all accepted, 1 fallback accepted, 2 restart).
 * fp32 arithmetic; one CTA per sequence.
 */
int ripe_accept(int nseq, int k, int V, const float* zp, const float* zq, const float* zf, const int32_t* x1,
                const int32_t* x2, const float* u, float temperature, int32_t* n_accepted, int32_t* token,
                int32_t* path, ripe_stream_t stream);

/*
 * Test hook for the bounded-wait error path (the pages have no counterpart).  The
 * next all-depths verify on this cache that runs in the persistent sm_100a kernel
 * makes its softmax warps first wait, at most `cycles` SM clock cycles (0 <= cycles
 * <= 2^31; 0 turns the hook off), on a barrier that nothing signals.  The wait runs
 * out, the kernel records RIPE_DEVERR_TIMEOUT, lets its copies and tensor-core
 * operations in flight finish, and returns with that call's outputs incomplete;
 * ripe_get_device_error then reports it, and later calls are exact again.  No
 * fault, trap or unbounded wait is involved.
 */
int ripe_debug_stall_next_verify(ripe_cache_t cache, long long cycles);

/* Device pointers of the store parts (tests compare them byte for byte); any
 * output may be NULL. */
int ripe_cache_buffers(ripe_cache_t cache, void** kdeep, void** vdeep, void** kwin, void** vwin,
                       int32_t** len, int32_t** ws, int32_t** rfloor);

/* Copy fbase and fpos (fork metadata, see ripe_fork) of all max_seqs sequences to
 * host arrays (each may be NULL; synchronises stream). */
int ripe_read_forks(ripe_cache_t cache, int32_t* fbase_host, int32_t* fpos_host, ripe_stream_t stream);

/* Copy len, ws and rfloor of all max_seqs sequences to host arrays (each may be
 * NULL; synchronises stream). */
int ripe_read_meta(ripe_cache_t cache, int32_t* len_host, int32_t* ws_host, int32_t* rfloor_host,
                   ripe_stream_t stream);

/* Read and clear the device error word (synchronises stream). */
int ripe_get_device_error(ripe_cache_t cache, int32_t* code_host, ripe_stream_t stream);

/* Number of kernel launches the library has issued since load (all caches). */
uint64_t ripe_launch_count(void);

/* Static description of a status code, and the calling thread's last message. */
const char* ripe_error_string(int status);
const char* ripe_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* RIPE_H_ */
