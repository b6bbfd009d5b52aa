/*
 * msa.h -- C ABI of libmsa.so, the B200 (sm_100a) training hot path of
 * MiniMax Sparse Attention (MSA).
 *
 * The method (pages: "Flash-MSA: Open-Source Sparse Attention Kernels Debut",
 * section "How MSA works"; the ai-beat news post on Flash-MSA training,
 * paragraphs 1-4): an Index Branch scores every causal (query, key) pair with
 * one small proxy head per GQA group, max-pools the scores over 128-key
 * blocks and picks, per query, the blocks it will read; the picked block ids
 * are cached.  A Main Branch then runs exact softmax attention (GQA) over
 * only those blocks, forward and backward.
 *
 * Conventions for every entry point
 *  - All tensor pointers are DEVICE pointers, row-major, last index fastest,
 *    16-byte aligned, owned by the caller.  bf16 tensors are passed as void*.
 *  - Shapes:  q, o, dout, dq  [B][T][Hq][d]   bf16
 *             k, v, dk, dv    [B][T][Hkv][d]  bf16
 *             qp, kp          [B][T][Hp][dp]  bf16   (Hp == Hkv)
 *             idx             [B][Hp][T][topk] int32, ascending, -1 padded
 *             nsel            [B][Hp][T]       int32
 *             lse             [B][Hq][T]       fp32 (natural-log logsumexp)
 *  - `ws` is a caller-owned device workspace of at least
 *    msa_workspace_size(dims, which) bytes (256-byte aligned).  Its content
 *    on entry is irrelevant; the library keeps no state between calls.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  All work is
 *    enqueued on it; no entry point synchronises or allocates.
 *  - Arguments are validated before anything is enqueued; on an error code
 *    nothing has been launched.  Kernels never trap: a device wait that
 *    gives up or an index outside its range writes a status word inside `ws`,
 *    which msa_check_status() reads.
 *  - Limits: block == 128; Hq % Hkv == 0 with G = Hq/Hkv in {1,2,4,8,16};
 *    d in {64,128}; dp a multiple of 8 in [8,64]; 1 <= topk <= 128;
 *    0 <= T <= 2^20.  B == 0 or T == 0 is a valid empty call.
 *  - Inputs must be finite.
 */
#ifndef MSA_H
#define MSA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MSA_API __attribute__((visibility("default")))
#else
#define MSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct msa_dims {
    int B;      /* batch                                                  */
    int T;      /* sequence length (any value; the last block may be short) */
    int Hq;     /* query heads                                            */
    int Hkv;    /* key/value heads = GQA groups                           */
    int Hp;     /* proxy heads, one per group: must equal Hkv             */
    int d;      /* head dim of the Main Branch                            */
    int dp;     /* head dim of the proxy head                             */
    int block;  /* KV block length: must be 128                           */
    int topk;   /* blocks read per query, own block included              */
    float scale;/* softmax scale of the Main Branch; 0 -> 1/sqrt(d)       */
    int window; /* forced blocks per query (own block included); 0 -> 1  */
    int dilation;/* stride between forced blocks; 0 -> 1                 */
    int q_begin;/* first query row computed: a multiple of 128 in [0, T]; 0 = all */
} msa_dims;

/*
 * q_begin (context-parallel shards).  Queries before q_begin are neither
 * scored, selected nor attended: msa_proxy_select writes idx/nsel (and
 * pooled_dbg) rows q_begin .. T-1 only, msa_fwd writes those rows of o and lse only, msa_bwd
 * writes those rows of dq only, and its dk/dv hold the contributions of those
 * query rows alone -- a partial sum over the keys 0 .. T-1, which the shards
 * of one sequence add up.  Rows before q_begin of q, qp, dout, o and lse are
 * not read.  A rank owning query rows [r0, r1) of a sequence passes T = r1,
 * q_begin = r0, its rows in place and the keys 0 .. r1-1 (the causal prefix
 * its queries can see).  q_begin = T computes no row: no kernel runs and no
 * tensor is read; msa_bwd writes zero dk/dv, msa_proxy_bwd zero dkp, and
 * every entry point still clears the workspace's status words (so it needs
 * the device), which msa_check_status then reports as MSA_OK.  Decode
 * requires q_begin = 0.
 */

enum msa_status {
    MSA_OK = 0,
    MSA_ERR_INVALID_DIMS = -1,  /* a size outside the limits above            */
    MSA_ERR_NULL_PTR = -2,      /* a required pointer is NULL                 */
    MSA_ERR_MISALIGNED = -3,    /* a pointer is not 16-byte aligned (ws: 256) */
    MSA_ERR_WS_TOO_SMALL = -4,  /* ws_bytes < msa_workspace_size()            */
    MSA_ERR_LAUNCH = -5,        /* a CUDA launch or async call failed         */
    MSA_ERR_TIMEOUT = -6,       /* a bounded device wait gave up              */
    MSA_ERR_DEVICE = -7,        /* current device is not sm_100               */
    MSA_ERR_DRIVER = -8,        /* tensor-map encoding unavailable or failed  */
    MSA_ERR_INDEX = -9          /* an idx entry outside its valid range       */
};

enum msa_phase { MSA_SELECT = 0, MSA_FWD = 1, MSA_BWD = 2, MSA_DECODE = 3, MSA_PROXY_BWD = 4 };

/* Bytes of workspace `which` (an msa_phase) needs for these dims.
 * Returns 0 for invalid dims. */
MSA_API size_t msa_workspace_size(const msa_dims* dims, int which);

/*
 * Index Branch ("How MSA works": KVs selected in 128-key blocks by
 * max-pooling proxy scores; one proxy head per group; indices cached).
 *   score(b,g,i,j) = sum_c qp[b,i,g,c] * kp[b,j,g,c]        for j <= i
 *   pooled(b,g,i,n) = max of score over the keys of block n (n <= i/128)
 * Query i keeps its own block i/128 and the topk-1 best earlier blocks by
 * pooled score, equal scores going to the lower block id; with at most topk
 * eligible blocks it keeps them all.
 *   Forced pattern ("Flash-MSA: Train on a million tokens without breaking
 *   the compute bank", section "Under the hood": the block pattern is
 *   configurable by window size and dilation): with window w and dilation s,
 *   the blocks i/128, i/128 - s, ..., i/128 - (w-1)s that exist are always
 *   kept and count toward topk; the remaining slots go to the best of the
 *   other blocks.  w = 1 (the default) forces the own block only.  Requires
 *   w <= topk.  msa_fwd and msa_bwd read any valid idx and ignore both
 *   fields.  idx rows are written ascending and
 * padded with -1; nsel = number of valid entries.  Scores are accumulated in
 * fp32 on the tensor cores and compared in fp32; the T x T score matrix
 * never leaves the chip.
 *   pooled_dbg: optional (NULL = off) [B][Hp][T][nblk] fp32 output of the
 *   pooled scores, -inf past the query's own block; for tests, it costs an
 *   extra write of B*Hp*T*nblk floats.
 */
MSA_API int msa_proxy_select(const msa_dims* dims, const void* qp, const void* kp, int32_t* idx,
                     int32_t* nsel, float* pooled_dbg, void* ws, size_t ws_bytes, void* stream);

/*
 * Main Branch forward (ai-beat post, paragraph 1: exact softmax attention
 * over only the selected blocks; "How MSA works": GQA).  For every query
 * head h of group g = h / (Hq/Hkv) and query i, the keys read are
 * { j : j/128 in idx[b,g,i,:nsel], j <= i };
 *   S_ij = scale * q_i . k_j,  L_i = log sum_j exp(S_ij),
 *   O_i  = sum_j exp(S_ij - L_i) v_j.
 * Writes o (bf16) and lse (fp32).  idx/nsel are the cached output of
 * msa_proxy_select and must be valid (ascending, in range); entries outside
 * [0, i/128] are reported as MSA_ERR_INDEX by msa_check_status.
 */
MSA_API int msa_fwd(const msa_dims* dims, const void* q, const void* k, const void* v, const int32_t* idx,
            const int32_t* nsel, void* o, float* lse, void* ws, size_t ws_bytes, void* stream);

/*
 * Main Branch backward (ai-beat post, paragraph 2: training needs custom
 * backward kernels).  With P_ij = exp(S_ij - L_i) from the cached idx and
 * lse, D_i = dout_i . o_i and dS_ij = P_ij (dout_i . v_j - D_i):
 *   dq_i = scale sum_j dS_ij k_j,
 *   dk_j = scale sum_{i,h in group} dS_ij q_i,  dv_j = sum_{i,h} P_ij dout_i.
 * The block selection is piecewise constant: no gradient is produced for
 * qp/kp.  Writes dq, dk, dv (bf16).
 */
MSA_API int msa_bwd(const msa_dims* dims, const void* q, const void* k, const void* v, const void* o,
            const void* dout, const float* lse, const int32_t* idx, const int32_t* nsel, void* dq,
            void* dk, void* dv, void* ws, size_t ws_bytes, void* stream);

/*
 * msa_fwd without a workspace argument (the pages have no counterpart: this
 * is a library convenience).  For callers that cannot allocate device
 * memory or hand over a workspace -- a plugin or custom-op host that owns all
 * device memory through its own pool and gives an operator only its inputs
 * and outputs, or a latency-critical loop where cudaMalloc/cudaFree (which
 * can synchronise the device) is not allowed.  Same arguments, layouts and
 * results as msa_fwd; the workspace is a fixed 64 MiB array inside the
 * library that every GPU loading this part of the library keeps until the
 * process exits.  The call allocates nothing.
 *  - Problems whose forward workspace (msa_workspace_size(dims, MSA_FWD))
 *    exceeds 64 MiB are rejected with MSA_ERR_WS_TOO_SMALL before any launch.
 *  - The first call on a device looks up the array's device address (once
 *    per device, with that device current); make that first call before any
 *    stream capture.
 *  - All calls on a device share the array and it keeps the last call's
 *    contents (whatever must start at zero is cleared by every call).  Calls
 *    whose work overlaps on the GPU race on it: serialise them.
 *  - Device-side status (timeouts, malformed idx) stays in the shared array;
 *    msa_fwd_noalloc_status reads it.
 */
MSA_API int msa_fwd_noalloc(const msa_dims* dims, const void* q, const void* k, const void* v,
                            const int32_t* idx, const int32_t* nsel, void* o, float* lse, void* stream);

/*
 * msa_check_status for msa_fwd_noalloc: synchronises `stream` and reads the
 * status words that the last msa_fwd_noalloc on the current device left in
 * the library's scratch array (every call clears them first).  Returns
 * MSA_OK, MSA_ERR_TIMEOUT or MSA_ERR_INDEX (with *code as msa_check_status
 * sets it; code may be NULL), MSA_ERR_LAUNCH if the stream or the copy
 * failed, MSA_ERR_DEVICE if the scratch array cannot be found on the current
 * device.  Before any msa_fwd_noalloc on the device it reports MSA_OK.
 */
MSA_API int msa_fwd_noalloc_status(void* stream, uint32_t* code);

/*
 * Decode: attention of one new query token per sequence against caches, with
 * its own block selection (the inference side of the Index and Main
 * Branches: "How MSA works"; the MiniMax inference kernels are not public, so
 * this is our construction from the same two steps).  For sequence b the
 * token sits at position i = lens[b] - 1 (lens NULL: every sequence has
 * length T); its key, value and proxy key must already be in the caches.
 * Computes exactly what msa_proxy_select + msa_fwd compute for the last row
 * of a sequence of length lens[b]: the pooled proxy scores of i against keys
 * 0..i, the selection (own block, forced window, topk - nf best others; same
 * order and ties), then softmax attention of the G heads over the selected
 * keys j <= i.
 *   q   [B][Hq][d] bf16, qp [B][Hp][dp] bf16   (the new token)
 *   k, v [B][T][Hkv][d] bf16, kp [B][T][Hp][dp] bf16   (caches, T = capacity)
 *   lens [B] int32 on the device, 1 <= lens[b] <= T (others: status word set,
 *        the sequence gets nsel 0, O = 0 and lse = -inf)
 *   idx [B][Hp][topk] int32 out (ascending, -1 padded), nsel [B][Hp] out
 *   o [B][Hq][d] bf16 out, lse [B][Hq] fp32 out (natural log)
 *   ws: msa_workspace_size(dims, MSA_DECODE) bytes.
 * Scores are accumulated in fp32 on CUDA cores (the work per token is a few
 * MFLOP; the cache reads set the time).
 */
MSA_API int msa_decode(const msa_dims* dims, const int32_t* lens, const void* q, const void* qp, const void* k,
                       const void* v, const void* kp, int32_t* idx, int32_t* nsel, void* o, float* lse, void* ws,
                       size_t ws_bytes, void* stream);

/*
 * msa_fwd / msa_bwd with flags.  MSA_REUSE_INDEX: the workspace already holds
 * the block -> query inverse index of exactly these idx, nsel and dims, left
 * there by an earlier msa_fwd_ex / msa_bwd_ex on the same workspace (both
 * layouts keep the index at the same offsets, so one workspace of
 * max(msa_workspace_size(MSA_FWD), msa_workspace_size(MSA_BWD)) bytes serves
 * a forward and the backward that follows it); the call skips rebuilding it.
 * Reusing an index built from different idx is undefined.  flags = 0 is
 * msa_fwd / msa_bwd.
 */
enum msa_flags { MSA_REUSE_INDEX = 1, MSA_DKV_F32 = 2, MSA_BLOCK_MASS = 4 };
/* MSA_BLOCK_MASS (msa_fwd_ex): the forward also keeps, in `ws`, the softmax
 * weight each query row puts on each of its selected blocks, for a following
 * msa_proxy_bwd on the same workspace.  `ws` must then hold
 * msa_workspace_size(dims, MSA_PROXY_BWD) bytes; that layout keeps the
 * forward's and the backward's regions at their usual offsets, so one such
 * workspace serves msa_fwd_ex, msa_bwd_ex (MSA_REUSE_INDEX) and
 * msa_proxy_bwd of one step. */
/* MSA_DKV_F32 (msa_bwd_ex): dk and dv are fp32 [B][T][Hkv][d] and receive the
 * unrounded sums, so that partial gradients of several query shards can be
 * added (a reduce-scatter) before one rounding to bf16 (msa_f32_to_bf16). */
MSA_API int msa_fwd_ex(const msa_dims* dims, const void* q, const void* k, const void* v, const int32_t* idx,
                       const int32_t* nsel, void* o, float* lse, void* ws, size_t ws_bytes, void* stream, int flags);
MSA_API int msa_bwd_ex(const msa_dims* dims, const void* q, const void* k, const void* v, const void* o,
                       const void* dout, const float* lse, const int32_t* idx, const int32_t* nsel, void* dq,
                       void* dk, void* dv, void* ws, size_t ws_bytes, void* stream, int flags);

/*
 * Proxy-head gradient (the ai-beat post on Flash-MSA training, paragraph 2:
 * gradients through the gating mechanism; paragraph 4: the proxy heads are
 * trained).  The pages do not define the training signal; this entry point
 * computes one reading of it, the KL divergence that distils the Main
 * Branch's attention into the Index Branch (as DeepSeek's indexer is trained,
 * which "How MSA works" likens MSA to).  Per query row (b, g, i) over its
 * selected blocks S (idx, nsel):
 *   p(n) = (1/G) sum over the group's heads of the softmax weight the
 *          forward put on the keys of block n (held constant),
 *   z(n) = the pooled proxy score of block n (max over its keys j <= i),
 *   q    = softmax over S of z,   loss[b][g][i] = KL(p || q),
 * and with dz(n) = q(n) sum_m p(m) - p(n) and j*(n) the argmax key of block
 * n (the lowest key on ties), dqp_i = sum_n dz(n) kp_j*(n),
 * dkp_j = sum over (i, n) with j*(n) = j of dz(n) qp_i.
 *   dqp [B][T][Hp][dp] fp32 (rows q_begin .. T-1 written), dkp
 *   [B][T][Hp][dp] fp32 (every row written), loss [B][Hp][T] fp32 (rows
 *   q_begin .. T-1).
 * `ws` (msa_workspace_size(dims, MSA_PROXY_BWD) bytes) must hold what an
 * earlier msa_fwd_ex with MSA_BLOCK_MASS left there for exactly these dims,
 * idx and nsel; a msa_bwd_ex on the same workspace in between is allowed.
 * A row whose forward weights overflowed (only rows the exact fallback redid,
 * msa_fallback_rows, can) gets loss 0 and no gradient.
 */
MSA_API int msa_proxy_bwd(const msa_dims* dims, const void* qp, const void* kp, const int32_t* idx,
                          const int32_t* nsel, float* dqp, float* dkp, float* loss, void* ws, size_t ws_bytes,
                          void* stream);

/* dst[i] = bf16(src[i]) (round to nearest even) for i < n: fp32 -> bf16 on
 * the device.  n must be a multiple of 8; both pointers device, 16-byte
 * aligned.  Used to round partial gradients once they have been summed. */
MSA_API int msa_f32_to_bf16(const float* src, void* dst, int64_t n, void* stream);

/* Synchronises `stream`, then reads the status word a previous call left in
 * `ws`: MSA_OK, MSA_ERR_TIMEOUT or MSA_ERR_INDEX.  `code` (nullable)
 * receives the raw device code (which wait or check failed). */
MSA_API int msa_check_status(const void* ws, void* stream, uint32_t* code);

/* Synchronises `stream`, then reads how many query rows the last msa_fwd /
 * msa_fwd_ex on this workspace recomputed with its exact two-pass softmax
 * (rows whose fixed softmax shift left their weights outside the fp32 range
 * the forward accepts: only a row whose best score lies more than about
 * 140 nats above the score of the query's own key).
 * Any later call on the same workspace resets the count. */
MSA_API int msa_fallback_rows(const void* ws, void* stream, int64_t* rows);

/* Human-readable text for a status code (static storage). */
MSA_API const char* msa_strerror(int status);

/* ---- tracing (no counterpart on the pages) -------------------------------- */

enum msa_kernel { MSA_KERNEL_PROXY = 0, MSA_KERNEL_FWD_MAIN = 1, MSA_KERNEL_BWD_MAIN = 2 };

/* From now on, calls made by this host thread record the CUDA event `start`
 * (a cudaEvent_t) on the call's stream just before launching the named
 * kernel, and `stop` just after it, so a caller can time that kernel alone.
 * NULL stops recording.  The events stay owned by the caller. */
MSA_API int msa_set_kernel_events(int kernel, void* start, void* stop);

/* Number of kernels this library has enqueued in this process since it was
 * loaded (every launch of every entry point, counted on the host as it is
 * made; thread-safe).  Callers take the difference around a region. */
MSA_API uint64_t msa_kernel_launches(void);

/* ---- diagnostics (no counterpart on the pages; used by the GPU tests) ---- */

/* One 128 x N x K tcgen05 MMA, D[m][n] = sum_k A[m][k] * B[n][k], with the
 * operands staged the way the kernels stage them.  A: [128][K] bf16, B:
 * [N][K] bf16, D: [128][N] fp32, all device pointers.  mode: 0 = A,B K-major
 * in shared memory; 1 = A K-major, B MN-major; 2 = A,B MN-major; 3 = A in
 * tensor memory, B MN-major; 4 = A in tensor memory, B K-major.
 * N in {64,128}, K in {64,128};
 * `ws` needs 256 bytes.  Synchronous. */
MSA_API int msa_diag_umma(int mode, int N, int K, const void* A, const void* B, float* D, void* ws,
                  void* stream);

/* Launches a kernel whose mbarrier wait can never complete, bounded by
 * limit_ns; returns what msa_check_status reports (MSA_ERR_TIMEOUT when the
 * bound works).  `ws` needs 256 bytes.  Synchronous. */
MSA_API int msa_diag_wait_timeout(uint64_t limit_ns, void* ws, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MSA_H */
