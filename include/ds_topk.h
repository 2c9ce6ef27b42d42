/*
 * ds_topk.h -- C ABI of libdstopk.so, the selection step of DeepSeek-style
 * sparse attention on B200 (sm_100a).
 *
 * Five operations, as described on the pages this library follows:
 *
 *  - Row-wise top-k of given scores (DeepSelect hub page, use-case paragraphs:
 *    pick the top-k positions of every score row; bfloat16 rows for the
 *    lightning indexer, float32 rows over a ~129K vocabulary for sampling;
 *    options sorted_index and return_value).
 *
 *  - The lightning-indexer score followed by top-k (NKI pull request "Add
 *    DeepSeek-V4 CSA attention kernels", "How the algorithm works", steps
 *    table rows 2 and 3): for every query row t and key position s,
 *        score[t,s] = sum_h w[t,h] * max(0, q[t,h,:] . k[s,:])
 *    over a 128-channel bfloat16 key cache shared by all rows, then the k
 *    highest-scoring positions of each row.
 *
 *  - The compressor's 4:1 fold of new rows into the compressed caches (steps
 *    table row 1; the gate is a stated reading, the pages give none).
 *
 *  - The indexer query projection that produces the scorer's queries and
 *    per-head weights (the same pull request, steps table row 2).
 *
 *  - The attention that consumes the selection (the same pull request, steps
 *    table row 4): multi-query softmax attention of every query head over
 *    the selected compressed KV rows plus a sliding window of recent rows.
 *
 * Conventions shared by every entry point
 *  - All tensor arguments are DEVICE pointers to caller-owned memory, row-major
 *    and contiguous.  Nothing is copied to or from the host.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream).  Every call only enqueues work on that stream and returns; no
 *    call synchronises the host, except ds_get_device_status.
 *  - The return value is DS_OK (0) or a negative DS_ERR_* code.  Argument
 *    errors are detected on the host before anything is enqueued.  Errors
 *    found on the device (a bounded wait that ran out) are recorded in a
 *    per-device status word that ds_get_device_status reads and clears.
 *    libdstopk_debug.so, the same library built with DS_DEBUG, also records
 *    inputs read on the device outside their documented range there.
 *  - Index outputs are int32.  Ties between equal scores go to the lower
 *    position; -0.0 equals +0.0; every NaN ranks above +inf and all NaNs are
 *    equal.  Positions s >= valid_len[row] are never selected.  When a row
 *    has fewer than k eligible positions, the missing slots hold index -1 and
 *    value / score -inf.
 *  - The library owns only scratch memory: ds_indexer_topk (score rows and
 *    per-row key histograms) and ds_sparse_attention each allocate
 *    per-device, grow-only buffers with cudaMalloc on first use and on calls
 *    larger than any before (so make those calls outside CUDA-graph
 *    capture); ds_release frees them.
 *  - Calls on different streams may run concurrently, except that calls of
 *    ds_indexer_topk on one device share the scratch buffer and must be
 *    ordered on one stream.
 */
#ifndef DS_TOPK_H
#define DS_TOPK_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* element types of score rows */
typedef enum { DS_F32 = 0, DS_BF16 = 1 } ds_dtype;

/* status codes */
#define DS_OK 0
#define DS_ERR_ARG (-1)         /* bad argument: null pointer, size, dtype, k, alignment */
#define DS_ERR_CUDA (-2)        /* a CUDA runtime call or kernel launch failed */
#define DS_ERR_TIMEOUT (-3)     /* a bounded wait inside a kernel ran out (device status) */
#define DS_ERR_UNSUPPORTED (-4) /* the current device is not an sm_100 GPU */
#define DS_ERR_NOMEM (-5)       /* the scratch buffer could not be allocated */
#define DS_ERR_RANGE (-6)       /* DS_DEBUG builds: an input read on the device was out of
                                   range (device status) */

/* limits */
#define DS_MAX_K 2048            /* largest k of either operation */
#define DS_INDEXER_DIM 128       /* indexer channels d (fixed) */
#define DS_INDEXER_MAX_HEADS 64  /* largest number of indexer heads */
#define DS_ATTN_MAX_DIM 512      /* largest head_dim of ds_sparse_attention */
#define DS_ATTN_MAX_WINDOW 4096  /* largest sliding window of ds_sparse_attention */
#define DS_ATTN_MAX_HEADS 4096   /* largest number of query heads of ds_sparse_attention */

/*
 * ds_topk -- top-k of every row of a [batch, n] score matrix.
 *   (DeepSelect hub page: the top-k operator of the lightning indexer and of
 *    sampling; options sorted_index and return_value.)
 *
 * scores       device, [batch, n] of `dtype` (float32 or bfloat16), read only.
 * batch, n     rows and row length; batch >= 1, 1 <= n <= 16777216.
 * k            1 <= k <= DS_MAX_K.  k may exceed n (extra slots are padding).
 * dtype        DS_F32 or DS_BF16.
 * valid_len    device int32 [batch] or NULL.  Row t considers positions
 *              0 .. min(max(valid_len[t], 0), n) - 1 only.  NULL means n.
 * out_idx      device int32 [batch, k]: the selected positions.  Without
 *              sorted_index their order is unspecified; with it they are in
 *              ascending position order.  Slots past the number of eligible
 *              positions hold -1.
 * out_val      device [batch, k] of `dtype`: the stored bit pattern of each
 *              selected score, -inf in padding slots.  Written only when
 *              return_value != 0; may be NULL otherwise.
 * return_value 0 or 1.
 * sorted_index 0 or 1.
 * stream       cudaStream_t as void*.
 * Returns DS_OK, DS_ERR_ARG, DS_ERR_UNSUPPORTED or DS_ERR_CUDA.  Output and
 * input buffers must not overlap.
 */
int ds_topk(const void* scores, int batch, int n, int k, int dtype,
            const int32_t* valid_len, int32_t* out_idx, void* out_val,
            int return_value, int sorted_index, void* stream);

/*
 * ds_indexer_score -- the lightning-indexer score rows, written in full.
 *   (NKI pull request "Add DeepSeek-V4 CSA attention kernels", "How the
 *    algorithm works", steps table row 2.)
 *
 * q          device bfloat16 [batch, heads, d]: indexer queries.
 * kcache     device bfloat16 [S, d]: the indexer key cache shared by all rows;
 *            16-byte aligned.
 * w          device float32 [batch, heads]: per-row, per-head weights.
 * batch      >= 1;  heads 1..DS_INDEXER_MAX_HEADS;  d == DS_INDEXER_DIM;  S >= 1.
 * valid_len  device int32 [batch] or NULL (= S): row t is scored at positions
 *            s < min(max(valid_len[t], 0), S) only.
 * out_score  device float32 [batch, S]: score[t, s] for s < valid_len[t];
 *            positions at or beyond valid_len[t] are set to -inf.
 * The products are bfloat16 x bfloat16 accumulated in float32 on the tensor
 * cores; ReLU, weighting and the head sum are float32.
 * Returns DS_OK, DS_ERR_ARG, DS_ERR_UNSUPPORTED or DS_ERR_CUDA.
 */
int ds_indexer_score(const void* q, const void* kcache, const float* w,
                     int batch, int heads, int d, int S,
                     const int32_t* valid_len, float* out_score, void* stream);

/*
 * ds_indexer_topk -- indexer score followed by the top-k positions of each row.
 *   (NKI pull request "Add DeepSeek-V4 CSA attention kernels", steps table
 *    rows 2 and 3, and "The top-k on the GPSIMD engine": the scores feed the
 *    top-k as they are produced.)
 *
 * The scorer writes the score rows to the scratch buffer and also counts
 * every score in an exact per-row histogram of its key's top 12 bits; the
 * selection starts from the threshold bin those counts give.  Rows scored by
 * several CTAs (few rows, as in decode) are selected by a cluster per row
 * that splits the row; rows scored whole by one CTA (many rows, as in
 * prefill) by ds_topk's one-pass kernel, which then draws no sample.  The
 * result is the same either way.
 *
 * q, kcache, w, batch, heads, d, S, valid_len  as for ds_indexer_score.
 * k          1 <= k <= DS_MAX_K.
 * S          additionally S <= 16777216.
 * out_idx    device int32 [batch, k]: selected positions, order unspecified,
 *            -1 in padding slots.
 * out_score  device float32 [batch, k] or NULL: the float32 score of each
 *            selected position, -inf in padding slots.
 * Uses the library's scratch buffer (see above).
 * Returns DS_OK, DS_ERR_ARG, DS_ERR_UNSUPPORTED, DS_ERR_NOMEM or DS_ERR_CUDA.
 */
int ds_indexer_topk(const void* q, const void* kcache, const float* w,
                    int batch, int heads, int d, int S,
                    const int32_t* valid_len, int k,
                    int32_t* out_idx, float* out_score, void* stream);

/*
 * ds_indexer_topk_ex -- ds_indexer_topk with a key cache per row and
 * position-sorted output.
 *   (NKI pull request "Add DeepSeek-V4 CSA attention kernels", "Launching a
 *    full block": the indexer key cache is [B, T_c, index_head_dim], one per
 *    batch row; DeepSelect hub page, options paragraph: sorted_index.)
 *
 * kcache_batch_stride  0: kcache is one [S, d] cache shared by every row (as
 *            in ds_indexer_topk); otherwise row t reads the S x d cache that
 *            starts t * kcache_batch_stride rows after kcache, and the stride
 *            must be >= S (for example S for a [batch, S, d] array).
 * sorted_index 0 or 1: with 1 each row's selection is in ascending position
 *            order (the selection itself is the same).
 * The other arguments, outputs and results are those of ds_indexer_topk,
 * including its use of the scratch buffer and its choice of selection.
 */
int ds_indexer_topk_ex(const void* q, const void* kcache, int64_t kcache_batch_stride, const float* w,
                       int batch, int heads, int d, int S, const int32_t* valid_len, int k,
                       int sorted_index, int32_t* out_idx, float* out_score, void* stream);

/*
 * ds_indexer_topk_noalloc -- ds_indexer_topk for callers that must not
 * allocate device memory.
 *   (The pages have no counterpart: this is a deployment variant of the same
 *    computation.)
 *
 * Some callers cannot call cudaMalloc: a serving engine that has reserved all
 * device memory for its own pool, code running while another framework
 * captures a CUDA graph in a mode that forbids allocation, or a latency-bound
 * path that cannot take the device-wide synchronisation a first cudaMalloc may
 * cause.  This entry point never allocates or frees anything: the score rows
 * go to a fixed 1 MiB array inside the library (held by every GPU that loads
 * the library until the process exits).
 *
 * Arguments, outputs and results are those of ds_indexer_topk, with one more
 * limit: batch * S <= 262144 (for example 8 rows x 32768 positions); larger
 * calls return DS_ERR_ARG.
 * The first call on a device looks up the array's device address (a one-time
 * set-up with that device current); make that first call before any stream
 * capture.  Every call on a device uses the same array, which keeps the last
 * call's contents: calls that overlap on the GPU (different streams, no
 * ordering between them) race with each other, so order them on one stream.
 */
int ds_indexer_topk_noalloc(const void* q, const void* kcache, const float* w,
                            int batch, int heads, int d, int S,
                            const int32_t* valid_len, int k,
                            int32_t* out_idx, float* out_score, void* stream);

/*
 * ds_indexer_qproj -- the indexer query projection: the per-head queries and
 * weights that ds_indexer_score / ds_indexer_topk take, from one input vector
 * per token.
 *   (NKI pull request "Add DeepSeek-V4 CSA attention kernels", "How the
 *    algorithm works", steps table row 2: the indexer query is projected into
 *    128 channels; launch list: the query projection runs as a GEMV ahead of
 *    the scoring launch.)
 *
 *     q[t, h, c] = sum_i x[t, i] * wq[h * d + c, i]    rounded to bfloat16
 *     w[t, h]    = sum_i x[t, i] * ww[h, i]             float32
 *
 * x       device bfloat16 [T, d_in]; 16-byte aligned.
 * wq      device bfloat16 [heads * d, d_in] (row-major, one row per output
 *         channel); 16-byte aligned.
 * ww      device bfloat16 [heads, d_in] or NULL; 16-byte aligned.
 * T       1 .. 524280 tokens (decode batches are the intended use: every group
 *         of 8 tokens streams the weights once).
 * d_in    a multiple of 8, 8 <= d_in <= 8192.
 * heads   1 .. DS_INDEXER_MAX_HEADS;  d == DS_INDEXER_DIM.
 * q_out   device bfloat16 [T, heads, d] (the layout ds_indexer_topk reads).
 * w_out   device float32 [T, heads]; must be NULL exactly when ww is NULL.
 * The products of the exact bfloat16 inputs are accumulated in float32 on the
 * CUDA cores (packed two-lane FMAs); q is rounded to the nearest bfloat16.
 * Returns DS_OK, DS_ERR_ARG, DS_ERR_UNSUPPORTED or DS_ERR_CUDA.
 */
int ds_indexer_qproj(const void* x, const void* wq, const void* ww, int T, int d_in, int heads, int d,
                     void* q_out, float* w_out, void* stream);

/*
 * ds_compress_fold -- the compressor's 4:1 fold: 4 rows into 1 by a gated
 * weighted sum.
 *   (NKI pull request "Add DeepSeek-V4 CSA attention kernels", "How the
 *    algorithm works", steps table row 1: the compressor folds 4 tokens into
 *    1 with a gated weighted sum, once every 4 decode steps.)
 *
 * The pages do not give the gate.  The reading implemented: per-token scores
 * s_i = gate . x_i (float32 from the bf16 products), weights
 * a = softmax(s_0..s_3), folded row = sum_i a_i x_i, rounded to bfloat16.
 *
 * rows     device bfloat16: batch row b's 4 rows of D elements start
 *          rows_batch_stride * b elements after rows, each D after the last
 *          (a [batch, 4, D] array: stride 4 * D); 16-byte aligned.
 * batch    >= 1.   D: a multiple of 8, 8 <= D <= 4096.
 * rows_batch_stride  >= 4 * D, a multiple of 8 (elements).
 * gate     device bfloat16 [D]; 16-byte aligned.
 * out      device bfloat16: batch row b's folded row at out +
 *          out_batch_stride * b (for instance position j of a [batch, T_c, D]
 *          cache: out = cache + j * D, out_batch_stride = T_c * D);
 *          16-byte aligned.
 * out_batch_stride  >= D, a multiple of 8 (elements).
 * Returns DS_OK, DS_ERR_ARG, DS_ERR_UNSUPPORTED or DS_ERR_CUDA.
 */
int ds_compress_fold(const void* rows, int batch, int D, int64_t rows_batch_stride, const void* gate,
                     void* out, int64_t out_batch_stride, void* stream);

/*
 * ds_sparse_attention -- multi-query decode attention over the selected
 * compressed rows plus a sliding window.
 *   (NKI pull request "Add DeepSeek-V4 CSA attention kernels", "How the
 *    algorithm works": the attention reads only the selected compressed
 *    positions plus a local window, and steps table row 4 "Concatenate and
 *    attend"; "The top-k on the GPSIMD engine", last paragraph: K and V are
 *    the same embedding; "Launching a full block": the window cache
 *    [B, W, head_dim] and the compressed cache [B, T_c, head_dim].)
 *
 * For batch row b and head h, with r over the attended rows -- the cache rows
 * kv_b[idx[b, j]] of every slot j with 0 <= idx[b, j] < T, then the window
 * rows win[b, i] for i < win_len[b] -- each row serving as key and value:
 *     z[r]        = scale * (q[b, h, :] . row_r)
 *     out[b, h, :] = sum_r e^z[r] row_r / (sum_r e^z[r] + e^sink[h])
 *     lse[b, h]    = log(sum_r e^z[r] + e^sink[h])
 * The sink terms are absent when sink is NULL.  With nothing attended and no
 * sink, out is 0 and lse is -inf.
 *
 * q            device bfloat16 [batch, heads, d]; 16-byte aligned.
 * kv           device bfloat16: batch row b's compressed cache is the T rows of
 *              d elements that start kv_batch_stride * b rows after kv;
 *              16-byte aligned.
 * kv_batch_stride  rows from one batch row's cache to the next, >= 0: 0 for one
 *              cache shared by every batch row, T for a [batch, T, d] array.
 * T            rows of each cache, >= 1.
 * idx          device int32 [batch, k]: the selected rows (for instance the
 *              output of ds_indexer_topk).  Slots outside [0, T), such as the
 *              -1 padding of the top-k, are skipped; every other slot is
 *              attended, so a repeated index counts once per slot.
 * k            slots per batch row, 0 <= k <= DS_MAX_K; idx may be NULL if k = 0.
 * win          device bfloat16 [batch, W, d] or NULL (then W must be 0);
 *              16-byte aligned.
 * W            window rows per batch row, 0 <= W <= DS_ATTN_MAX_WINDOW.
 * win_len      device int32 [batch] or NULL (= W): window rows
 *              0 .. min(max(win_len[b], 0), W) - 1 are attended.
 * sink         device float32 [heads] or NULL: one logit per head.
 * batch        1 .. 65535;  heads 1 .. DS_ATTN_MAX_HEADS;
 * d            a multiple of 64, 64 <= d <= DS_ATTN_MAX_DIM.
 * scale        finite score factor (1/sqrt(d) for the usual attention).
 * out          device bfloat16 [batch, heads, d]; 16-byte aligned.
 * lse          device float32 [batch, heads] or NULL (natural logarithm).
 * Inputs are expected to be finite.  The products q . row are bf16 x bf16
 * accumulated in float32 on the tensor cores; the softmax is float32 with its
 * weights rounded to bfloat16 for the weighted sum (also a tensor-core
 * product), and the normaliser sums those rounded weights; out is rounded to
 * the nearest bfloat16.
 * Uses a scratch buffer of its own (per device, grow-only, allocated with
 * cudaMalloc on first use and by calls larger than any before, so make such
 * calls outside CUDA-graph capture; freed by ds_release): calls of
 * ds_sparse_attention on one device must be ordered on one stream.
 * Returns DS_OK, DS_ERR_ARG, DS_ERR_UNSUPPORTED, DS_ERR_NOMEM or DS_ERR_CUDA.
 */
int ds_sparse_attention(const void* q, const void* kv, int64_t kv_batch_stride, int T,
                        const int32_t* idx, int k, const void* win, int W, const int32_t* win_len,
                        const float* sink, int batch, int heads, int d, float scale,
                        void* out, float* lse, void* stream);

/*
 * ds_get_device_status -- synchronise `stream`, then return and clear the
 * current device's status word: DS_OK; DS_ERR_TIMEOUT if a kernel's bounded
 * wait ran out since the last call (the outputs of that call are then
 * unspecified, but every index is -1 or a valid position); DS_ERR_RANGE
 * (libdstopk_debug.so only) if a kernel read an input outside its documented
 * range -- a valid_len outside [0, n], an attention slot other than -1
 * outside [0, T), a win_len outside [0, W] -- which it then clamped or skipped
 * exactly as the release build does; or DS_ERR_CUDA if the synchronisation
 * itself failed.  The first error recorded since the last call is the one
 * returned.
 * (No counterpart on the pages: the library's error reporting.)
 */
int ds_get_device_status(void* stream);

/*
 * ds_set_wait_limit -- the limit of every bounded wait inside the kernels
 * (an mbarrier wait for a copy, a tensor-core result or a peer CTA), in
 * nanoseconds of the GPU's global timer: 0 restores the default of one
 * second; 0 <= ns <= 60 s, else DS_ERR_ARG.  Read by every launch enqueued
 * after the call (a CUDA graph keeps the limit it was captured with).  A wait
 * that runs out records DS_ERR_TIMEOUT and lets its kernel finish.
 * (No counterpart on the pages: the library's failure detection.)
 */
int ds_set_wait_limit(int64_t ns);

/*
 * ds_plant_wait_fault -- testing the failure detection: the next `launches`
 * indexer scorer launches (of ds_indexer_score, ds_indexer_topk and its
 * variants) each carry a planted fault: in their first CTA one epilogue warp
 * skips its first release of a tensor-core accumulator, so that the MMA warp's
 * wait for that accumulator, and the waits behind it, run out after the wait
 * limit.  The kernel then scores that CTA's remaining positions as -inf, lets
 * its copies in flight land, frees its tensor memory and returns; the call's
 * status is DS_ERR_TIMEOUT.  0 disarms.  launches >= 0, else DS_ERR_ARG.
 * Nothing traps, and the next call without the fault runs normally.  A
 * launch captured into a CUDA graph keeps the fault it was captured with.
 * (No counterpart on the pages.)
 */
int ds_plant_wait_fault(int launches);

/* ds_debug_build -- 1 in libdstopk_debug.so (compiled with DS_DEBUG: device
 * range checks that record DS_ERR_RANGE, and phase stamps), 0 in libdstopk.so. */
int ds_debug_build(void);

/*
 * ds_debug_stash_stamps -- libdstopk_debug.so only: the %globaltimer stamps
 * (ns) that thread 0 of each of the first `ctas` CTAs of the stash top-k
 * kernel recorded at the end of its phases since the last read, as `ctas` rows
 * of 10 uint64 into host_dst (0: phase not reached); the stamps are cleared.
 * Slots: start, prologue, sample counted, threshold, streamed, merged; then,
 * in a row's leader CTA only: stash counted, bin of the k-th key, bin
 * resolved, emission written.  Synchronises the device.  1 <= ctas <= 1024,
 * else DS_ERR_ARG; DS_ERR_UNSUPPORTED in libdstopk.so.
 * (No counterpart on the pages: measurement.)
 */
int ds_debug_stash_stamps(uint64_t* host_dst, int ctas);

/*
 * ds_read_floor -- enqueue a kernel that only reads `bytes` bytes at p (device,
 * 16-byte aligned, bytes a multiple of 16) with 16-byte loads, split evenly
 * over `ctas` CTAs of 1024 threads (1 .. 65535): the floor that a one-pass
 * kernel over the same bytes cannot beat.  DS_ERR_ARG on a bad argument.
 * (No counterpart on the pages: measurement.)
 */
int ds_read_floor(const void* p, int64_t bytes, int ctas, void* stream);

/* ds_strerror -- a static, human-readable name for a status code. */
const char* ds_strerror(int code);

/* ds_release -- free the scratch buffers of every device this process used.
 * No call may be in flight. */
void ds_release(void);

#ifdef __cplusplus
}
#endif

#endif /* DS_TOPK_H */
