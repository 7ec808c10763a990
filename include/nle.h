/*
 * nle.h -- C ABI of libnle.so: varlen block self-attention and windowed
 * cross-attention on NVIDIA B200 (sm_100a), with full-utterance attention,
 * the BPE head's posterior-weighted pooling and CTC greedy decoding (each
 * documented at its entry point below).
 *
 * The operations (sources are the web pages this library follows):
 *
 *  Block self-attention -- granite-speech-4.1-2b-nar model card, "Model
 *  Architecture", (1) CTC Speech Encoder: the encoder uses block attention
 *  with 4-second audio blocks.  At 50 Hz encoder frames (100 Hz log-mel,
 *  2-frame stacking) a block is 200 frames.  Utterances are packed back to
 *  back ("Usage / Installation": sequence packing, is_causal=False).  Block j
 *  of utterance i covers frames [cu[i] + j*B, cu[i] + min((j+1)*B, T_i)) with
 *  T_i = cu[i+1] - cu[i]; every frame attends, bidirectionally, to every frame
 *  of its block and to nothing else:
 *      S = scale * Q_blk K_blk^T,  P = softmax_rows(S),  O_blk = P V_blk.
 *
 *  Windowed cross-attention -- same card, (2) Q-Former Projector: each
 *  15-frame window is reduced to 3 queries via cross-attention.  Windows are
 *  cut per utterance from its frame 0 like the blocks (the last one may be
 *  partial); window g of the packed batch owns query rows
 *  queries_per_window*g ... +queries_per_window-1, each attending to the
 *  window's frames.
 *
 * Conventions for every attention entry point below (the pooling and CTC
 * entry points state their own layouts):
 *  - Tensor pointers (q, k, v, out, cu_seqlens, dev_status) are DEVICE
 *    pointers owned by the caller.  The kernel entry points never allocate,
 *    free or synchronise; every launch is asynchronous on `stream` (a
 *    cudaStream_t; NULL = the legacy default stream).  Host-side table
 *    functions take HOST pointers and say so.  The one exception is
 *    nle_path_fwd_host, which creates two streams and three events per
 *    device on its first call (kept for the life of the process) and whose
 *    copies block the calling thread unless the host buffers are pinned.
 *  - q, k, v, out hold bf16 values, row-major [rows][heads][d_head]: one row
 *    per frame (or per query), heads next, d_head contiguous.  d_head must be
 *    64.  Base pointers must be 16-byte aligned.
 *  - cu_seqlens is int32 [n_seq + 1], non-decreasing, within
 *    [0, total_frames]; normally cu[0] = 0 and cu[n_seq] = total_frames, but
 *    a slice of a longer cu (absolute offsets) processes just those
 *    utterances.  The kernels read it on the device; a sequence whose
 *    offsets fall outside [0, total_frames] or decrease is skipped (no output
 *    is written for it) and, where a dev_status word is given, reported as
 *    NLE_ERR_INVALID_ARG.  No access ever leaves the buffers described by
 *    total_frames / n_query_rows.
 *  - Softmax runs in fp32 with the scale folded into exp2; QK^T and PV
 *    accumulate in fp32; P is rounded to bf16 before PV; out is rounded to
 *    bf16 (round to nearest even).
 *  - out must not alias q, k or v.
 *  - Errors found on the host are returned before anything is launched:
 *    NLE_ERR_INVALID_ARG, NLE_ERR_UNSUPPORTED, NLE_ERR_MISALIGNED.  A launch
 *    failure returns NLE_ERR_CUDA.  n_seq == 0 or total_frames == 0 is a
 *    successful no-op.
 *  - Every wait inside a kernel is bounded.  Past the limit the kernel stores
 *    NLE_ERR_TIMEOUT into *dev_status (when given), releases what it holds and
 *    returns; the CUDA context stays usable.
 */
#ifndef NLE_H
#define NLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define NLE_ABI_VERSION 2

typedef enum {
    NLE_OK = 0,
    NLE_ERR_INVALID_ARG = -1, /* null pointer with work to do, bad sizes    */
    NLE_ERR_UNSUPPORTED = -2, /* d_head != 64, block_frames > 256, ...      */
    NLE_ERR_MISALIGNED = -3,  /* pointer or row stride not 16-byte aligned  */
    NLE_ERR_CUDA = -4,        /* launch or device-query failure             */
    NLE_ERR_TIMEOUT = -5      /* a bounded in-kernel wait expired           */
} nle_status;

/* Flags for the _ex entry points. */
#define NLE_FLAG_NONE 0
/* Test hook: the load of the first work item is never issued, so its
 * consumers' bounded waits expire and the kernel reports NLE_ERR_TIMEOUT.
 * Exercises the timeout path without hanging the GPU. */
#define NLE_FLAG_TEST_SKIP_FIRST_LOAD 1
/* Work split of nle_block_attn_fwd_ex (results are identical either way).
 * By default a batch whose (block, head) items number at most the device's
 * SM count runs each row tile of a block as its own work item, so the two
 * 128-row tiles of a block run at once on two chains (lower latency for
 * short batches, K and V read once per row tile); larger batches run whole
 * items.  These flags force one or the other. */
#define NLE_FLAG_WHOLE_ITEMS 2
#define NLE_FLAG_SPLIT_ITEMS 4

/* ABI version (NLE_ABI_VERSION of the build). */
int nle_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char *nle_status_string(int status);

/* ---------------------------------------------------------------------
 * Block self-attention (model card, "Model Architecture" (1)).
 *
 * q, k, v, out   device bf16 [total_frames][heads][64]
 * cu_seqlens     device int32 [n_seq + 1]
 * n_seq          number of packed utterances (>= 0)
 * total_frames   rows of q/k/v/out (>= cu[n_seq]); < 2^31
 * heads          >= 1
 * d_head         must be 64
 * block_frames   frames per block, 1..256 (200 for 4 s at 50 Hz)
 * stream         cudaStream_t
 * Returns NLE_OK or a negative nle_status.
 */
int nle_block_attn_fwd(const void *q, const void *k, const void *v, void *out,
                       const int32_t *cu_seqlens, int n_seq,
                       int64_t total_frames, int heads, int d_head,
                       int block_frames, void *stream);

/* As nle_block_attn_fwd, plus:
 * softmax_scale    <= 0 selects 1/sqrt(d_head)
 * row_stride_qkv   elements between consecutive frames of q, k and v (for
 *                  a fused QKV buffer); 0 selects heads*d_head; must be a
 *                  multiple of 8 and >= heads*d_head.  out is always dense
 *                  (row stride heads*d_head).
 * dev_status       device int32 or NULL; receives the first in-kernel error
 *                  (NLE_ERR_TIMEOUT or NLE_ERR_INVALID_ARG); never reset by
 *                  the library.
 * flags            NLE_FLAG_* (0 in production: the test hook, and the
 *                  work-split overrides)
 * wait_limit_ns    limit of every in-kernel wait; 0 selects 1 s.
 */
int nle_block_attn_fwd_ex(const void *q, const void *k, const void *v,
                          void *out, const int32_t *cu_seqlens, int n_seq,
                          int64_t total_frames, int heads, int d_head,
                          int block_frames, float softmax_scale,
                          int64_t row_stride_qkv, int32_t *dev_status,
                          int flags, int64_t wait_limit_ns, void *stream);

/* ---------------------------------------------------------------------
 * QKV projection fused with block self-attention (model card, "Model
 * Architecture" (1): each encoder layer's self-attention projects its
 * hidden states to queries, keys and values and attends within 4 s blocks).
 * For every block and head h:
 *     [Q_h | K_h | V_h] = bf16(X_blk W_h^T + b_h)  (fp32 accumulation, one
 *                                                   rounding to bf16)
 *     O_blk,h = softmax(scale * Q_h K_h^T) V_h     (as nle_block_attn_fwd)
 * Q, K and V are formed on chip and never written to memory.
 *
 * x              device bf16 [total_frames][d_model], dense rows
 * w_qkv          device bf16 [3 * heads * 64][d_model]: a linear layer's
 *                weight (output features x input features); rows
 *                [0, H*64) give Q, [H*64, 2*H*64) K, [2*H*64, 3*H*64) V,
 *                head h taking rows h*64 .. h*64+63 of each
 * bias           nullable device bf16 [3 * heads * 64], same row order
 * out            device bf16 [total_frames][heads][64]
 * cu_seqlens     device int32 [n_seq + 1] (as nle_block_attn_fwd)
 * d_model        input features: a multiple of 64, at most 16384
 * heads, d_head  heads >= 1, d_head must be 64
 * block_frames   1..256 (200 for 4 s at 50 Hz)
 * x, w_qkv, bias and out must be 16-byte aligned.  Errors as
 * nle_block_attn_fwd (NLE_ERR_UNSUPPORTED also for d_model not a multiple
 * of 64 or above 16384).  No allocation; asynchronous on `stream`.
 * The _ex form adds softmax_scale (<= 0: 1/sqrt(d_head)), dev_status, flags
 * and wait_limit_ns, as nle_block_attn_fwd_ex.
 */
int nle_block_attn_qkv_fwd(const void *x, const void *w_qkv, const void *bias,
                           void *out, const int32_t *cu_seqlens, int n_seq,
                           int64_t total_frames, int d_model, int heads,
                           int d_head, int block_frames, void *stream);

int nle_block_attn_qkv_fwd_ex(const void *x, const void *w_qkv,
                              const void *bias, void *out,
                              const int32_t *cu_seqlens, int n_seq,
                              int64_t total_frames, int d_model, int heads,
                              int d_head, int block_frames,
                              float softmax_scale, int32_t *dev_status,
                              int flags, int64_t wait_limit_ns, void *stream);

/* ---------------------------------------------------------------------
 * Windowed cross-attention (model card, "Model Architecture" (2)).
 *
 * q, out          device bf16 [n_query_rows][heads][64]; n_query_rows must be
 *                 queries_per_window * (number of windows), see
 *                 nle_window_plan_host
 * k, v            device bf16 [total_frames][heads][64]
 * cu_seqlens_kv   device int32 [n_seq + 1] over the key/value frames
 * window_frames   1..32 (15 on the pages)
 * queries_per_window 1..16 (3 on the pages)
 */
int nle_window_xattn_fwd(const void *q, const void *k, const void *v,
                         void *out, const int32_t *cu_seqlens_kv, int n_seq,
                         int64_t total_frames, int64_t n_query_rows, int heads,
                         int d_head, int window_frames,
                         int queries_per_window, void *stream);

/* As nle_window_xattn_fwd with an explicit scale (<= 0: 1/sqrt(d_head)),
 * status word, test flags and wait limit (see nle_block_attn_fwd_ex). */
int nle_window_xattn_fwd_ex(const void *q, const void *k, const void *v,
                            void *out, const int32_t *cu_seqlens_kv, int n_seq,
                            int64_t total_frames, int64_t n_query_rows,
                            int heads, int d_head, int window_frames,
                            int queries_per_window, float softmax_scale,
                            int32_t *dev_status, int flags,
                            int64_t wait_limit_ns, void *stream);

/* ---------------------------------------------------------------------
 * Full bidirectional self-attention inside each packed utterance, any
 * length (granite-speech-4.1-2b-nar model card, "Model Architecture" (3)
 * Bidirectional LLM Editor: the LLM with its causal mask removed; "Usage /
 * Installation": packed sequences, is_causal=False): for every utterance i
 * and head h,  O = softmax(scale * Q K^T) V  over all T_i frames of the
 * utterance -- block attention with one block per utterance.  Keys are
 * walked in tiles of 64 with an online softmax (fp32, exact power-of-two
 * rescaling), P rounded to bf16 before PV, O rounded to bf16.
 *
 * Arguments, layouts, ownership and errors as nle_block_attn_fwd, without
 * block_frames (and no limit on T_i).  The _ex form adds softmax_scale
 * (<= 0: 1/sqrt(d_head)), row_stride_qkv, dev_status, flags and the wait
 * limit, as nle_block_attn_fwd_ex.
 */
int nle_varlen_attn_fwd(const void *q, const void *k, const void *v, void *out,
                        const int32_t *cu_seqlens, int n_seq, int64_t total_frames,
                        int heads, int d_head, void *stream);

int nle_varlen_attn_fwd_ex(const void *q, const void *k, const void *v, void *out,
                           const int32_t *cu_seqlens, int n_seq, int64_t total_frames,
                           int heads, int d_head, float softmax_scale,
                           int64_t row_stride_qkv, int32_t *dev_status, int flags,
                           int64_t wait_limit_ns, void *stream);

/* ---------------------------------------------------------------------
 * CTC greedy decoding of the encoder's CTC head (q4-RTN ONNX page,
 * "Inference note (NAR decode)"): the head emits n_classes per frame with
 * the blank at class 0, and a non-blank class c is token c - 1.  Per frame
 * the class of the largest logit is taken (bf16 compared exactly; among
 * equal largest logits the lowest class, -0 equal to +0; NaN logits are no
 * candidates and a frame of NaNs takes the blank); per
 * utterance, runs of equal consecutive classes become one (runs never cross
 * utterances), blanks are dropped and classes become tokens.
 *
 * logits       device bf16 [total_frames][row_stride]; the first n_classes
 *              of each row are used; base 16-byte aligned, rows may start
 *              at any element
 * row_stride   elements between frames, >= n_classes
 * cu_seqlens   device int32 [n_seq + 1] (as for the attention kernels)
 * frame_class  device int32 [total_frames], out: class of each frame
 * tokens       device int32 [total_frames], out: utterance i's tokens at
 *              tokens[cu[i]] .. tokens[cu[i] + n_tokens[i] - 1]; the rest of
 *              its frame range is left untouched
 * n_tokens     device int32 [n_seq], out: tokens of each utterance (0 for an
 *              utterance whose offsets are invalid)
 * Two kernels on `stream` (argmax, then collapse); no allocation.
 * Errors (before launch): NLE_ERR_INVALID_ARG for n_seq < 0, total_frames
 * < 0, n_classes < 1, row_stride < n_classes or a null pointer with work to
 * do; NLE_ERR_UNSUPPORTED for total_frames > 2^31 - 1 or a device other than
 * compute capability 10.x; NLE_ERR_MISALIGNED when logits is not 16-byte
 * aligned; NLE_ERR_CUDA for a launch error.
 */
int nle_ctc_greedy_fwd(const void *logits, int64_t row_stride, int n_classes, const int32_t *cu_seqlens,
                       int n_seq, int64_t total_frames, int32_t *frame_class, int32_t *tokens,
                       int32_t *n_tokens, void *stream);

/* ---------------------------------------------------------------------
 * Posterior-weighted pooling for the BPE CTC head (granite-speech-4.1-2b-nar
 * model card, "Model Architecture" (1) CTC Speech Encoder): frames are
 * pooled over windows, each weighted by 1 - blank probability of the
 * mid-layer CTC head.  Per utterance, windows of pool_frames frames are cut
 * from its frame 0 without overlap (the last may be partial); window g of
 * the packed batch is pooled row g:
 *     w_t = 1 - softmax(z_t)[0],   pooled_g = sum_t w_t h_t / sum_t w_t,
 * a zero row when every weight of the window is 0 (w_t = 0 exactly when
 * every non-blank logit is -inf).  The page's window of 4 counts 10 ms input
 * frames, i.e. pool_frames = 2 encoder frames at 50 Hz (844 mel frames give
 * 211 rows of the BPE head).  fp32 arithmetic, weights formed in the log
 * domain; pooled rows rounded to bf16.  Logits must be finite or -inf.
 *
 * hidden         device bf16 [total_frames][hidden_stride]; the first dim
 *                columns are pooled; 16-byte aligned, hidden_stride and dim
 *                multiples of 8
 * logits         device bf16 [total_frames][logits_stride] of the mid-layer
 *                head, blank at class 0; the first n_classes used
 * cu_seqlens     device int32 [n_seq + 1] (as for the attention kernels;
 *                invalid utterances are skipped and reported)
 * n_pooled_rows  rows of `pooled`: sum_i ceil(T_i / pool_frames); windows
 *                past it are not written and are reported
 * pooled         device bf16 [n_pooled_rows][dim], out; 16-byte aligned
 * weights        nullable device float32 [total_frames], out: w_t
 * dev_status     nullable device int32, receives NLE_ERR_INVALID_ARG for a
 *                bad utterance or too few rows (never reset by the library)
 * One kernel on `stream`; no allocation.  Errors (before launch):
 * NLE_ERR_INVALID_ARG for negative sizes, dim < 1, n_classes < 1,
 * pool_frames < 1, a stride below its width or a null pointer with work to
 * do; NLE_ERR_MISALIGNED for dim or hidden_stride not a multiple of 8,
 * hidden or pooled not 16-byte aligned; NLE_ERR_UNSUPPORTED for
 * total_frames > 2^31 - 1, pool_frames > 4096 or a device other than
 * compute capability 10.x; NLE_ERR_CUDA for a launch error.
 */
int nle_posterior_pool_fwd(const void *hidden, int64_t hidden_stride, int dim, const void *logits,
                           int64_t logits_stride, int n_classes, const int32_t *cu_seqlens, int n_seq,
                           int64_t total_frames, int pool_frames, int64_t n_pooled_rows, void *pooled,
                           float *weights, int32_t *dev_status, void *stream);

/* ---------------------------------------------------------------------
 * The whole path from host memory: block self-attention of (q, k, v) and
 * windowed cross-attention of (qw, kw, vw) over the same n_seq packed
 * utterances (cu), with the copies in and out.
 *
 * Host buffers (pinned memory lets the copies overlap the kernels):
 *   q, k, v, out        [total_frames][heads][64] bf16
 *   qw, out_w           [n_query_rows][heads][64] bf16, n_query_rows =
 *                       queries_per_window * (number of windows)
 *   kw, vw              [total_frames][heads][64] bf16
 *   cu                  int32 [n_seq + 1], non-decreasing from 0
 * Device buffers, owned by the caller, of the same shapes: d_q ... d_cu.
 *
 * Resources: on its first call on a device this entry point creates two
 * non-blocking streams and three events for that device, kept until the
 * process exits (it allocates no memory).  The host buffers should be
 * page-locked (cudaHostAlloc / cudaHostRegister): with pageable memory the
 * copies are staged by the driver and block the calling thread.
 *
 * The utterances are split into n_chunks chunks of consecutive utterances
 * (0 selects 8; at most n_seq).  For each chunk the input rows are copied to
 * the device, both kernels run on the chunk (each kernel call takes the
 * chunk's slice of cu, whose offsets stay absolute), and the output rows are
 * copied back; chunks alternate between two internal streams, so the copies
 * of one chunk overlap the kernels and copies of another.  Everything is
 * ordered after the work already on `stream`, and `stream` waits for all of
 * it: the call returns at once, like cudaMemcpyAsync, and the host buffers
 * must stay valid until `stream` has reached this point.
 * Returns NLE_OK or the first error (argument checks as for the two kernel
 * entry points; NLE_ERR_INVALID_ARG if cu is not non-decreasing from 0 or
 * the query rows do not match the windows).
 */
typedef struct {
    const void *q, *k, *v;     /* host inputs of block self-attention       */
    void *out;                 /* host output of block self-attention       */
    const void *qw, *kw, *vw;  /* host inputs of windowed cross-attention   */
    void *out_w;               /* host output of windowed cross-attention   */
    const int32_t *cu;         /* host cu_seqlens                           */
    void *d_q, *d_k, *d_v, *d_out, *d_qw, *d_kw, *d_vw, *d_out_w;
    int32_t *d_cu;             /* device copies (caller-owned)              */
    int32_t *d_status;         /* nullable device int32: receives the first
                                  in-kernel error of either kernel (a wait
                                  that ran out: NLE_ERR_TIMEOUT); never
                                  reset by the library.  With NULL such an
                                  error goes unreported and the rows of the
                                  work item concerned are left unwritten.  */
} nle_path_buffers;

int nle_path_fwd_host(const nle_path_buffers *b, int n_seq, int64_t total_frames, int64_t n_query_rows,
                      int heads, int d_head, int block_frames, int window_frames, int queries_per_window,
                      int n_chunks, void *stream);

/* ---------------------------------------------------------------------
 * Block / window plans (the integer scheduling the kernels perform).
 *
 * nle_block_plan_host: HOST pointers.  Enumerates the blocks of the packed
 * batch in order: out_seq[b] = utterance, out_j[b] = block index inside it,
 * out_start[b] = first frame, out_len[b] = frames in the block.  Output
 * arrays may be NULL to only count.  *n_blocks receives the count.
 * Returns NLE_ERR_INVALID_ARG if cu is not non-decreasing from 0, or if the
 * count exceeds capacity while arrays are given.
 */
int nle_block_plan_host(const int32_t *cu_host, int n_seq, int block_frames,
                        int32_t *out_seq, int32_t *out_j, int32_t *out_start,
                        int32_t *out_len, int capacity, int *n_blocks);

/* The same table computed on the device by the walker the kernels use.
 * cu_dev and the out_* arrays are DEVICE pointers (out_* may be NULL);
 * n_blocks_dev (device int32, required) receives the total count; entries
 * past `capacity` are not written.  Asynchronous on `stream`. */
int nle_block_plan_dev(const int32_t *cu_dev, int n_seq, int64_t total_frames,
                       int block_frames, int32_t *out_seq, int32_t *out_j,
                       int32_t *out_start, int32_t *out_len, int capacity,
                       int32_t *n_blocks_dev, void *stream);

/* Window table on the host (HOST pointers): as nle_block_plan_host with
 * window_frames, plus out_qrow[g] = queries_per_window * g.  *n_windows
 * receives the count; the query tensor then has
 * queries_per_window * (*n_windows) rows. */
int nle_window_plan_host(const int32_t *cu_host, int n_seq, int window_frames,
                         int queries_per_window, int32_t *out_seq,
                         int32_t *out_w, int32_t *out_start, int32_t *out_len,
                         int32_t *out_qrow, int capacity, int *n_windows);

/* ---------------------------------------------------------------------
 * Multi-GPU data parallelism (replicas by utterance; no collective on the
 * data path).  HOST pointers.  Splits n_seq utterances of the given lengths
 * into world_size contiguous shards balancing the attention cost
 * sum over blocks of len^2.  out_bounds[r] .. out_bounds[r+1] is rank r's
 * utterance range (out_bounds has world_size + 1 entries).
 */
int nle_shard_plan_host(const int32_t *lengths_host, int n_seq,
                        int block_frames, int world_size, int32_t *out_bounds);

#ifdef __cplusplus
}
#endif

#endif /* NLE_H */
