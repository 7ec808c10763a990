/*
 * oracle.c -- plain, slow, fp64 CPU oracle for chunked (block) bidirectional
 * self-attention and for the projector's windowed cross-attention.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the definition the CUDA path is
 * checked against.  Only the test suite, the smoke check and the bench's CPU
 * baseline leg may load it.  It shares no code, header, table or helper with
 * the CUDA library: it re-derives every index and every number itself.
 *
 * What it computes (sources):
 *  - granite-speech-4.1-2b-nar model card, "Model Architecture", (1) CTC
 *    Speech Encoder: block attention over 4-second audio blocks.  With 100 Hz
 *    log-mel frames stacked by 2 the encoder runs at 50 Hz, so one block is
 *    200 encoder frames.  Every frame attends to every frame of its own block
 *    (no causal mask: "Usage / Installation" requires a backend that keeps
 *    is_causal=False and supports sequence packing) and to nothing outside.
 *  - Reading taken where the pages are silent: blocks are cut per utterance
 *    starting at the utterance's frame 0 (the portable README's rank-5
 *    windowed MatMuls run per fixed-length bucket); the last block of an
 *    utterance is partial and attends only to its own frames.
 *  - granite-speech-4.1-2b-nar model card, "Model Architecture", (2) Q-Former
 *    Projector: each 15-frame window is reduced to 3 queries by
 *    cross-attention.  Reading: windows are cut per utterance from frame 0,
 *    do not overlap, and the last one may be partial; window g (counted over
 *    the whole packed batch) owns query rows 3g..3g+2.
 *
 * Arithmetic: inputs are bf16 bit patterns, widened exactly to double.
 * Everything after that is double: S = scale * q.k, p = exp(S - max) / sum,
 * o = sum_c p_c v_c.  No blocking, fusion or reordering beyond the definition.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* ------------------------------------------------------------------ */
/* bf16 bit pattern -> double (exact: bf16 is the top half of a float) */
static double bf16_to_double(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------ */
/* Block enumeration.  Utterance i holds frames [cu[i], cu[i+1]).  Its
 * blocks are j = 0, 1, ... while j*B < T_i; block j covers frames
 * [cu[i] + j*B, cu[i] + min((j+1)*B, T_i)).  Blocks are numbered over the
 * packed batch in utterance order.  Returns the number of blocks, or -1 if
 * cu is not non-decreasing from 0, or if capacity is too small (when the
 * output arrays are given). */
int orc_block_table(const int32_t *cu, int n_seq, int block_frames,
                    int32_t *out_seq, int32_t *out_j, int32_t *out_start,
                    int32_t *out_len, int capacity)
{
    if (n_seq < 0 || block_frames <= 0)
        return -1;
    if (n_seq > 0 && cu[0] != 0)
        return -1;
    int count = 0;
    for (int i = 0; i < n_seq; ++i) {
        int32_t t = cu[i + 1] - cu[i];
        if (t < 0)
            return -1;
        for (int32_t j = 0; (int64_t)j * block_frames < t; ++j) {
            int32_t first = j * block_frames;
            int32_t len = t - first;
            if (len > block_frames)
                len = block_frames;
            if (out_seq) {
                if (count >= capacity)
                    return -1;
                out_seq[count] = i;
                out_j[count] = j;
                out_start[count] = cu[i] + first;
                out_len[count] = len;
            }
            ++count;
        }
    }
    return count;
}

/* Window enumeration for the projector: identical cutting rule with
 * window_frames in place of block_frames; additionally reports the first
 * query row of each window, queries_per_window * (global window index). */
int orc_window_table(const int32_t *cu, int n_seq, int window_frames,
                     int queries_per_window, int32_t *out_seq, int32_t *out_w,
                     int32_t *out_start, int32_t *out_len, int32_t *out_qrow,
                     int capacity)
{
    if (queries_per_window <= 0)
        return -1;
    int n = orc_block_table(cu, n_seq, window_frames, out_seq, out_w,
                            out_start, out_len, capacity);
    if (n < 0 || !out_qrow)
        return n;
    for (int g = 0; g < n; ++g)
        out_qrow[g] = queries_per_window * g;
    return n;
}

/* ------------------------------------------------------------------ */
/* One query row attending over a contiguous key range.
 *   qrow   : pointer to d bf16 values of the query
 *   k0, v0 : pointer to the first key / value row of the range
 *   stride : elements between consecutive key (value) rows
 *   n_keys : number of keys in the range (>= 1)
 *   probs  : if not NULL, receives the n_keys softmax probabilities
 *   out    : receives d doubles
 * Scratch for the n_keys scores is allocated here (plain, not fast). */
static int attend_row(const uint16_t *qrow, const uint16_t *k0,
                      const uint16_t *v0, int64_t stride, int n_keys, int d,
                      double scale, double *probs, double *out)
{
    double *s = (double *)malloc(sizeof(double) * (size_t)n_keys);
    if (!s)
        return -1;
    /* S_c = scale * sum_e q_e k_{c,e} */
    for (int c = 0; c < n_keys; ++c) {
        const uint16_t *kr = k0 + (int64_t)c * stride;
        double acc = 0.0;
        for (int e = 0; e < d; ++e)
            acc += bf16_to_double(qrow[e]) * bf16_to_double(kr[e]);
        s[c] = scale * acc;
    }
    /* p_c = exp(S_c - m) / sum_c' exp(S_c' - m) */
    double m = s[0];
    for (int c = 1; c < n_keys; ++c)
        if (s[c] > m)
            m = s[c];
    double l = 0.0;
    for (int c = 0; c < n_keys; ++c) {
        s[c] = exp(s[c] - m);
        l += s[c];
    }
    for (int c = 0; c < n_keys; ++c)
        s[c] /= l;
    if (probs)
        for (int c = 0; c < n_keys; ++c)
            probs[c] = s[c];
    /* o_e = sum_c p_c v_{c,e} */
    for (int e = 0; e < d; ++e) {
        double acc = 0.0;
        for (int c = 0; c < n_keys; ++c)
            acc += s[c] * bf16_to_double(v0[(int64_t)c * stride + e]);
        out[e] = acc;
    }
    free(s);
    return 0;
}

/* The block holding frame `row`: utterance i with cu[i] <= row < cu[i+1],
 * block j = (row - cu[i]) / B.  Returns 0 and the block's first frame and
 * length, or -1 if the row is in no utterance. */
static int block_of_row(const int32_t *cu, int n_seq, int block_frames,
                        int64_t row, int64_t *start, int *len)
{
    for (int i = 0; i < n_seq; ++i) {
        if (row >= cu[i] && row < cu[i + 1]) {
            int64_t off = row - cu[i];
            int64_t j = off / block_frames;
            int64_t first = j * block_frames;
            int64_t t = cu[i + 1] - cu[i];
            *start = cu[i] + first;
            *len = (int)((t - first) < block_frames ? (t - first) : block_frames);
            return 0;
        }
    }
    return -1;
}

/* ------------------------------------------------------------------ */
/* Block self-attention, all outputs.
 * q, k, v : bf16 bit patterns, row-major [total_frames][heads][d]
 * out     : doubles, same layout.  Rows outside every utterance are not
 *           written.
 * The work is split over (block, head) pairs on n_threads POSIX threads
 * (0 = all online cores); each pair is computed by attend_row above. */
typedef struct {
    const uint16_t *q, *k, *v;
    int heads, d;
    double scale;
    const int32_t *blk_start, *blk_len;
    int n_items;
    double *out;
    int next_item;
    pthread_mutex_t lock;
    int failed;
} block_job;

static void *block_worker(void *arg)
{
    block_job *job = (block_job *)arg;
    for (;;) {
        pthread_mutex_lock(&job->lock);
        int item = job->next_item++;
        pthread_mutex_unlock(&job->lock);
        if (item >= job->n_items)
            break;
        int b = item / job->heads, h = item % job->heads;
        int64_t stride = (int64_t)job->heads * job->d;
        int64_t s0 = job->blk_start[b];
        int len = job->blk_len[b];
        for (int r = 0; r < len; ++r) {
            int64_t row = s0 + r;
            if (attend_row(job->q + row * stride + (int64_t)h * job->d,
                           job->k + s0 * stride + (int64_t)h * job->d,
                           job->v + s0 * stride + (int64_t)h * job->d, stride,
                           len, job->d, job->scale, NULL,
                           job->out + row * stride + (int64_t)h * job->d) != 0)
                job->failed = 1;
        }
    }
    return NULL;
}

static int run_threads(void *(*fn)(void *), void *job, int n_threads)
{
    if (n_threads <= 0) {
        long n = sysconf(_SC_NPROCESSORS_ONLN);
        n_threads = n > 0 ? (int)n : 1;
    }
    pthread_t *tid = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)n_threads);
    if (!tid)
        return -1;
    int started = 0;
    for (int t = 0; t < n_threads; ++t) {
        if (pthread_create(&tid[t], NULL, fn, job) != 0)
            break;
        ++started;
    }
    if (started == 0)
        fn(job);
    for (int t = 0; t < started; ++t)
        pthread_join(tid[t], NULL);
    free(tid);
    return started > 0 ? started : 1;
}

int orc_block_attn(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                   const int32_t *cu, int n_seq, int heads, int d,
                   int block_frames, double scale, double *out, int n_threads)
{
    int n_blocks = orc_block_table(cu, n_seq, block_frames, NULL, NULL, NULL,
                                   NULL, 0);
    if (n_blocks < 0 || heads <= 0 || d <= 0)
        return -1;
    if (n_blocks == 0)
        return 0;
    int32_t *seq = (int32_t *)malloc(sizeof(int32_t) * (size_t)n_blocks * 4);
    if (!seq)
        return -1;
    int32_t *jj = seq + n_blocks, *st = jj + n_blocks, *ln = st + n_blocks;
    orc_block_table(cu, n_seq, block_frames, seq, jj, st, ln, n_blocks);
    block_job job = {q, k, v, heads, d, scale, st, ln, n_blocks * heads, out,
                     0, PTHREAD_MUTEX_INITIALIZER, 0};
    int used = run_threads(block_worker, &job, n_threads);
    free(seq);
    return job.failed ? -1 : used;
}

/* Selected outputs only: for each pair (rows[i], heads_sel[i]) write the d
 * outputs of that frame and head to out[i*d .. i*d+d).  Used to check the
 * full-size launches at sampled positions. */
int orc_block_attn_rows(const uint16_t *q, const uint16_t *k,
                        const uint16_t *v, const int32_t *cu, int n_seq,
                        int heads, int d, int block_frames, double scale,
                        const int64_t *rows, const int32_t *heads_sel, int n,
                        double *out)
{
    int64_t stride = (int64_t)heads * d;
    for (int i = 0; i < n; ++i) {
        int64_t s0;
        int len;
        if (block_of_row(cu, n_seq, block_frames, rows[i], &s0, &len) != 0)
            return -1;
        int h = heads_sel[i];
        if (attend_row(q + rows[i] * stride + (int64_t)h * d,
                       k + s0 * stride + (int64_t)h * d,
                       v + s0 * stride + (int64_t)h * d, stride, len, d, scale,
                       NULL, out + (int64_t)i * d) != 0)
            return -1;
    }
    return 0;
}

/* The softmax probabilities of one (row, head): writes the first key's frame
 * index to *key_start, the number of keys to *n_keys and the probabilities to
 * probs (capacity >= block_frames). */
int orc_block_attn_probs(const uint16_t *q, const uint16_t *k,
                         const uint16_t *v, const int32_t *cu, int n_seq,
                         int heads, int d, int block_frames, double scale,
                         int64_t row, int head, double *probs, int *n_keys,
                         int64_t *key_start, double *out)
{
    int64_t stride = (int64_t)heads * d;
    int64_t s0;
    int len;
    if (block_of_row(cu, n_seq, block_frames, row, &s0, &len) != 0)
        return -1;
    *n_keys = len;
    *key_start = s0;
    return attend_row(q + row * stride + (int64_t)head * d,
                      k + s0 * stride + (int64_t)head * d,
                      v + s0 * stride + (int64_t)head * d, stride, len, d,
                      scale, probs, out);
}

/* ------------------------------------------------------------------ */
/* Windowed cross-attention (projector).
 * q   : bf16 [queries_per_window * n_windows][heads][d]
 * k,v : bf16 [total_frames][heads][d]
 * out : doubles shaped like q.
 * Window g of utterance i covers frames [start, start + len); its query rows
 * are queries_per_window*g .. +queries_per_window-1 and each attends to the
 * window's len frames. */
typedef struct {
    const uint16_t *q, *k, *v;
    int heads, d, qpw;
    double scale;
    const int32_t *w_start, *w_len;
    int n_items;
    double *out;
    int next_item;
    pthread_mutex_t lock;
    int failed;
} window_job;

static void *window_worker(void *arg)
{
    window_job *job = (window_job *)arg;
    for (;;) {
        pthread_mutex_lock(&job->lock);
        int item = job->next_item++;
        pthread_mutex_unlock(&job->lock);
        if (item >= job->n_items)
            break;
        int g = item / job->heads, h = item % job->heads;
        int64_t stride = (int64_t)job->heads * job->d;
        int64_t s0 = job->w_start[g];
        for (int r = 0; r < job->qpw; ++r) {
            int64_t qrow = (int64_t)job->qpw * g + r;
            if (attend_row(job->q + qrow * stride + (int64_t)h * job->d,
                           job->k + s0 * stride + (int64_t)h * job->d,
                           job->v + s0 * stride + (int64_t)h * job->d, stride,
                           job->w_len[g], job->d, job->scale, NULL,
                           job->out + qrow * stride + (int64_t)h * job->d) != 0)
                job->failed = 1;
        }
    }
    return NULL;
}

int orc_window_xattn(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                     const int32_t *cu, int n_seq, int heads, int d,
                     int window_frames, int queries_per_window, double scale,
                     double *out, int n_threads)
{
    int n_win = orc_block_table(cu, n_seq, window_frames, NULL, NULL, NULL,
                                NULL, 0);
    if (n_win < 0 || heads <= 0 || d <= 0 || queries_per_window <= 0)
        return -1;
    if (n_win == 0)
        return 0;
    int32_t *buf = (int32_t *)malloc(sizeof(int32_t) * (size_t)n_win * 4);
    if (!buf)
        return -1;
    int32_t *ww = buf + n_win, *st = ww + n_win, *ln = st + n_win;
    orc_block_table(cu, n_seq, window_frames, buf, ww, st, ln, n_win);
    window_job job = {q, k, v, heads, d, queries_per_window, scale, st, ln,
                      n_win * heads, out, 0, PTHREAD_MUTEX_INITIALIZER, 0};
    int used = run_threads(window_worker, &job, n_threads);
    free(buf);
    return job.failed ? -1 : used;
}

/* Selected query rows of the windowed cross-attention: for each pair
 * (qrows[i], heads_sel[i]) write d outputs to out[i*d ..). */
int orc_window_xattn_rows(const uint16_t *q, const uint16_t *k,
                          const uint16_t *v, const int32_t *cu, int n_seq,
                          int heads, int d, int window_frames,
                          int queries_per_window, double scale,
                          const int64_t *qrows, const int32_t *heads_sel,
                          int n, double *out)
{
    int64_t stride = (int64_t)heads * d;
    for (int i = 0; i < n; ++i) {
        int64_t g = qrows[i] / queries_per_window;
        /* find window g by walking utterances in order */
        int64_t before = 0, s0 = -1;
        int len = 0;
        for (int s = 0; s < n_seq && s0 < 0; ++s) {
            int64_t t = cu[s + 1] - cu[s];
            int64_t nw = (t + window_frames - 1) / window_frames;
            if (g < before + nw) {
                int64_t w = g - before;
                s0 = cu[s] + w * window_frames;
                len = (int)((t - w * window_frames) < window_frames
                                ? (t - w * window_frames)
                                : window_frames);
            }
            before += nw;
        }
        if (s0 < 0)
            return -1;
        int h = heads_sel[i];
        if (attend_row(q + qrows[i] * stride + (int64_t)h * d,
                       k + s0 * stride + (int64_t)h * d,
                       v + s0 * stride + (int64_t)h * d, stride, len, d, scale,
                       NULL, out + (int64_t)i * d) != 0)
            return -1;
    }
    return 0;
}
