// host_path.cpp -- the whole path from host memory: copies in, block
// self-attention and windowed cross-attention, copies out, pipelined over
// chunks of utterances on two internal streams (see nle_path_fwd_host in
// nle.h).
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>
#include <vector>

#include "nle.h"
#include "nle_host.h"

namespace {

constexpr int kMaxDevices = 64;
constexpr int kDefaultChunks = 8;

// Two non-blocking streams and the events that order them, per device,
// created on first use and kept for the life of the process.
struct PathStreams {
    cudaStream_t s[2] = {nullptr, nullptr};
    cudaEvent_t start = nullptr, done[2] = {nullptr, nullptr};
    bool ok = false;
    std::mutex call;   // one call at a time per device: the events are shared
};

PathStreams g_streams[kMaxDevices];
std::mutex g_streams_mu;

PathStreams *path_streams(int dev)
{
    if (dev < 0 || dev >= kMaxDevices)
        return nullptr;
    std::lock_guard<std::mutex> lock(g_streams_mu);
    PathStreams &ps = g_streams[dev];
    if (!ps.ok) {
        for (int i = 0; i < 2; ++i)
            if (cudaStreamCreateWithFlags(&ps.s[i], cudaStreamNonBlocking) != cudaSuccess ||
                cudaEventCreateWithFlags(&ps.done[i], cudaEventDisableTiming) != cudaSuccess)
                return nullptr;
        if (cudaEventCreateWithFlags(&ps.start, cudaEventDisableTiming) != cudaSuccess)
            return nullptr;
        ps.ok = true;
    }
    return &ps;
}

inline const char *at(const void *base, int64_t row, int64_t row_bytes)
{
    return static_cast<const char *>(base) + row * row_bytes;
}

inline char *at(void *base, int64_t row, int64_t row_bytes) { return static_cast<char *>(base) + row * row_bytes; }

} // namespace

extern "C" int nle_path_fwd_host(const nle_path_buffers *b, int n_seq, int64_t total_frames, int64_t n_query_rows,
                                 int heads, int d_head, int block_frames, int window_frames,
                                 int queries_per_window, int n_chunks, void *stream)
{
    if (!b || n_seq < 0 || total_frames < 0 || n_query_rows < 0 || heads <= 0 || block_frames <= 0 ||
        window_frames <= 0 || queries_per_window <= 0 || n_chunks < 0)
        return NLE_ERR_INVALID_ARG;
    if (d_head != 64)
        return NLE_ERR_UNSUPPORTED;
    if (n_seq == 0)
        return NLE_OK;
    const void *host_in[] = {b->q, b->k, b->v, b->qw, b->kw, b->vw, b->cu, b->out, b->out_w};
    const void *dev_in[] = {b->d_q, b->d_k, b->d_v, b->d_qw, b->d_kw, b->d_vw, b->d_cu, b->d_out, b->d_out_w};
    for (const void *ptr : host_in)
        if (!ptr)
            return NLE_ERR_INVALID_ARG;
    for (const void *ptr : dev_in)
        if (!ptr)
            return NLE_ERR_INVALID_ARG;

    // the windows of each utterance, and the cu checks the kernels would
    // otherwise report on the device
    const int32_t *cu = b->cu;
    if (cu[0] != 0 || (int64_t)cu[n_seq] != total_frames)
        return NLE_ERR_INVALID_ARG;
    std::vector<int64_t> win_before((size_t)n_seq + 1, 0);   // windows of utterances [0, i)
    for (int i = 0; i < n_seq; ++i) {
        const int64_t t = (int64_t)cu[i + 1] - cu[i];
        if (t < 0)
            return NLE_ERR_INVALID_ARG;
        win_before[i + 1] = win_before[i] + (t + window_frames - 1) / window_frames;
    }
    if ((int64_t)queries_per_window * win_before[n_seq] != n_query_rows)
        return NLE_ERR_INVALID_ARG;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return NLE_ERR_CUDA;
    PathStreams *ps = path_streams(dev);
    if (!ps)
        return NLE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(ps->call);
    cudaStream_t user = static_cast<cudaStream_t>(stream);

    // chunk boundaries: consecutive utterances, about total_frames / chunks
    // frames each
    int chunks = n_chunks ? n_chunks : kDefaultChunks;
    if (chunks > n_seq)
        chunks = n_seq;
    std::vector<int> first(1, 0);
    for (int c = 1; c < chunks; ++c) {
        const int64_t target = total_frames * c / chunks;
        int i = first.back() + 1;
        while (i < n_seq && cu[i] < target)
            ++i;
        if (i < n_seq)
            first.push_back(i);
    }
    first.push_back(n_seq);
    chunks = (int)first.size() - 1;

    const int64_t row_bytes = (int64_t)heads * 64 * 2;
    const int Qw = queries_per_window;
    // everything waits for the work already on the caller's stream
    if (cudaEventRecord(ps->start, user) != cudaSuccess ||
        cudaStreamWaitEvent(ps->s[0], ps->start, 0) != cudaSuccess ||
        cudaStreamWaitEvent(ps->s[1], ps->start, 0) != cudaSuccess)
        return NLE_ERR_CUDA;
    // cu once, on stream 0; stream 1 waits for it
    if (cudaMemcpyAsync(b->d_cu, cu, sizeof(int32_t) * ((size_t)n_seq + 1), cudaMemcpyHostToDevice, ps->s[0]) !=
            cudaSuccess ||
        cudaEventRecord(ps->done[0], ps->s[0]) != cudaSuccess ||
        cudaStreamWaitEvent(ps->s[1], ps->done[0], 0) != cudaSuccess)
        return NLE_ERR_CUDA;

    int rc = NLE_OK;
    for (int c = 0; c < chunks && rc == NLE_OK; ++c) {
        cudaStream_t s = ps->s[c & 1];
        const int i0 = first[c], i1 = first[c + 1];
        const int64_t f0 = cu[i0], nf = (int64_t)cu[i1] - cu[i0];
        const int64_t r0 = Qw * win_before[i0], nr = Qw * (win_before[i1] - win_before[i0]);
        const void *in_src[] = {b->q, b->k, b->v, b->kw, b->vw};
        void *in_dst[] = {b->d_q, b->d_k, b->d_v, b->d_kw, b->d_vw};
        for (int t = 0; t < 5 && rc == NLE_OK; ++t)
            if (nf > 0 && cudaMemcpyAsync(at(in_dst[t], f0, row_bytes), at(in_src[t], f0, row_bytes),
                                          (size_t)(nf * row_bytes), cudaMemcpyHostToDevice, s) != cudaSuccess)
                rc = NLE_ERR_CUDA;
        if (rc == NLE_OK && nr > 0 &&
            cudaMemcpyAsync(at(b->d_qw, r0, row_bytes), at(b->qw, r0, row_bytes), (size_t)(nr * row_bytes),
                            cudaMemcpyHostToDevice, s) != cudaSuccess)
            rc = NLE_ERR_CUDA;
        if (rc != NLE_OK)
            break;
        // the chunk's slice of cu keeps absolute frame offsets; the window
        // kernel numbers the chunk's windows from 0, so its query and output
        // pointers start at the chunk's first query row
        rc = nle_block_attn_fwd_ex(b->d_q, b->d_k, b->d_v, b->d_out, b->d_cu + i0, i1 - i0, total_frames, heads,
                                   d_head, block_frames, 0.f, 0, b->d_status, 0, 0, s);
        if (rc != NLE_OK)
            break;
        rc = nle_window_xattn_fwd_ex(at(b->d_qw, r0, row_bytes), b->d_kw, b->d_vw, at(b->d_out_w, r0, row_bytes),
                                     b->d_cu + i0, i1 - i0, total_frames, nr, heads, d_head, window_frames, Qw, 0.f,
                                     b->d_status, 0, 0, s);
        if (rc != NLE_OK)
            break;
        if ((nf > 0 && cudaMemcpyAsync(at(b->out, f0, row_bytes), at(static_cast<const void *>(b->d_out), f0,
                                                                        row_bytes),
                                       (size_t)(nf * row_bytes), cudaMemcpyDeviceToHost, s) != cudaSuccess) ||
            (nr > 0 && cudaMemcpyAsync(at(b->out_w, r0, row_bytes), at(static_cast<const void *>(b->d_out_w), r0,
                                                                          row_bytes),
                                       (size_t)(nr * row_bytes), cudaMemcpyDeviceToHost, s) != cudaSuccess))
            rc = NLE_ERR_CUDA;
    }
    // the caller's stream waits for both internal streams (also after an
    // error, so nothing issued is left unordered)
    for (int i = 0; i < 2; ++i)
        if (cudaEventRecord(ps->done[i], ps->s[i]) != cudaSuccess ||
            cudaStreamWaitEvent(user, ps->done[i], 0) != cudaSuccess)
            return NLE_ERR_CUDA;
    return rc;
}
