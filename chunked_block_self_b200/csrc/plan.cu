// plan.cu -- the integer scheduling of the packed batch (S1): the host copy
// and the device copy (the warp-level PlanWalker every kernel runs), plus
// the host-side shard plan for data-parallel replicas.
//
// Cutting rule (granite-speech-4.1-2b-nar model card, "Model Architecture"
// (1) and (2)): utterance i = frames [cu[i], cu[i+1]); units (200-frame
// blocks, or 15-frame windows) are cut from its frame 0; the last one may be
// partial; units are numbered over the batch in utterance order.
#include <vector>

#include "nle.h"
#include "nle_device.cuh"

namespace {

__global__ void plan_kernel(const int32_t *cu, int n_seq, int total, int unit, int32_t *out_seq,
                            int32_t *out_j, int32_t *out_start, int32_t *out_len, int capacity,
                            int32_t *n_units)
{
    const int lane = threadIdx.x & 31;
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int n_warps = (gridDim.x * blockDim.x) >> 5;
    nle::PlanWalker w;
    w.init(cu, n_seq, total, unit, lane);
    for (long long u = warp; u < capacity; u += n_warps) {
        int f0, L, s;
        if (!w.find(u, lane, f0, L, s))
            break;
        if (lane == 0) {
            int cu_s = __ldg(cu + s);
            if (out_seq)
                out_seq[u] = s;
            if (out_j)
                out_j[u] = (f0 - cu_s) / unit;
            if (out_start)
                out_start[u] = f0;
            if (out_len)
                out_len[u] = L;
        }
    }
    if (warp == 0) {
        // total unit count: walk to the end of the batch
        nle::PlanWalker t;
        t.init(cu, n_seq, total, unit, lane);
        while (t.base + 32 < n_seq) {
            t.before += t.group_units;
            t.base += 32;
            t.load_group(lane);
        }
        if (lane == 0)
            *n_units = t.before + t.group_units;
    }
}

int host_units(const int32_t *cu, int n_seq, int unit, int32_t *a, int32_t *b, int32_t *c,
               int32_t *d, int capacity, int *count)
{
    if (!count || n_seq < 0 || unit <= 0 || (n_seq > 0 && !cu))
        return NLE_ERR_INVALID_ARG;
    if (n_seq > 0 && cu[0] != 0)
        return NLE_ERR_INVALID_ARG;
    const bool write = a || b || c || d;
    long long n = 0;
    for (int i = 0; i < n_seq; ++i) {
        const long long t = (long long)cu[i + 1] - cu[i];
        if (t < 0)
            return NLE_ERR_INVALID_ARG;
        const long long nu = (t + unit - 1) / unit;
        for (long long j = 0; j < nu; ++j) {
            if (write) {
                if (n >= capacity)
                    return NLE_ERR_INVALID_ARG;
                if (a)
                    a[n] = i;
                if (b)
                    b[n] = (int32_t)j;
                if (c)
                    c[n] = (int32_t)(cu[i] + j * unit);
                if (d)
                    d[n] = (int32_t)((t - j * unit) < unit ? (t - j * unit) : unit);
            }
            ++n;
        }
    }
    if (n > 0x7fffffffLL)
        return NLE_ERR_INVALID_ARG;
    *count = (int)n;
    return NLE_OK;
}

} // namespace

extern "C" int nle_block_plan_host(const int32_t *cu_host, int n_seq, int block_frames,
                                   int32_t *out_seq, int32_t *out_j, int32_t *out_start,
                                   int32_t *out_len, int capacity, int *n_blocks)
{
    return host_units(cu_host, n_seq, block_frames, out_seq, out_j, out_start, out_len, capacity,
                      n_blocks);
}

extern "C" int nle_window_plan_host(const int32_t *cu_host, int n_seq, int window_frames,
                                    int queries_per_window, int32_t *out_seq, int32_t *out_w,
                                    int32_t *out_start, int32_t *out_len, int32_t *out_qrow,
                                    int capacity, int *n_windows)
{
    if (queries_per_window <= 0)
        return NLE_ERR_INVALID_ARG;
    int rc = host_units(cu_host, n_seq, window_frames, out_seq, out_w, out_start, out_len, capacity,
                        n_windows);
    if (rc != NLE_OK)
        return rc;
    if ((long long)*n_windows * queries_per_window > 0x7fffffffLL)
        return NLE_ERR_INVALID_ARG;
    if (out_qrow)
        for (int g = 0; g < *n_windows; ++g)
            out_qrow[g] = queries_per_window * g;
    return NLE_OK;
}

extern "C" int nle_block_plan_dev(const int32_t *cu_dev, int n_seq, int64_t total_frames,
                                  int block_frames, int32_t *out_seq, int32_t *out_j,
                                  int32_t *out_start, int32_t *out_len, int capacity,
                                  int32_t *n_blocks_dev, void *stream)
{
    if (n_seq < 0 || block_frames <= 0 || capacity < 0 || total_frames < 0 ||
        total_frames > 0x7fffffffLL || !n_blocks_dev || (n_seq > 0 && !cu_dev))
        return NLE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (n_seq == 0) {
        if (cudaMemsetAsync(n_blocks_dev, 0, sizeof(int32_t), s) != cudaSuccess)
            return NLE_ERR_CUDA;
        return NLE_OK;
    }
    int blocks = (capacity + 255) / 256;  // 8 warps per block, ~32 units per warp
    if (blocks < 1)
        blocks = 1;
    if (blocks > 1024)
        blocks = 1024;
    plan_kernel<<<blocks, 256, 0, s>>>(cu_dev, n_seq, (int)total_frames, block_frames, out_seq,
                                       out_j, out_start, out_len, capacity, n_blocks_dev);
    return cudaGetLastError() == cudaSuccess ? NLE_OK : NLE_ERR_CUDA;
}

extern "C" int nle_shard_plan_host(const int32_t *lengths_host, int n_seq, int block_frames,
                                   int world_size, int32_t *out_bounds)
{
    if (n_seq < 0 || block_frames <= 0 || world_size <= 0 || !out_bounds ||
        (n_seq > 0 && !lengths_host))
        return NLE_ERR_INVALID_ARG;
    // cost of an utterance: sum over its blocks of len^2 (the attention work)
    std::vector<double> prefix(n_seq + 1, 0.0);
    for (int i = 0; i < n_seq; ++i) {
        const long long t = lengths_host[i];
        if (t < 0)
            return NLE_ERR_INVALID_ARG;
        const long long full = t / block_frames, rem = t % block_frames;
        const double c = (double)full * block_frames * block_frames + (double)rem * rem;
        prefix[i + 1] = prefix[i] + c;
    }
    // contiguous split: rank r ends at the first utterance whose prefix cost
    // reaches (r+1)/world_size of the total (ties go to the earlier rank)
    out_bounds[0] = 0;
    int i = 0;
    for (int r = 1; r < world_size; ++r) {
        const double target = prefix[n_seq] * r / world_size;
        while (i < n_seq && prefix[i + 1] <= target)
            ++i;
        // pick the closer of the two cut points i and i+1
        if (i < n_seq && (prefix[i + 1] - target) < (target - prefix[i]))
            ++i;
        if (i < out_bounds[r - 1])
            i = out_bounds[r - 1];
        out_bounds[r] = i;
    }
    out_bounds[world_size] = n_seq;
    return NLE_OK;
}
