// pool_sm100a.cu -- posterior-weighted pooling for the BPE CTC head on B200.
//
// Operation (granite-speech-4.1-2b-nar model card, "Model Architecture" (1)
// CTC Speech Encoder): the BPE head pools encoder frames over windows, each
// frame weighted by 1 - blank probability of the mid-layer CTC head.  Per
// utterance, windows of pool_frames frames are cut from its frame 0 (the
// last may be partial); window g of the packed batch is pooled row g:
//     w_t      = 1 - softmax(z_t)[0] = sum_{c>=1} e^{z_tc} / sum_c e^{z_tc}
//     pooled_g = sum_t w_t h_t / sum_t w_t      (a zero row if every w_t = 0)
// Weights are kept as logarithms, log w_t = lse(z_t[1:]) - lse(z_t), each
// sum taken about its own maximum, and a window divides e^{log w_t - max}
// by its sum: no underflow when the blank dominates by far.
//
// One kernel, HBM-bound (reads each frame's hidden row and logits once,
// writes each pooled row once).  A CTA takes whole windows: its warps reduce
// the window's frames' logits (a warp per frame), then every thread forms
// 8 output elements (one 16-byte chunk of the hidden dimension) from the
// window's frames.
#include <climits>

#include "nle.h"
#include "nle_device.cuh"
#include "nle_host.h"

namespace {

using namespace nle;

constexpr int kPoolThreads = 128;
constexpr int kPoolWarps = kPoolThreads / 32;
constexpr int kMaxPoolFrames = 4096;
constexpr float kLog2e = 1.4426950408889634f;

struct PoolParams {
    const __nv_bfloat16 *hidden;
    long long h_stride;   // elements between frames
    int dim;              // hidden size, a multiple of 8
    const __nv_bfloat16 *logits;
    long long z_stride;
    int n_classes;
    const int32_t *cu;
    int n_seq;
    int total;
    int P;                // frames per window
    long long n_rows;     // pooled rows the caller allocated
    __nv_bfloat16 *pooled;
    float *weights;       // nullable: w_t per frame
    int32_t *status;      // nullable
};

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
    return v;
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v += __shfl_xor_sync(kFull, v, o);
    return v;
}

// log(1 - p_blank) of one frame, on every lane of the warp (-inf: weight 0)
__device__ __forceinline__ float frame_log_weight(const __nv_bfloat16 *__restrict__ z, int C, int lane)
{
    float m = -INFINITY, mnb = -INFINITY;
    for (int c = lane; c < C; c += 32) {
        const float v = __bfloat162float(z[c]);
        m = fmaxf(m, v);
        if (c > 0)
            mnb = fmaxf(mnb, v);
    }
    m = warp_max(m);
    mnb = warp_max(mnb);
    if (mnb == -INFINITY)
        return -INFINITY;   // no non-blank class has any probability
    // m >= mnb > -inf: both sums are >= 1 (their maximum term is 1)
    float s = 0.f, snb = 0.f;
    for (int c = lane; c < C; c += 32) {
        const float v = __bfloat162float(z[c]);
        s += exp2f((v - m) * kLog2e);
        if (c > 0)
            snb += exp2f((v - mnb) * kLog2e);
    }
    s = warp_sum(s);
    snb = warp_sum(snb);
    return (mnb - m) + (logf(snb) - logf(s));
}

__global__ void __launch_bounds__(kPoolThreads) posterior_pool_kernel(PoolParams p)
{
    extern __shared__ float s_lw[];   // [P] log weights of the current window
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n_chunks = p.dim >> 3;
    PlanWalker w;
    w.init(p.cu, p.n_seq, p.total, p.P, lane);
    for (long long g = blockIdx.x;; g += gridDim.x) {
        int f0, L, seq;
        if (!w.find(g, lane, f0, L, seq))
            break;
        if (g >= p.n_rows) {
            // more windows than pooled rows: nothing past the buffer is written
            if (tid == 0)
                report(p.status, NLE_ERR_INVALID_ARG);
            break;
        }
        for (int t = warp; t < L; t += kPoolWarps) {
            const float lw = frame_log_weight(p.logits + (long long)(f0 + t) * p.z_stride, p.n_classes, lane);
            if (lane == 0) {
                s_lw[t] = lw;
                if (p.weights)
                    p.weights[f0 + t] = expf(lw);
            }
        }
        __syncthreads();
        float M = -INFINITY;
        for (int t = 0; t < L; ++t)
            M = fmaxf(M, s_lw[t]);
        __nv_bfloat16 *orow = p.pooled + g * (long long)p.dim;
        for (int ch = tid; ch < n_chunks; ch += kPoolThreads) {
            uint4 res = make_uint4(0u, 0u, 0u, 0u);
            if (M != -INFINITY) {
                float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                float wsum = 0.f;
                const __nv_bfloat16 *hrow = p.hidden + (long long)f0 * p.h_stride + 8 * ch;
                for (int t = 0; t < L; ++t) {
                    const float r = exp2f((s_lw[t] - M) * kLog2e);   // 0 for a weight of 0
                    const uint4 q = __ldcs(reinterpret_cast<const uint4 *>(hrow + (long long)t * p.h_stride));
                    const uint32_t wd[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        acc[2 * e] = fmaf(r, __uint_as_float(wd[e] << 16), acc[2 * e]);
                        acc[2 * e + 1] = fmaf(r, __uint_as_float(wd[e] & 0xffff0000u), acc[2 * e + 1]);
                    }
                    wsum += r;
                }
                const float inv = 1.f / wsum;   // wsum >= 1: the largest weight contributes 1
                res = make_uint4(pack_bf16x2(acc[0] * inv, acc[1] * inv), pack_bf16x2(acc[2] * inv, acc[3] * inv),
                                 pack_bf16x2(acc[4] * inv, acc[5] * inv), pack_bf16x2(acc[6] * inv, acc[7] * inv));
            }
            *reinterpret_cast<uint4 *>(orow + 8 * ch) = res;
        }
        __syncthreads();   // s_lw is rewritten by the next window
    }
    if (w.bad && tid == 0)
        report(p.status, NLE_ERR_INVALID_ARG);
}

} // namespace

extern "C" int nle_posterior_pool_fwd(const void *hidden, int64_t hidden_stride, int dim, const void *logits,
                                      int64_t logits_stride, int n_classes, const int32_t *cu_seqlens, int n_seq,
                                      int64_t total_frames, int pool_frames, int64_t n_pooled_rows, void *pooled,
                                      float *weights, int32_t *dev_status, void *stream)
{
    if (n_seq < 0 || total_frames < 0 || dim <= 0 || n_classes < 1 || pool_frames < 1 || n_pooled_rows < 0 ||
        hidden_stride < dim || logits_stride < n_classes)
        return NLE_ERR_INVALID_ARG;
    if (dim % 8 != 0 || hidden_stride % 8 != 0)
        return NLE_ERR_MISALIGNED;
    if (total_frames > 0x7fffffffLL || pool_frames > kMaxPoolFrames)
        return NLE_ERR_UNSUPPORTED;
    if (n_seq == 0 || total_frames == 0 || n_pooled_rows == 0)
        return NLE_OK;
    if (!hidden || !logits || !cu_seqlens || !pooled)
        return NLE_ERR_INVALID_ARG;
    if (!nle::aligned16(hidden) || !nle::aligned16(pooled) || (reinterpret_cast<uintptr_t>(logits) & 1u))
        return NLE_ERR_MISALIGNED;
    nle::DeviceInfo di;
    int dev = 0;
    if (!nle::current_device_info(&di, &dev))
        return NLE_ERR_CUDA;
    if (di.cc_major != 10)
        return NLE_ERR_UNSUPPORTED;
    PoolParams p;
    p.hidden = static_cast<const __nv_bfloat16 *>(hidden);
    p.h_stride = hidden_stride;
    p.dim = dim;
    p.logits = static_cast<const __nv_bfloat16 *>(logits);
    p.z_stride = logits_stride;
    p.n_classes = n_classes;
    p.cu = cu_seqlens;
    p.n_seq = n_seq;
    p.total = (int)total_frames;
    p.P = pool_frames;
    p.n_rows = n_pooled_rows;
    p.pooled = static_cast<__nv_bfloat16 *>(pooled);
    p.weights = weights;
    p.status = dev_status;
    const long long cap = (long long)di.sm_count * 16;
    const int grid = (int)(n_pooled_rows < cap ? n_pooled_rows : cap);
    posterior_pool_kernel<<<grid, kPoolThreads, sizeof(float) * pool_frames, static_cast<cudaStream_t>(stream)>>>(p);
    return cudaGetLastError() == cudaSuccess ? NLE_OK : NLE_ERR_CUDA;
}
