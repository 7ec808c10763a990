// ctc_sm100a.cu -- CTC greedy decoding of the encoder's CTC head on B200.
//
// Operation (ibm-granite-speech-4.1-2b-nar-q4-rtn-onnx page, "Inference note
// (NAR decode)"): the head emits vocab + 1 classes per frame with the blank
// at class 0, and a non-blank class c is token c - 1.  Per frame: the class
// of the largest logit; per utterance: runs of equal consecutive classes
// become one, blanks are dropped, classes become tokens.
//
// Two kernels:
//   ctc_argmax_kernel    streams the logits once (HBM-bound: 2 bytes per
//                        class per frame).  A CTA takes whole frames; its
//                        threads read the frame's row as 16-byte aligned
//                        chunks (rows may start at any 2-byte offset: the
//                        chunk elements outside the row are masked), keep
//                        the largest value and its lowest class, and reduce
//                        across the CTA (ties go to the lowest class).
//   ctc_collapse_kernel  one CTA per utterance: keeps frame i when its class
//                        is not the blank and differs from frame i - 1's
//                        (the utterance's first frame has no predecessor),
//                        compacts the kept classes - 1 with a block-wide
//                        scan at the utterance's own frame offset, and
//                        writes the count.
#include <climits>

#include "nle.h"
#include "nle_device.cuh"
#include "nle_host.h"

namespace {

using namespace nle;

constexpr int kArgmaxThreads = 256;
constexpr int kCollapseThreads = 256;

// (value, class) pair order: larger value first, then the lower class.
__device__ __forceinline__ bool better(float v, int c, float bv, int bc)
{
    return v > bv || (v == bv && c < bc);
}

__global__ void __launch_bounds__(kArgmaxThreads)
    ctc_argmax_kernel(const __nv_bfloat16 *__restrict__ logits, long long row_stride, int n_classes,
                      long long total_frames, int32_t *__restrict__ frame_class)
{
    __shared__ float s_val[kArgmaxThreads / 32];
    __shared__ int s_cls[kArgmaxThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // 16-byte chunks are only read below the last 16-byte boundary of the
    // tensor; a row's elements past it (at most 7) are read one by one
    const uintptr_t end = reinterpret_cast<uintptr_t>(logits + (total_frames - 1) * row_stride + n_classes);
    const uintptr_t end16 = end & ~uintptr_t(15);
    for (long long r = blockIdx.x; r < total_frames; r += gridDim.x) {
        const uintptr_t row = reinterpret_cast<uintptr_t>(logits + r * row_stride);
        const uintptr_t a0 = row & ~uintptr_t(15);
        const uintptr_t row_end = row + 2ull * n_classes;
        const long long n_cover = (long long)((row_end - a0 + 15) >> 4);   // chunks covering the row
        const long long n_safe = (long long)((end16 - a0) >> 4);             // chunks below end16
        const long long n_chunks = n_cover < n_safe ? n_cover : n_safe;
        const bool tail = n_cover > n_chunks;
        // class of the first element of chunk 0 (negative: before the row)
        const long long c_first = -(long long)((row - a0) >> 1);
        float bv = -INFINITY;
        int bc = INT_MAX;
        long long k = tid;
        // four independent 16-byte loads in flight per thread
        for (; k + 3 * kArgmaxThreads < n_chunks; k += 4 * kArgmaxThreads) {
            uint4 q[4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
                q[j] = __ldcs(reinterpret_cast<const uint4 *>(a0) + k + j * kArgmaxThreads);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const long long c0 = c_first + 8 * (k + j * kArgmaxThreads);
                const uint32_t w[4] = {q[j].x, q[j].y, q[j].z, q[j].w};
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const long long c = c0 + e;
                    const float v = __uint_as_float(e & 1 ? w[e >> 1] & 0xffff0000u : w[e >> 1] << 16);
                    if (c >= 0 && c < n_classes && better(v, (int)c, bv, bc)) {
                        bv = v;
                        bc = (int)c;
                    }
                }
            }
        }
        if (tail && tid == 0) {
            // the row's elements from end16 on: element loads only
            const __nv_bfloat16 *p = reinterpret_cast<const __nv_bfloat16 *>(a0) + 8 * n_chunks;
            for (long long c = c_first + 8 * n_chunks; c < n_classes; ++c, ++p) {
                const float v = __bfloat162float(*p);
                if (c >= 0 && better(v, (int)c, bv, bc)) {
                    bv = v;
                    bc = (int)c;
                }
            }
        }
        for (; k < n_chunks; k += kArgmaxThreads) {
            const uint4 q = __ldcs(reinterpret_cast<const uint4 *>(a0) + k);
            const long long c0 = c_first + 8 * k;
            const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const long long c = c0 + e;
                const float v = __uint_as_float(e & 1 ? w[e >> 1] & 0xffff0000u : w[e >> 1] << 16);
                if (c >= 0 && c < n_classes && better(v, (int)c, bv, bc)) {
                    bv = v;
                    bc = (int)c;
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(kFull, bv, o);
            const int oc = __shfl_xor_sync(kFull, bc, o);
            if (better(ov, oc, bv, bc)) {
                bv = ov;
                bc = oc;
            }
        }
        if (lane == 0) {
            s_val[warp] = bv;
            s_cls[warp] = bc;
        }
        __syncthreads();
        if (tid == 0) {
            for (int i = 1; i < kArgmaxThreads / 32; ++i)
                if (better(s_val[i], s_cls[i], bv, bc)) {
                    bv = s_val[i];
                    bc = s_cls[i];
                }
            // all logits NaN: no class compared larger; report the blank
            frame_class[r] = bc == INT_MAX ? 0 : bc;
        }
        __syncthreads();
    }
}

__global__ void __launch_bounds__(kCollapseThreads)
    ctc_collapse_kernel(const int32_t *__restrict__ cu, int n_seq, long long total_frames,
                        const int32_t *__restrict__ frame_class, int32_t *__restrict__ tokens,
                        int32_t *__restrict__ n_tokens)
{
    __shared__ int s_warp[kCollapseThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int u = blockIdx.x; u < n_seq; u += gridDim.x) {
        const int s = cu[u], e = cu[u + 1];
        if (s < 0 || e < s || (long long)e > total_frames) {
            if (tid == 0)
                n_tokens[u] = 0;   // invalid offsets: nothing decoded
            continue;
        }
        int count = 0;
        for (int base = s; base < e; base += kCollapseThreads) {
            const int i = base + tid;
            bool keep = false;
            int c = 0;
            if (i < e) {
                c = frame_class[i];
                keep = c != 0 && (i == s || c != frame_class[i - 1]);
            }
            const unsigned m = __ballot_sync(kFull, keep);
            if (lane == 0)
                s_warp[warp] = __popc(m);
            __syncthreads();
            int before = 0, total = 0;
#pragma unroll
            for (int w = 0; w < kCollapseThreads / 32; ++w) {
                before += w < warp ? s_warp[w] : 0;
                total += s_warp[w];
            }
            if (keep)
                tokens[s + count + before + __popc(m & ((1u << lane) - 1))] = c - 1;
            count += total;
            __syncthreads();
        }
        if (tid == 0)
            n_tokens[u] = count;
    }
}

} // namespace

extern "C" int nle_ctc_greedy_fwd(const void *logits, int64_t row_stride, int n_classes, const int32_t *cu_seqlens,
                                  int n_seq, int64_t total_frames, int32_t *frame_class, int32_t *tokens,
                                  int32_t *n_tokens, void *stream)
{
    if (n_seq < 0 || total_frames < 0 || n_classes < 1 || row_stride < n_classes)
        return NLE_ERR_INVALID_ARG;
    if (total_frames > 0x7fffffffLL)
        return NLE_ERR_UNSUPPORTED;
    if (n_seq == 0 && total_frames == 0)
        return NLE_OK;
    if (!logits || !frame_class || (n_seq > 0 && (!cu_seqlens || !tokens || !n_tokens)))
        return NLE_ERR_INVALID_ARG;
    if (!nle::aligned16(logits))
        return NLE_ERR_MISALIGNED;
    nle::DeviceInfo di;
    int dev = 0;
    if (!nle::current_device_info(&di, &dev))
        return NLE_ERR_CUDA;
    if (di.cc_major != 10)
        return NLE_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (total_frames > 0) {
        const long long grid = total_frames < (long long)di.sm_count * 8 ? total_frames : (long long)di.sm_count * 8;
        ctc_argmax_kernel<<<(int)grid, kArgmaxThreads, 0, st>>>(static_cast<const __nv_bfloat16 *>(logits),
                                                                 (long long)row_stride, n_classes, total_frames,
                                                                 frame_class);
    }
    if (n_seq > 0) {
        const int grid = n_seq < di.sm_count * 16 ? n_seq : di.sm_count * 16;
        ctc_collapse_kernel<<<grid, kCollapseThreads, 0, st>>>(cu_seqlens, n_seq, (long long)total_frames,
                                                               frame_class, tokens, n_tokens);
    }
    return cudaGetLastError() == cudaSuccess ? NLE_OK : NLE_ERR_CUDA;
}
