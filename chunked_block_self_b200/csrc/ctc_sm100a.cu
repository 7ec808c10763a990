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
//                        chunks (rows may start at any 2-byte offset), keep
//                        the largest value and its lowest class, and reduce
//                        across the CTA (ties go to the lowest class; NaN
//                        logits are skipped; a frame of NaNs takes the
//                        blank).
//   ctc_collapse_kernel  one CTA per utterance: keeps frame i when its class
//                        is not the blank and differs from frame i - 1's
//                        (the utterance's first frame has no predecessor),
//                        compacts the kept classes - 1 with a block-wide
//                        scan at the utterance's own frame offset, and
//                        writes the count.
#include <climits>
#include <cstring>

#include "nle.h"
#include "nle_device.cuh"
#include "nle_host.h"

namespace {

using namespace nle;

constexpr int kArgmaxThreads = 256;
constexpr int kArgmaxCtasPerSm = 4;   // 55 registers: four CTAs of 256 threads fit an SM
constexpr int kArgmaxUnroll = 8;      // 16-byte loads in flight per thread (32 KB per CTA)
constexpr int kCollapseThreads = 256;

// (value, class) pair order: larger value first, then the lower class.
__device__ __forceinline__ bool better(float v, int c, float bv, int bc)
{
    return v > bv || (v == bv && c < bc);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ __nv_bfloat162 as_bf162(uint32_t w)
{
    __nv_bfloat162 r;
    memcpy(&r, &w, 4);
    return r;
}

// largest of a chunk's 8 values (NaN only when all 8 are NaN)
__device__ __forceinline__ float chunk_max(const uint4 &q)
{
    const __nv_bfloat162 m =
        __hmax2(__hmax2(as_bf162(q.x), as_bf162(q.y)), __hmax2(as_bf162(q.z), as_bf162(q.w)));
    uint32_t u;
    memcpy(&u, &m, 4);
    return fmaxf(bf16_lo(u), bf16_hi(u));
}

__device__ __forceinline__ float chunk_elem(const uint4 &q, int e)
{
    const uint32_t w = e < 2 ? q.x : e < 4 ? q.y : e < 6 ? q.z : q.w;
    return e & 1 ? bf16_hi(w) : bf16_lo(w);
}

// Per frame: a CTA reads the row's whole 16-byte chunks with 16-byte loads,
// eight in flight per thread (128 KB per SM: enough to cover DRAM latency at
// full bandwidth), and keeps, per thread, only the largest chunk maximum,
// the first chunk that reached it and that chunk's 8 values (packed bf16 max:
// about one instruction per logit, so the loop stays under the HBM time);
// the class inside that chunk is found from the kept values, so no logit is
// read twice.  The row's elements before its first 16-byte boundary and after its
// last one (at most 7 each) are read one by one.
__global__ void __launch_bounds__(kArgmaxThreads, kArgmaxCtasPerSm)
    ctc_argmax_kernel(const __nv_bfloat16 *__restrict__ logits, long long row_stride, int n_classes,
                      long long total_frames, int32_t *__restrict__ frame_class)
{
    __shared__ float s_val[kArgmaxThreads / 32];
    __shared__ int s_cls[kArgmaxThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (long long r = blockIdx.x; r < total_frames; r += gridDim.x) {
        const __nv_bfloat16 *row = logits + r * row_stride;
        // logits are 16-byte aligned, so a row starts on a 2-byte boundary
        const int mis = (int)((reinterpret_cast<uintptr_t>(row) & 15) >> 1);
        const int head = min((8 - mis) & 7, n_classes);   // elements before the first boundary
        const int nfull = (n_classes - head) >> 3;        // whole chunks
        const int tail0 = head + 8 * nfull;                // elements [tail0, n_classes) after them
        const uint4 *chunks = reinterpret_cast<const uint4 *>(row + head);

        float best = -INFINITY;
        int bk = -1;   // first chunk of this thread whose maximum is best (-1: none above -inf)
        uint4 bq = make_uint4(0u, 0u, 0u, 0u);   // that chunk's values
        int k = tid;
        for (; k + (kArgmaxUnroll - 1) * kArgmaxThreads < nfull; k += kArgmaxUnroll * kArgmaxThreads) {
            uint4 q[kArgmaxUnroll];
#pragma unroll
            for (int j = 0; j < kArgmaxUnroll; ++j)
                q[j] = __ldcs(chunks + k + j * kArgmaxThreads);
#pragma unroll
            for (int j = 0; j < kArgmaxUnroll; ++j) {
                const float f = chunk_max(q[j]);
                if (f > best) {
                    best = f;
                    bk = k + j * kArgmaxThreads;
                    bq = q[j];
                }
            }
        }
        for (; k < nfull; k += kArgmaxThreads) {
            const uint4 q = __ldcs(chunks + k);
            const float f = chunk_max(q);
            if (f > best) {
                best = f;
                bk = k;
                bq = q;
            }
        }

        float bv = -INFINITY;
        int bc = INT_MAX;
        if (bk >= 0) {
            // the lowest class of the chunk that holds the maximum
            const uint4 q = bq;
#pragma unroll
            for (int e = 7; e >= 0; --e)
                if (chunk_elem(q, e) == best)
                    bc = head + 8 * bk + e;
            bv = best;
        } else {
            // rare: this thread's chunks hold only -inf and NaN; the first
            // -inf is its candidate
            for (int kk = tid; kk < nfull; kk += kArgmaxThreads) {
                const uint4 q = chunks[kk];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float v = chunk_elem(q, e);
                    const int c = head + 8 * kk + e;
                    if (better(v, c, bv, bc)) {
                        bv = v;
                        bc = c;
                    }
                }
            }
        }
        // the row's loose elements: the head on lanes of warp 0, the tail on
        // lanes of warp 1
        {
            int c = -1;
            if (tid < head)
                c = tid;
            else if (tid >= 32 && tid - 32 < n_classes - tail0)
                c = tail0 + tid - 32;
            if (c >= 0) {
                const float v = __bfloat162float(row[c]);
                if (better(v, c, bv, bc)) {
                    bv = v;
                    bc = c;
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
            // all logits NaN: no candidate; the blank
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
        // every CTA resident at once; rows in a grid-stride loop
        const long long cap = (long long)di.sm_count * kArgmaxCtasPerSm;
        const long long grid = total_frames < cap ? total_frames : cap;
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
