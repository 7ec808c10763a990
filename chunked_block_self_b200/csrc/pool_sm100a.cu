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
// HBM-bound (reads each frame's hidden row and logits once, writes each
// pooled row once).  A warp takes whole windows: it reduces each frame's
// logits to the frame's log weight, then every lane forms 8 output elements
// (16-byte chunks of the hidden dimension) at a time.  Two kernels:
//   posterior_pool_pipe_kernel<NCH>  the encoder's shapes (windows of <= 2
//                  frames, width <= 1024, <= 256 classes in 16-byte chunks):
//                  two windows in flight per warp through a cp.async ring in
//                  shared memory, offsets fixed at compile time for NCH
//                  hidden chunks per lane, packed fp32 FMAs;
//   posterior_pool_kernel  any other shape: loads in registers.
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

__device__ __forceinline__ void chunk_vals(const uint4 &q, float (&v)[8])
{
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        v[2 * e] = __uint_as_float(w[e] << 16);
        v[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
    }
}

// log(1 - p_blank) of one frame, on every lane of the warp (-inf: weight 0).
// With m the frame's largest logit, both sums are taken about m with one
// exp per logit: log w = log sum_{c>=1} e^{z_c - m} - log sum_c e^{z_c - m}.
// When the non-blank maximum mnb lies more than 60 below m (a blank that
// dominates by far), the non-blank sum is taken again about mnb so that it
// cannot underflow.  vec: rows 16-byte aligned and C a multiple of 8 (the
// logits are read as 16-byte chunks of 8 classes).
__device__ __forceinline__ float frame_log_weight(const __nv_bfloat16 *__restrict__ z, int C, bool vec, int lane)
{
    float m = -INFINITY, mnb = -INFINITY;
    float s = 0.f, snb = 0.f;
    if (vec && C <= 256) {
        // at most one chunk per lane: the values stay in registers
        float v[8];
        const bool has = 8 * lane < C;
        if (has) {
            chunk_vals(__ldcs(reinterpret_cast<const uint4 *>(z) + lane), v);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                m = fmaxf(m, v[e]);
                if (lane > 0 || e > 0)
                    mnb = fmaxf(mnb, v[e]);
            }
        }
        m = warp_max(m);
        mnb = warp_max(mnb);
        if (mnb == -INFINITY)
            return -INFINITY;   // no non-blank class has any probability
        if (has) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float x = exp2f((v[e] - m) * kLog2e);
                s += x;
                if (lane > 0 || e > 0)
                    snb += x;
            }
        }
        if (mnb - m < -60.f) {
            snb = 0.f;
            if (has)
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    if (lane > 0 || e > 0)
                        snb += exp2f((v[e] - mnb) * kLog2e);
        }
    } else if (vec) {
        const uint4 *zc = reinterpret_cast<const uint4 *>(z);
        for (int k = lane; 8 * k < C; k += 32) {
            float v[8];
            chunk_vals(zc[k], v);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                m = fmaxf(m, v[e]);
                if (k > 0 || e > 0)
                    mnb = fmaxf(mnb, v[e]);
            }
        }
        m = warp_max(m);
        mnb = warp_max(mnb);
        if (mnb == -INFINITY)
            return -INFINITY;
        const bool far = mnb - m < -60.f;   // warp-uniform
        const float mr = far ? mnb : m;      // shift of the non-blank sum
        for (int k = lane; 8 * k < C; k += 32) {
            float v[8];
            chunk_vals(zc[k], v);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float x = exp2f((v[e] - m) * kLog2e);
                s += x;
                if (k > 0 || e > 0)
                    snb += far ? exp2f((v[e] - mr) * kLog2e) : x;
            }
        }
    } else {
        for (int c = lane; c < C; c += 32) {
            const float v = __bfloat162float(z[c]);
            m = fmaxf(m, v);
            if (c > 0)
                mnb = fmaxf(mnb, v);
        }
        m = warp_max(m);
        mnb = warp_max(mnb);
        if (mnb == -INFINITY)
            return -INFINITY;
        const bool far = mnb - m < -60.f;
        const float mr = far ? mnb : m;
        for (int c = lane; c < C; c += 32) {
            const float v = __bfloat162float(z[c]);
            const float x = exp2f((v - m) * kLog2e);
            s += x;
            if (c > 0)
                snb += far ? exp2f((v - mr) * kLog2e) : x;
        }
    }
    s = warp_sum(s);
    snb = warp_sum(snb);
    // s >= 1 (its largest term is 1); snb > 0: mnb > -inf, and about mnb
    // its largest term is 1
    const float shift = mnb - m < -60.f ? mnb - m : 0.f;
    return shift + (logf(snb) - logf(s));
}

// log(1 - p_blank) from one 16-byte logit chunk per lane already in
// registers (rows 16-byte aligned, C a multiple of 8, C <= 256); the same
// arithmetic as frame_log_weight's first branch.
__device__ __forceinline__ float chunk_log_weight(const uint4 &q, int C, int lane)
{
    float v[8];
    chunk_vals(q, v);
    const bool has = 8 * lane < C;
    float m = -INFINITY, mnb = -INFINITY;
    if (has)
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            m = fmaxf(m, v[e]);
            if (lane > 0 || e > 0)
                mnb = fmaxf(mnb, v[e]);
        }
    m = warp_max(m);
    mnb = warp_max(mnb);
    if (mnb == -INFINITY)
        return -INFINITY;
    const bool far = mnb - m < -60.f;
    const float mr = far ? mnb : m;
    float s = 0.f, snb = 0.f;
    if (has)
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float x = exp2f((v[e] - m) * kLog2e);
            s += x;
            if (lane > 0 || e > 0)
                snb += far ? exp2f((v[e] - mr) * kLog2e) : x;
        }
    s = warp_sum(s);
    snb = warp_sum(snb);
    return (far ? mnb - m : 0.f) + (logf(snb) - logf(s));
}

constexpr int kPF = 2;   // frames of a window whose chunks are loaded up front
constexpr int kCG = 4;   // hidden chunks per lane per group (128 chunks = 1024 columns)

// One warp per window: the warp loads the first frames' hidden chunks and
// logit chunks together, forms the weights, then pools.  No CTA-wide
// barrier, so every warp keeps its own loads in flight.
__global__ void __launch_bounds__(kPoolThreads) posterior_pool_kernel(PoolParams p)
{
    extern __shared__ float s_lw_all[];   // [warps][P] log weights of each warp's window
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    float *s_lw = s_lw_all + warp * p.P;
    const int n_chunks = p.dim >> 3;
    const bool vec = (reinterpret_cast<uintptr_t>(p.logits) & 15) == 0 && (p.z_stride & 7) == 0 &&
                     (p.n_classes & 7) == 0;
    const bool zreg = vec && p.n_classes <= 256;
    PlanWalker w;
    w.init(p.cu, p.n_seq, p.total, p.P, lane);
    const long long stride = (long long)gridDim.x * kPoolWarps;
    for (long long g = (long long)blockIdx.x * kPoolWarps + warp;; g += stride) {
        int f0, L, seq;
        if (!w.find(g, lane, f0, L, seq))
            break;
        if (g >= p.n_rows) {
            // more windows than pooled rows: nothing past the buffer is written
            if (lane == 0)
                report(p.status, NLE_ERR_INVALID_ARG);
            break;
        }
        uint4 hv[kPF][kCG], zv[kPF];
#pragma unroll
        for (int t = 0; t < kPF; ++t) {
            if (t < L) {
                const __nv_bfloat16 *hrow = p.hidden + (long long)(f0 + t) * p.h_stride;
#pragma unroll
                for (int i = 0; i < kCG; ++i)
                    if (lane + 32 * i < n_chunks)
                        hv[t][i] = __ldcs(reinterpret_cast<const uint4 *>(hrow) + lane + 32 * i);
                if (zreg && 8 * lane < p.n_classes)
                    zv[t] = __ldcs(reinterpret_cast<const uint4 *>(p.logits + (long long)(f0 + t) * p.z_stride) +
                                   lane);
            }
        }
        float lw0 = -INFINITY;
        for (int t = 0; t < L; ++t) {
            float lw;
            if (zreg && t < kPF)
                lw = chunk_log_weight(t == 0 ? zv[0] : zv[kPF - 1], p.n_classes, lane);
            else
                lw = frame_log_weight(p.logits + (long long)(f0 + t) * p.z_stride, p.n_classes, vec, lane);
            lw0 = fmaxf(lw0, lw);
            if (lane == 0) {
                s_lw[t] = lw;
                if (p.weights)
                    p.weights[f0 + t] = expf(lw);
            }
        }
        __syncwarp();
        const float M = lw0;   // warp-uniform: every lane formed the same log weights
        __nv_bfloat16 *orow = p.pooled + g * (long long)p.dim;
        for (int cg = 0; 32 * kCG * cg < n_chunks; ++cg) {
#pragma unroll
            for (int i = 0; i < kCG; ++i) {
                const int ch = 32 * kCG * cg + lane + 32 * i;
                if (ch >= n_chunks)
                    continue;
                uint4 res = make_uint4(0u, 0u, 0u, 0u);
                if (M != -INFINITY) {
                    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                    float wsum = 0.f;
#pragma unroll
                    for (int t = 0; t < kPF; ++t) {
                        if (t < L) {
                            const float r = exp2f((s_lw[t] - M) * kLog2e);   // 0 for a weight of 0
                            const uint4 q = cg == 0 ? hv[t][i]
                                                    : __ldcs(reinterpret_cast<const uint4 *>(
                                                                 p.hidden + (long long)(f0 + t) * p.h_stride) +
                                                             ch);
                            float v[8];
                            chunk_vals(q, v);
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                acc[e] = fmaf(r, v[e], acc[e]);
                            wsum += r;
                        }
                    }
                    for (int t = kPF; t < L; ++t) {
                        const float r = exp2f((s_lw[t] - M) * kLog2e);
                        const uint4 q =
                            __ldcs(reinterpret_cast<const uint4 *>(p.hidden + (long long)(f0 + t) * p.h_stride) + ch);
                        float v[8];
                        chunk_vals(q, v);
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            acc[e] = fmaf(r, v[e], acc[e]);
                        wsum += r;
                    }
                    const float inv = 1.f / wsum;   // wsum >= 1: the largest weight contributes 1
                    res = make_uint4(pack_bf16x2(acc[0] * inv, acc[1] * inv), pack_bf16x2(acc[2] * inv, acc[3] * inv),
                                     pack_bf16x2(acc[4] * inv, acc[5] * inv), pack_bf16x2(acc[6] * inv, acc[7] * inv));
                }
                *reinterpret_cast<uint4 *>(orow + 8 * ch) = res;
            }
        }
        __syncwarp();   // s_lw is rewritten by the warp's next window
    }
    if (w.bad && lane == 0)
        report(p.status, NLE_ERR_INVALID_ARG);
}

// ---------------------------------------------------------------- pipelined path
// For the common shape (windows of at most kPipeMaxP frames, hidden width at
// most 1024, at most 256 logit classes read as 16-byte chunks) every warp
// keeps the next window's bytes in flight while it pools the current one:
// the frames' hidden rows and logits are copied into a per-warp
// shared-memory ring with cp.async (16 bytes per lane per copy), with no
// registers held for them, and the frames' weight reductions run
// interleaved.  The arithmetic is the one of posterior_pool_kernel.  Small
// per-warp rings keep up to 20 warps on an SM: the measured time fell from
// three windows in flight per warp (12 warps per SM) to two (16 warps), and
// rose with four (8 warps).
constexpr int kPipe = 2;       // windows in flight per warp
constexpr int kPipeMaxP = 2;   // frames per window on this path
constexpr uint32_t kPipeHdr = (kPipe * sizeof(int2) + 15) / 16 * 16;   // slot headers, padded to 16 bytes

// Shared memory of one warp on the pipelined path with NCH hidden chunks
// per lane: kPipe slots of kPipeMaxP frames, each frame NCH 512-byte rows
// of hidden chunks (chunk 32 i + lane at row i, column lane) and one of
// logit chunks, then the slots' headers.
template <int NCH>
__host__ __device__ constexpr uint32_t pipe_warp_bytes()
{
    return kPipe * kPipeMaxP * (NCH + 1) * 512 + kPipeHdr;
}

// (d.x, d.y) = (a.x b.x + c.x, a.y b.y + c.y): two fp32 FMAs in one packed
// instruction, each rounded as fmaf rounds it.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c)
{
    float2 d;
    asm("{.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\t"
        "mov.b64 rb, {%4, %5};\n\t"
        "mov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\t"
        "mov.b64 {%0, %1}, rd;}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// log(1 - p_blank) of frames t < L of a window (the others -inf), from one
// 16-byte logit chunk per lane and frame (C <= 256, a multiple of 8): the
// arithmetic of chunk_log_weight with the frames' warp reductions
// interleaved.  Each exponent is one FMA, z log2(e) - m log2(e), and one
// ex2; the shift's rounding multiplies every term of a frame's two sums by
// the same factor, which the ratio cancels.  The re-summation about the
// non-blank maximum (a blank that dominates by more than 60) is a
// warp-uniform branch of its own.
__device__ __forceinline__ void window_log_weights(const uint4 (&q)[kPipeMaxP], int C, int L, int lane,
                                                   float (&lw)[kPipeMaxP])
{
    const bool has = 8 * lane < C;
    float v[kPipeMaxP][8], m[kPipeMaxP], mnb[kPipeMaxP];
#pragma unroll
    for (int t = 0; t < kPipeMaxP; ++t) {
        chunk_vals(q[t], v[t]);
        m[t] = -INFINITY;
        mnb[t] = -INFINITY;
        if (has && t < L) {
            mnb[t] = fmax3(fmax3(v[t][1], v[t][2], v[t][3]), fmax3(v[t][4], v[t][5], v[t][6]), v[t][7]);
            m[t] = fmaxf(mnb[t], v[t][0]);
            if (lane > 0)
                mnb[t] = m[t];
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int t = 0; t < kPipeMaxP; ++t) {
            m[t] = fmaxf(m[t], __shfl_xor_sync(kFull, m[t], o));
            mnb[t] = fmaxf(mnb[t], __shfl_xor_sync(kFull, mnb[t], o));
        }
    float sm[kPipeMaxP], snb[kPipeMaxP];
    bool far = false;
#pragma unroll
    for (int t = 0; t < kPipeMaxP; ++t) {
        sm[t] = 0.f;
        snb[t] = 0.f;
        if (has && t < L && mnb[t] != -INFINITY) {
            const float ms = m[t] * kLog2e;
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
                x[e] = ex2_approx(fmaf(v[t][e], kLog2e, -ms));
            const float rest = ((x[1] + x[2]) + (x[3] + x[4])) + ((x[5] + x[6]) + x[7]);
            sm[t] = x[0] + rest;
            snb[t] = lane > 0 ? sm[t] : rest;
        }
        far |= t < L && mnb[t] != -INFINITY && mnb[t] - m[t] < -60.f;
    }
    if (far) {   // warp-uniform: m and mnb are the warp's
#pragma unroll
        for (int t = 0; t < kPipeMaxP; ++t)
            if (t < L && mnb[t] != -INFINITY && mnb[t] - m[t] < -60.f) {
                const float ms = mnb[t] * kLog2e;
                float acc = 0.f;
                if (has)
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        if (lane > 0 || e > 0)
                            acc += ex2_approx(fmaf(v[t][e], kLog2e, -ms));
                snb[t] = acc;
            }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int t = 0; t < kPipeMaxP; ++t) {
            sm[t] += __shfl_xor_sync(kFull, sm[t], o);
            snb[t] += __shfl_xor_sync(kFull, snb[t], o);
        }
#pragma unroll
    for (int t = 0; t < kPipeMaxP; ++t)
        lw[t] = (t < L && mnb[t] != -INFINITY)
                    ? (mnb[t] - m[t] < -60.f ? mnb[t] - m[t] : 0.f) + (logf(snb[t]) - logf(sm[t]))
                    : -INFINITY;
}

// NCH = ceil(dim / 256) hidden chunks per lane (dim <= 1024).  Every shared
// memory offset is a compile-time constant from the lane's column of the
// ring, every global one a constant from the lane's first chunk of a row.
template <int NCH>
__global__ void __launch_bounds__(kPoolThreads) posterior_pool_pipe_kernel(PoolParams p)
{
    constexpr uint32_t kFrame = (NCH + 1) * 512;   // one frame of a slot
    constexpr uint32_t kSlot = kPipeMaxP * kFrame;
    extern __shared__ __align__(16) uint8_t pool_smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint8_t *ring = pool_smem + (size_t)warp * pipe_warp_bytes<NCH>();
    int2 *hdr = reinterpret_cast<int2 *>(ring + kPipe * kSlot);
    uint8_t *col = ring + 16 * lane;   // this lane's 16-byte column
    const uint32_t col_s = smem_u32(col);
    const int n_chunks = p.dim >> 3;
    // bit i: this lane's chunk 32 i + lane exists
    const uint32_t hl = n_chunks >= 32 * NCH ? (1u << NCH) - 1u : (1u << ((n_chunks - lane + 31) >> 5)) - 1u;
    const bool zl = 8 * lane < p.n_classes;
    // windows gw, gw + stride, ...: at any moment the warps of the grid work
    // on neighbouring windows (DRAM pages shared), each keeping kPipe of its
    // own in flight
    const long long gw = (long long)blockIdx.x * kPoolWarps + warp;
    const long long stride = (long long)gridDim.x * kPoolWarps;
    if (gw >= p.n_rows)
        return;
    PlanWalker w;
    w.init(p.cu, p.n_seq, p.total, p.P, lane);
    long long next = gw;   // next window whose copies are issued
    bool more = true;
    // copies of window `next` into slot s (or an end mark), as one group
    auto issue = [&](int s) {
        int f0 = 0, L = -1, seq;
        if (more && next < p.n_rows && w.find(next, lane, f0, L, seq)) {
            const uint32_t dst = col_s + s * kSlot;
#pragma unroll
            for (int t = 0; t < kPipeMaxP; ++t) {
                if (t < L) {
                    const __nv_bfloat16 *hrow = p.hidden + (long long)(f0 + t) * p.h_stride + 8 * lane;
#pragma unroll
                    for (int i = 0; i < NCH; ++i)
                        if (hl >> i & 1u)
                            cp_async16(dst + t * kFrame + i * 512, hrow + 256 * i);
                    if (zl)
                        cp_async16(dst + t * kFrame + NCH * 512, p.logits + (long long)(f0 + t) * p.z_stride + 8 * lane);
                }
            }
        } else {
            more = false;
            L = -1;
        }
        if (lane == 0)
            hdr[s] = make_int2(f0, L);
        next += stride;
        cp_async_commit();
    };
    issue(0);
    long long last = -1;   // the last window this warp pooled
    int s = 0;
    for (long long g = gw; g < p.n_rows; g += stride, s ^= 1) {
        issue(s ^ 1);                     // this warp's next window, into the slot freed last pass
        cp_async_wait<kPipe - 1>();       // this lane's copies of window g have landed
        __syncwarp();
        const int2 hd = hdr[s];
        if (hd.y < 0)
            break;   // past the batch's last window
        const int f0 = hd.x, L = hd.y;
        last = g;
        const uint8_t *src = col + s * kSlot;
        uint4 zq[kPipeMaxP];
#pragma unroll
        for (int t = 0; t < kPipeMaxP; ++t) {
            zq[t] = make_uint4(0u, 0u, 0u, 0u);
            if (t < L && zl)
                zq[t] = *reinterpret_cast<const uint4 *>(src + t * kFrame + NCH * 512);
        }
        float lw[kPipeMaxP];
        window_log_weights(zq, p.n_classes, L, lane, lw);
        float M = -INFINITY;
#pragma unroll
        for (int t = 0; t < kPipeMaxP; ++t) {
            if (t < L) {
                M = fmaxf(M, lw[t]);
                if (lane == 0 && p.weights)
                    p.weights[f0 + t] = expf(lw[t]);
            }
        }
        float r[kPipeMaxP];
        float wsum = 0.f;
#pragma unroll
        for (int t = 0; t < kPipeMaxP; ++t) {
            r[t] = (t < L && M != -INFINITY) ? exp2f((lw[t] - M) * kLog2e) : 0.f;   // 0 for a weight of 0
            wsum += r[t];
        }
        // wsum >= 1 when some weight is not 0; the frames' weights are
        // normalised before the FMAs
        const float inv = M != -INFINITY ? 1.f / wsum : 0.f;
#pragma unroll
        for (int t = 0; t < kPipeMaxP; ++t)
            r[t] *= inv;
        __nv_bfloat16 *orow = p.pooled + g * (long long)p.dim + 8 * lane;
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
            if (!(hl >> i & 1u))
                continue;
            float2 acc[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
            for (int t = 0; t < kPipeMaxP; ++t) {
                if (t < L && M != -INFINITY) {   // every weight 0: a zero row, whatever the frames hold
                    float v[8];
                    chunk_vals(*reinterpret_cast<const uint4 *>(src + t * kFrame + i * 512), v);
                    const float2 rr = make_float2(r[t], r[t]);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        acc[e] = ffma2(make_float2(v[2 * e], v[2 * e + 1]), rr, acc[e]);
                }
            }
            const uint4 res = make_uint4(pack_bf16x2(acc[0].x, acc[0].y), pack_bf16x2(acc[1].x, acc[1].y),
                                         pack_bf16x2(acc[2].x, acc[2].y), pack_bf16x2(acc[3].x, acc[3].y));
            __stcs(reinterpret_cast<uint4 *>(orow + 256 * i), res);
        }
        __syncwarp();   // slot s is refilled by the next pass
    }
    cp_async_wait<0>();
    // the warp that pooled row n_rows - 1 checks that the batch has no
    // further window (more windows than rows: nothing past the buffer is
    // written, the shortfall is reported)
    if (last == p.n_rows - 1) {
        int a, b, c;
        if (w.find(p.n_rows, lane, a, b, c) && lane == 0)
            report(p.status, NLE_ERR_INVALID_ARG);
    }
    if (w.bad && lane == 0)
        report(p.status, NLE_ERR_INVALID_ARG);
}

template <int NCH>
int launch_pool_pipe(const PoolParams &p, const nle::DeviceInfo &di, int dev, cudaStream_t stream)
{
    constexpr size_t smem_cta = (size_t)kPoolWarps * pipe_warp_bytes<NCH>();
    int per_sm = (int)((size_t)di.smem_optin / (smem_cta + 1024));
    per_sm = per_sm < 1 ? 1 : (per_sm > 6 ? 6 : per_sm);
    long long warps = (long long)di.sm_count * per_sm * kPoolWarps;
    if (warps > p.n_rows)
        warps = p.n_rows;
    const long long ctas = (warps + kPoolWarps - 1) / kPoolWarps;
    if (smem_cta > 48 * 1024 &&
        !nle::allow_max_dynamic_smem(reinterpret_cast<const void *>(posterior_pool_pipe_kernel<NCH>), dev,
                                     di.smem_optin))
        return NLE_ERR_CUDA;
    posterior_pool_pipe_kernel<NCH><<<(int)ctas, kPoolThreads, smem_cta, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? NLE_OK : NLE_ERR_CUDA;
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
    // a warp per window; 4 CTAs of 128 threads fit an SM at 128 registers
    const long long ctas = (n_pooled_rows + kPoolWarps - 1) / kPoolWarps, cap = (long long)di.sm_count * 4;
    const int grid = (int)(ctas < cap ? ctas : cap);
    const bool vec = (reinterpret_cast<uintptr_t>(logits) & 15) == 0 && logits_stride % 8 == 0 && n_classes % 8 == 0;
    if (vec && n_classes <= 256 && dim <= 1024 && pool_frames <= kPipeMaxP) {
        const cudaStream_t st = static_cast<cudaStream_t>(stream);
        switch ((dim / 8 + 31) / 32) {
        case 1: return launch_pool_pipe<1>(p, di, dev, st);
        case 2: return launch_pool_pipe<2>(p, di, dev, st);
        case 3: return launch_pool_pipe<3>(p, di, dev, st);
        default: return launch_pool_pipe<4>(p, di, dev, st);
        }
    }
    // per-warp log weights of a window: above 48 KB (pool_frames > 3072)
    // the kernel needs the opt-in shared memory limit
    const size_t smem = sizeof(float) * kPoolWarps * (size_t)pool_frames;
    if (smem > 48 * 1024 &&
        !nle::allow_max_dynamic_smem(reinterpret_cast<const void *>(posterior_pool_kernel), dev, di.smem_optin))
        return NLE_ERR_CUDA;
    posterior_pool_kernel<<<grid, kPoolThreads, smem, static_cast<cudaStream_t>(stream)>>>(p);
    return cudaGetLastError() == cudaSuccess ? NLE_OK : NLE_ERR_CUDA;
}
