// window_xattn_sm100a.cu -- windowed cross-attention of the Q-Former
// projector on B200 (sm_100a).
//
// Operation (granite-speech-4.1-2b-nar model card, "Model Architecture" (2)
// Q-Former Projector: each 15-frame window is reduced to 3 queries via
// cross-attention): window g of the packed batch covers frames
// [start, start + L) of one utterance (L <= window_frames, the last window of
// an utterance may be partial) and owns query rows Qw*g .. Qw*g + Qw - 1;
// each query row attends to the window's L frames, per head.
//
// The work is HBM-bound (about 2.5 flop per byte).  One persistent CTA per
// SM walks windows g = blockIdx.x, blockIdx.x + gridDim.x, ...:
//   warp 16     producer: per window three 128-byte-swizzled TMA boxes (no
//               multicast) into a ring of shared-memory stages: K and V of
//               all heads (16 frames per 16-key group) and the window's Qw
//               query rows of all heads, each through a 3-D tensor map
//               ordered (d, row, head) so that every head's rows land
//               together.
//   warps 0-15  one head each (heads h = warp, warp + 16, ...): the window's
//               S = Q K^T (at most 16 queries x 16 keys) and O = P V are
//               warp-level mma.sync m16n8k16 products (bf16 in, fp32
//               accumulate) fed by ldmatrix from the swizzled tiles; softmax
//               in fp32 with quad shuffles (keys >= L are 0 by index); P is
//               reused from the accumulator registers as the A fragment of
//               PV.  O is divided by the row sum, rounded to bf16 and written
//               as coalesced 128-byte rows.
// The tensor cores are used here only because the window's two products
// are dense contractions that map onto one warp; the kernel's bound is HBM.
#include <cmath>

#include "nle.h"
#include "nle_device.cuh"
#include "nle_host.h"

namespace {

using namespace nle;

constexpr int kComputeWarps = 16;
constexpr int kThreads = (kComputeWarps + 1) * 32;
constexpr int kMaxStages = 4;
constexpr int kMaxQw = 16;
constexpr int kTileBytes = 2048;   // 16 rows x 128 B, one head's keys (or values) per 16-key group
constexpr int kOStride = 144;      // output staging row: 128 B + 16 B so fragment stores hit distinct banks

struct WBars {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];    // kComputeWarps arrivals
    int abort_flag;
};

struct WParams {
    const int32_t *cu;
    int n_seq;
    int total;
    long long n_qrows;
    int heads;
    int W;        // window_frames
    int Qw;       // queries_per_window
    const __nv_bfloat16 *q;
    __nv_bfloat16 *out;
    int stages;
    uint32_t kv_bytes;    // K (or V) region of a stage: KT * heads * 2048, [kt][head]
    uint32_t q_bytes;     // Q rows of a window: heads * Qw * 128, [head][query]
    uint32_t stage_bytes;
    uint32_t ostage_off;  // per-warp output staging (Qw rows of kOStride bytes)
    uint32_t bars_off;
    float scale_log2;
    int32_t *status;
    unsigned long long wait_ns;
    int flags;
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr)
                 : "memory");
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr)
                 : "memory");
}

// D = A * B + D, m16n8k16, bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
                 "{%8, %9}, {%0, %1, %2, %3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Byte offset of (row, 16-byte chunk) in a 128-byte-swizzled tile whose
// base is 1024-byte aligned.
__device__ __forceinline__ uint32_t swz(int row, int chunk) { return row * 128 + ((chunk ^ (row & 7)) << 4); }

// KT = number of 16-key groups (window_frames <= 16 * KT).
template <int KT>
__global__ void __launch_bounds__(kThreads, 1)
    window_xattn_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_q, const WParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    WBars *bars = reinterpret_cast<WBars *>(smem + p.bars_off);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int H = p.heads;
    const long long row_elems = (long long)H * 64;

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(smem_u32(&bars->full[s]), 1);
            mbar_init(smem_u32(&bars->empty[s]), kComputeWarps);
        }
        bars->abort_flag = 0;
        fence_mbar_init();
    }
    if (threadIdx.x == 32) {
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_q);
    }
    __syncthreads();
    volatile int *abort_flag = &bars->abort_flag;
    const unsigned long long wait_ns = p.wait_ns;

    if (warp == kComputeWarps) {
        // ======================================================== producer
        PlanWalker w;
        w.init(p.cu, p.n_seq, p.total, p.W, lane);
        const uint64_t pol = policy_evict_first();
        int n = 0;
        for (;; ++n) {
            const long long g = blockIdx.x + (long long)n * gridDim.x;
            int f0, L, seq;
            if (!w.find(g, lane, f0, L, seq))
                break;
            const int s = n % p.stages;
            const uint32_t u = (uint32_t)(n / p.stages);
            if (u > 0 && !wait_bar(smem_u32(&bars->empty[s]), (u - 1) & 1, abort_flag, wait_ns, p.status))
                break;
            if (lane == 0 && !((p.flags & NLE_FLAG_TEST_SKIP_FIRST_LOAD) && n == 0)) {
                const uint32_t bar = smem_u32(&bars->full[s]);
                const uint32_t st = smem_u32(smem + s * p.stage_bytes);
                if ((long long)p.Qw * (g + 1) > p.n_qrows) {
                    mbar_arrive(bar);   // no query rows: consumers skip this window
                } else {
                    mbar_arrive_expect_tx(bar, 2u * p.kv_bytes + p.q_bytes);
                    // 16 frames of every head per 16-key group (frames past
                    // the window are masked, and zeroed in V, below)
                    for (int kt = 0; kt < KT; ++kt) {
                        tma_load_3d(st + kt * H * kTileBytes, &tm_k, 0, f0 + 16 * kt, 0, bar, pol);
                        tma_load_3d(st + p.kv_bytes + kt * H * kTileBytes, &tm_v, 0, f0 + 16 * kt, 0, bar, pol);
                    }
                    tma_load_3d(st + 2 * p.kv_bytes, &tm_q, 0, (int32_t)(p.Qw * g), 0, bar, pol);
                }
            }
            __syncwarp();
        }
        if (w.bad && lane == 0)
            report(p.status, NLE_ERR_INVALID_ARG);
        // drain: the last copy into each stage must land before exit
        if (lane == 0) {
            const bool skipped0 = (p.flags & NLE_FLAG_TEST_SKIP_FIRST_LOAD) != 0;
            for (int m = n - p.stages; m < n; ++m)
                if (m >= 0 && !(skipped0 && m == 0))
                    wait_bar_drain(smem_u32(&bars->full[m % p.stages]), (uint32_t)(m / p.stages) & 1, wait_ns);
        }
        __syncwarp();
    } else {
        // ======================================================== heads
        PlanWalker w;
        w.init(p.cu, p.n_seq, p.total, p.W, lane);
        const float sl2 = p.scale_log2;
        const int gq = lane >> 2;       // fragment row group (query)
        const int tq = lane & 3;        // thread in group
        uint8_t *ost = smem + p.ostage_off + warp * p.Qw * kOStride;
        for (int n = 0;; ++n) {
            const long long g = blockIdx.x + (long long)n * gridDim.x;
            int f0, L, seq;
            if (!w.find(g, lane, f0, L, seq))
                break;
            const int s = n % p.stages;
            if (!wait_bar(smem_u32(&bars->full[s]), (uint32_t)(n / p.stages) & 1, abort_flag, wait_ns, p.status))
                break;
            const bool q_ok = (long long)p.Qw * (g + 1) <= p.n_qrows;
            uint8_t *st = smem + s * p.stage_bytes;
            const uint32_t kbase = smem_u32(st), vbase = kbase + p.kv_bytes, qbase = kbase + 2 * p.kv_bytes;
            for (int h = warp; q_ok && h < H; h += kComputeWarps) {
                // ---- S = Q K^T: A = queries (rows >= Qw repeat query rows),
                // B = keys of this head (n-tiles of 8 keys)
                float sacc[2 * KT][4];
#pragma unroll
                for (int j = 0; j < 2 * KT; ++j)
                    sacc[j][0] = sacc[j][1] = sacc[j][2] = sacc[j][3] = 0.f;
                const int arow = (lane & 7) + ((lane >> 3) & 1) * 8;   // row this lane addresses in ldmatrix
                const int qline = h * p.Qw + arow % p.Qw;               // its 128-byte line in the Q tile
                const uint32_t qrow = qbase + (uint32_t)(qline * 128);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    uint32_t a[4];
                    ldsm_x4(qrow + (((2 * ks + (lane >> 4)) ^ (qline & 7)) << 4), a[0], a[1], a[2], a[3]);
#pragma unroll
                    for (int kt = 0; kt < KT; ++kt) {
                        // matrices: (keys 0-7, dims lo), (keys 0-7, dims hi),
                        // (keys 8-15, dims lo), (keys 8-15, dims hi)
                        const int krow = (lane & 7) + (lane >> 4) * 8;
                        const int kchunk = 2 * ks + ((lane >> 3) & 1);
                        uint32_t b0, b1, b2, b3;
                        ldsm_x4(kbase + (kt * H + h) * kTileBytes + swz(krow, kchunk), b0, b1, b2, b3);
                        mma_16816(sacc[2 * kt], a, b0, b1);
                        mma_16816(sacc[2 * kt + 1], a, b2, b3);
                    }
                }
                // ---- softmax over the keys of each query row (quad = row)
                float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
                for (int j = 0; j < 2 * KT; ++j) {
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int key = 8 * j + 2 * tq + e;
                        if (key >= L) {
                            sacc[j][e] = -INFINITY;
                            sacc[j][2 + e] = -INFINITY;
                        }
                        mx0 = fmaxf(mx0, sacc[j][e]);
                        mx1 = fmaxf(mx1, sacc[j][2 + e]);
                    }
                }
                mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, 1));
                mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, 2));
                mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, 1));
                mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, 2));
                const float m0 = mx0 * sl2, m1 = mx1 * sl2;
                float l0 = 0.f, l1 = 0.f;
                uint32_t pa[KT][4];   // P as the A fragment of PV, per 16-key group
#pragma unroll
                for (int kt = 0; kt < KT; ++kt) {
                    float pv[2][4];
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj) {
                        const int j = 2 * kt + jj;
                        pv[jj][0] = ex2_approx(fmaf(sacc[j][0], sl2, -m0));
                        pv[jj][1] = ex2_approx(fmaf(sacc[j][1], sl2, -m0));
                        pv[jj][2] = ex2_approx(fmaf(sacc[j][2], sl2, -m1));
                        pv[jj][3] = ex2_approx(fmaf(sacc[j][3], sl2, -m1));
                        l0 += pv[jj][0] + pv[jj][1];
                        l1 += pv[jj][2] + pv[jj][3];
                    }
                    pa[kt][0] = pack_bf16x2(pv[0][0], pv[0][1]);   // row g,   keys 2t..
                    pa[kt][1] = pack_bf16x2(pv[0][2], pv[0][3]);   // row g+8, keys 2t..
                    pa[kt][2] = pack_bf16x2(pv[1][0], pv[1][1]);   // row g,   keys 8+2t..
                    pa[kt][3] = pack_bf16x2(pv[1][2], pv[1][3]);   // row g+8, keys 8+2t..
                }
                l0 += __shfl_xor_sync(kFull, l0, 1);
                l0 += __shfl_xor_sync(kFull, l0, 2);
                l1 += __shfl_xor_sync(kFull, l1, 1);
                l1 += __shfl_xor_sync(kFull, l1, 2);
                // ---- value rows L..16*KT-1 hold frames past the window (the
                // next window's, or another utterance's); zero them so
                // nothing outside the window reaches PV (P is 0 there, but
                // 0 * Inf would be NaN)
                for (int i = lane; i < (16 * KT - L) * 8; i += 32) {
                    const int r = L + i / 8, c = i % 8;
                    const int kt = r >> 4;
                    *reinterpret_cast<uint4 *>(st + p.kv_bytes + (kt * H + h) * kTileBytes + swz(r & 15, c)) =
                        make_uint4(0, 0, 0, 0);
                }
                __syncwarp();
                // ---- O = P V: B = values via transposing ldmatrix
                float oacc[8][4];
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    oacc[j][0] = oacc[j][1] = oacc[j][2] = oacc[j][3] = 0.f;
#pragma unroll
                for (int kt = 0; kt < KT; ++kt) {
#pragma unroll
                    for (int jp = 0; jp < 4; ++jp) {
                        // matrices: (keys 0-7, dims 16jp..), (keys 8-15, dims 16jp..),
                        // (keys 0-7, dims 16jp+8..), (keys 8-15, dims 16jp+8..)
                        const int vrow = (lane & 7) + ((lane >> 3) & 1) * 8;
                        const int vchunk = 2 * jp + (lane >> 4);
                        uint32_t b0, b1, b2, b3;
                        ldsm_x4_t(vbase + (kt * H + h) * kTileBytes + swz(vrow, vchunk), b0, b1, b2, b3);
                        mma_16816(oacc[2 * jp], pa[kt], b0, b1);
                        mma_16816(oacc[2 * jp + 1], pa[kt], b2, b3);
                    }
                }
                // ---- normalise, stage the Qw rows of this head, write them
                // as coalesced 128-byte rows
                const float inv0 = 1.f / l0;
                if (gq < p.Qw) {
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        *reinterpret_cast<uint32_t *>(ost + gq * kOStride + j * 16 + tq * 4) =
                            pack_bf16x2(oacc[j][0] * inv0, oacc[j][1] * inv0);
                }
                if (gq + 8 < p.Qw) {
                    const float inv1 = 1.f / l1;
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        *reinterpret_cast<uint32_t *>(ost + (gq + 8) * kOStride + j * 16 + tq * 4) =
                            pack_bf16x2(oacc[j][2] * inv1, oacc[j][3] * inv1);
                }
                __syncwarp();
                for (int r = 0; r < p.Qw; ++r) {
                    const uint32_t v = *reinterpret_cast<const uint32_t *>(ost + r * kOStride + lane * 4);
                    *reinterpret_cast<uint32_t *>(p.out + ((long long)p.Qw * g + r) * row_elems + h * 64 + 2 * lane) = v;
                }
                __syncwarp();
            }
            if (!q_ok && warp == 0 && lane == 0)
                report(p.status, NLE_ERR_INVALID_ARG);
            // generic writes (zeroed rows) before the stage is refilled by TMA
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_u32(&bars->empty[s]));
        }
        if (w.bad && warp == 0 && lane == 0)
            report(p.status, NLE_ERR_INVALID_ARG);
    }
    __syncthreads();
}

using WKernel = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, WParams);

} // namespace

extern "C" int nle_window_xattn_fwd_ex(const void *q, const void *k, const void *v, void *out,
                                       const int32_t *cu_seqlens_kv, int n_seq, int64_t total_frames,
                                       int64_t n_query_rows, int heads, int d_head, int window_frames,
                                       int queries_per_window, float softmax_scale, int32_t *dev_status, int flags,
                                       int64_t wait_limit_ns, void *stream)
{
    if (n_seq < 0 || total_frames < 0 || n_query_rows < 0 || heads <= 0 || window_frames <= 0 ||
        queries_per_window <= 0 || wait_limit_ns < 0)
        return NLE_ERR_INVALID_ARG;
    if (d_head != 64 || window_frames > 32 || queries_per_window > kMaxQw || total_frames > 0x7fffffffLL ||
        n_query_rows > 0x7fffffffLL)
        return NLE_ERR_UNSUPPORTED;
    if (n_seq == 0 || total_frames == 0)
        return NLE_OK;
    if (!q || !k || !v || !out || !cu_seqlens_kv)
        return NLE_ERR_INVALID_ARG;
    if (!nle::aligned16(q) || !nle::aligned16(k) || !nle::aligned16(v) || !nle::aligned16(out))
        return NLE_ERR_MISALIGNED;

    nle::DeviceInfo di;
    int dev = 0;
    if (!nle::current_device_info(&di, &dev))
        return NLE_ERR_CUDA;
    if (di.cc_major != 10)
        return NLE_ERR_UNSUPPORTED;

    const int KT = window_frames <= 16 ? 1 : 2;
    WParams p{};
    p.cu = cu_seqlens_kv;
    p.n_seq = n_seq;
    p.total = (int)total_frames;
    p.n_qrows = n_query_rows;
    p.heads = heads;
    p.W = window_frames;
    p.Qw = queries_per_window;
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.kv_bytes = (uint32_t)heads * KT * kTileBytes;
    p.q_bytes = (uint32_t)queries_per_window * heads * 128u;
    p.stage_bytes = (2 * p.kv_bytes + p.q_bytes + 1023) / 1024 * 1024;
    const size_t ostage = (size_t)kComputeWarps * queries_per_window * kOStride;
    const size_t fixed = ostage + ((sizeof(WBars) + 127) / 128) * 128 + 1024;
    if ((size_t)di.smem_optin < fixed + 2 * (size_t)p.stage_bytes)
        return NLE_ERR_UNSUPPORTED;
    int stages = (int)(((size_t)di.smem_optin - fixed) / p.stage_bytes);
    if (stages > kMaxStages)
        stages = kMaxStages;
    p.stages = stages;
    p.ostage_off = stages * p.stage_bytes;
    p.bars_off = p.ostage_off + (uint32_t)ostage;
    const size_t smem = (size_t)p.bars_off + ((sizeof(WBars) + 127) / 128) * 128 + 1024;
    const double scale = softmax_scale > 0.f ? (double)softmax_scale : 1.0 / std::sqrt((double)d_head);
    p.scale_log2 = (float)(scale * 1.4426950408889634);
    p.status = dev_status;
    p.wait_ns = wait_limit_ns > 0 ? (unsigned long long)wait_limit_ns : 1000000000ull;
    p.flags = flags;

    // Tensor maps over [rows][heads][64] bf16 as (d, row, head): K/V boxes of
    // 16 frames x all heads, Q boxes of Qw rows x all heads; 128-byte
    // swizzle, zero fill past the end.  (A query tensor too short for some
    // window is reported by the kernel, which then loads no query rows for
    // that window.)
    CUtensorMap tk, tv, tq;
    const uint64_t hd = (uint64_t)heads;
    const uint64_t qrows = n_query_rows > 0 ? (uint64_t)n_query_rows : 1;
    if (!nle::encode_tmap_bf16_heads(&tk, k, (uint64_t)total_frames, hd, hd * 64, 16, (uint32_t)heads) ||
        !nle::encode_tmap_bf16_heads(&tv, v, (uint64_t)total_frames, hd, hd * 64, 16, (uint32_t)heads) ||
        !nle::encode_tmap_bf16_heads(&tq, q, qrows, hd, hd * 64, (uint32_t)queries_per_window, (uint32_t)heads))
        return NLE_ERR_CUDA;

    WKernel kern = KT == 1 ? window_xattn_kernel<1> : window_xattn_kernel<2>;
    if (!nle::allow_max_dynamic_smem(reinterpret_cast<const void *>(kern), dev, di.smem_optin))
        return NLE_ERR_CUDA;
    const long long max_windows = (long long)n_seq + total_frames / window_frames;
    const int grid = (int)(max_windows < di.sm_count ? max_windows : di.sm_count);
    kern<<<grid, kThreads, smem, static_cast<cudaStream_t>(stream)>>>(tk, tv, tq, p);
    return cudaGetLastError() == cudaSuccess ? NLE_OK : NLE_ERR_CUDA;
}

extern "C" int nle_window_xattn_fwd(const void *q, const void *k, const void *v, void *out,
                                    const int32_t *cu_seqlens_kv, int n_seq, int64_t total_frames,
                                    int64_t n_query_rows, int heads, int d_head, int window_frames,
                                    int queries_per_window, void *stream)
{
    return nle_window_xattn_fwd_ex(q, k, v, out, cu_seqlens_kv, n_seq, total_frames, n_query_rows, heads, d_head,
                                   window_frames, queries_per_window, 0.f, nullptr, 0, 0, stream);
}
