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
// The work is HBM-bound (about 2.5 flop per byte), so it runs on the CUDA
// cores.  One persistent CTA per SM (8 warps) walks windows g = blockIdx.x,
// blockIdx.x + gridDim.x, ...; the K rows, V rows and Q rows of a window are
// each one contiguous range of memory ([frames][heads][64] layout), fetched
// with a single bulk copy apiece into a ring of shared-memory stages.
// Per window, each warp takes a pair of heads: in QK^T one lane per key
// (half a warp per head, the 16-byte chunks of a key row visited in a
// lane-rotated order so the shared-memory reads do not collide), softmax
// by shuffles inside the half-warp, then PV with one lane per two output
// dimensions and coalesced 4-byte bf16x2 stores.
#include <cmath>

#include "nle.h"
#include "nle_device.cuh"
#include "nle_host.h"

namespace {

using namespace nle;

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxStages = 3;
constexpr int kMaxQw = 8;

struct WBars {
    uint64_t full[kMaxStages];
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
    const __nv_bfloat16 *q, *k, *v;
    __nv_bfloat16 *out;
    int stages;
    uint32_t kv_bytes;    // K (or V) region of a stage: W * heads * 128
    uint32_t q_bytes;     // Q region: Qw * heads * 128
    uint32_t stage_bytes;
    uint32_t qf_off;      // fp32 copy of the current window's queries
    uint32_t bars_off;
    float scale_log2;
    int32_t *status;
    unsigned long long wait_ns;
    int flags;
};

__device__ __forceinline__ void unpack8(const uint4 &x, float (&f)[8])
{
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

// KPL = lanes per head group: 16 (two heads per warp, W <= 16) or 32.
// QW = queries per window.
template <int KPL, int QW>
__global__ void __launch_bounds__(kThreads, 1) window_xattn_kernel(const WParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    WBars *bars = reinterpret_cast<WBars *>(smem + p.bars_off);
    float *qf = reinterpret_cast<float *>(smem + p.qf_off);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int H = p.heads;
    const long long row_elems = (long long)H * 64;

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s)
            mbar_init(smem_u32(&bars->full[s]), 1);
        bars->abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    volatile int *abort_flag = &bars->abort_flag;

    // ------------------------------------------------ producer (warp 0)
    PlanWalker pw;
    uint64_t pol = 0;
    long long issued = 0;      // windows issued so far (local index)
    bool prod_done = false;
    if (warp == 0) {
        pw.init(p.cu, p.n_seq, p.total, p.W, lane);
        pol = policy_evict_first();
    }
    auto issue = [&](long long n) {
        const long long g = blockIdx.x + n * (long long)gridDim.x;
        int f0, L, seq;
        if (!pw.find(g, lane, f0, L, seq)) {
            prod_done = true;
            return;
        }
        if (lane == 0 && !((p.flags & NLE_FLAG_TEST_SKIP_FIRST_LOAD) && n == 0)) {
            const int s = (int)(n % p.stages);
            const uint32_t bar = smem_u32(&bars->full[s]);
            const uint32_t dst = smem_u32(smem + s * p.stage_bytes);
            if ((long long)p.Qw * (g + 1) > p.n_qrows) {
                mbar_arrive(bar);   // no data: consumers skip this window
            } else {
                const uint32_t kvb = (uint32_t)L * H * 128u;
                mbar_arrive_expect_tx(bar, 2 * kvb + p.q_bytes);
                bulk_load(dst, p.k + (long long)f0 * row_elems, kvb, bar, pol);
                bulk_load(dst + p.kv_bytes, p.v + (long long)f0 * row_elems, kvb, bar, pol);
                bulk_load(dst + 2 * p.kv_bytes, p.q + (long long)p.Qw * g * row_elems, p.q_bytes, bar, pol);
            }
        }
        __syncwarp();
        issued = n + 1;
    };
    if (warp == 0)
        for (long long n = 0; n < p.stages - 1 && !prod_done; ++n)
            issue(n);

    // ------------------------------------------------ consumers (all warps)
    PlanWalker cw;
    cw.init(p.cu, p.n_seq, p.total, p.W, lane);
    const float sl2 = p.scale_log2;
    long long n = 0;
    for (;; ++n) {
        if (warp == 0 && !prod_done)
            issue(n + p.stages - 1);
        const long long g = blockIdx.x + n * (long long)gridDim.x;
        int f0, L, seq;
        if (!cw.find(g, lane, f0, L, seq))
            break;
        const int s = (int)(n % p.stages);
        const bool ok = wait_bar(smem_u32(&bars->full[s]), (uint32_t)(n / p.stages) & 1, abort_flag, p.wait_ns,
                                 p.status);
        if (__syncthreads_or(!ok))
            break;
        const bool q_ok = (long long)p.Qw * (g + 1) <= p.n_qrows;
        const uint8_t *st = smem + s * p.stage_bytes;
        if (q_ok) {
            // queries of this window -> fp32 (read many times below)
            const uint4 *qs = reinterpret_cast<const uint4 *>(st + 2 * p.kv_bytes);
            const int chunks = p.Qw * H * 8;
            for (int i = threadIdx.x; i < chunks; i += kThreads) {
                float f[8];
                unpack8(qs[i], f);
                float4 *d = reinterpret_cast<float4 *>(qf + i * 8);
                d[0] = make_float4(f[0], f[1], f[2], f[3]);
                d[1] = make_float4(f[4], f[5], f[6], f[7]);
            }
        }
        __syncthreads();
        if (q_ok) {
            const uint8_t *ks = st;
            const uint8_t *vs = st + p.kv_bytes;
            constexpr int HPG = 32 / KPL;          // heads per warp pass
            const int sub = lane / KPL;
            const int j = lane % KPL;               // key handled in QK^T
            for (int pair = warp; pair * HPG < H; pair += kWarps) {
                const int head = pair * HPG + sub;
                const bool kv_ok = head < H && j < L;
                float sc[QW];
#pragma unroll
                for (int r = 0; r < QW; ++r)
                    sc[r] = 0.f;
                if (kv_ok) {
                    const uint4 *krow = reinterpret_cast<const uint4 *>(ks + ((size_t)j * H + head) * 128);
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const int cc = (c + j) & 7;
                        float kf[8];
                        unpack8(krow[cc], kf);
#pragma unroll
                        for (int r = 0; r < QW; ++r) {
                            {
                                const float4 *qp = reinterpret_cast<const float4 *>(qf + ((size_t)(r * H + head) * 64 + cc * 8));
                                const float4 a = qp[0], b = qp[1];
                                sc[r] = fmaf(a.x, kf[0], sc[r]);
                                sc[r] = fmaf(a.y, kf[1], sc[r]);
                                sc[r] = fmaf(a.z, kf[2], sc[r]);
                                sc[r] = fmaf(a.w, kf[3], sc[r]);
                                sc[r] = fmaf(b.x, kf[4], sc[r]);
                                sc[r] = fmaf(b.y, kf[5], sc[r]);
                                sc[r] = fmaf(b.z, kf[6], sc[r]);
                                sc[r] = fmaf(b.w, kf[7], sc[r]);
                            }
                        }
                    }
                }
                // softmax over the keys of this head group (fp32, exp2)
#pragma unroll
                for (int r = 0; r < QW; ++r) {
                    {
                        const float x = kv_ok ? sc[r] * sl2 : -INFINITY;
                        float m = x;
#pragma unroll
                        for (int o = KPL / 2; o >= 1; o >>= 1)
                            m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
                        const float e = kv_ok ? ex2_approx(x - m) : 0.f;
                        float sum = e;
#pragma unroll
                        for (int o = KPL / 2; o >= 1; o >>= 1)
                            sum += __shfl_xor_sync(kFull, sum, o);
                        sc[r] = kv_ok ? e / sum : 0.f;
                    }
                }
                // PV: lane owns output dims 2*lane, 2*lane+1
#pragma unroll
                for (int hs = 0; hs < HPG; ++hs) {
                    const int hh = pair * HPG + hs;
                    if (hh >= H)
                        break;
                    float o[QW][2];
#pragma unroll
                    for (int r = 0; r < QW; ++r)
                        o[r][0] = o[r][1] = 0.f;
                    for (int jj = 0; jj < L; ++jj) {
                        const uint32_t vv =
                            *reinterpret_cast<const uint32_t *>(vs + ((size_t)jj * H + hh) * 128 + lane * 4);
                        const float v0 = __uint_as_float(vv << 16), v1 = __uint_as_float(vv & 0xffff0000u);
#pragma unroll
                        for (int r = 0; r < QW; ++r) {
                            {
                                const float pr = __shfl_sync(kFull, sc[r], hs * KPL + jj);
                                o[r][0] = fmaf(pr, v0, o[r][0]);
                                o[r][1] = fmaf(pr, v1, o[r][1]);
                            }
                        }
                    }
#pragma unroll
                    for (int r = 0; r < QW; ++r) {
                        {
                            __nv_bfloat16 *dst = p.out + ((long long)p.Qw * g + r) * row_elems + hh * 64 + 2 * lane;
                            *reinterpret_cast<uint32_t *>(dst) = pack_bf16x2(o[r][0], o[r][1]);
                        }
                    }
                }
            }
        } else if (threadIdx.x == 0) {
            report(p.status, NLE_ERR_INVALID_ARG);
        }
        __syncthreads();
    }
    if (warp == 0) {
        if (cw.bad && lane == 0)
            report(p.status, NLE_ERR_INVALID_ARG);
        // drain copies issued but not consumed (only after an abort)
        if (lane == 0)
            for (long long m = n; m < issued; ++m)
                if (!((p.flags & NLE_FLAG_TEST_SKIP_FIRST_LOAD) && m == 0))
                    wait_bar_drain(smem_u32(&bars->full[m % p.stages]), (uint32_t)(m / p.stages) & 1, p.wait_ns);
        __syncwarp();
    }
    __syncthreads();
}

using WKernel = void (*)(const WParams);

template <int KPL>
WKernel pick_qw(int qw)
{
    switch (qw) {
    case 1: return window_xattn_kernel<KPL, 1>;
    case 2: return window_xattn_kernel<KPL, 2>;
    case 3: return window_xattn_kernel<KPL, 3>;
    case 4: return window_xattn_kernel<KPL, 4>;
    case 5: return window_xattn_kernel<KPL, 5>;
    case 6: return window_xattn_kernel<KPL, 6>;
    case 7: return window_xattn_kernel<KPL, 7>;
    default: return window_xattn_kernel<KPL, 8>;
    }
}

int g_smem_set[2][kMaxQw + 1][64] = {};

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

    WParams p{};
    p.cu = cu_seqlens_kv;
    p.n_seq = n_seq;
    p.total = (int)total_frames;
    p.n_qrows = n_query_rows;
    p.heads = heads;
    p.W = window_frames;
    p.Qw = queries_per_window;
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.k = static_cast<const __nv_bfloat16 *>(k);
    p.v = static_cast<const __nv_bfloat16 *>(v);
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.kv_bytes = (uint32_t)window_frames * heads * 128u;
    p.q_bytes = (uint32_t)queries_per_window * heads * 128u;
    p.stage_bytes = (2 * p.kv_bytes + p.q_bytes + 127) / 128 * 128;
    const size_t qf_bytes = (size_t)queries_per_window * heads * 64 * 4;
    const size_t fixed = qf_bytes + ((sizeof(WBars) + 127) / 128) * 128 + 128;
    if ((size_t)heads * 128u * (2 * window_frames + queries_per_window) > (size_t)di.smem_optin)
        return NLE_ERR_UNSUPPORTED;
    int stages = (int)(((size_t)di.smem_optin - fixed) / p.stage_bytes);
    if (stages > kMaxStages)
        stages = kMaxStages;
    if (stages < 2)
        return NLE_ERR_UNSUPPORTED;
    p.stages = stages;
    p.qf_off = stages * p.stage_bytes;
    p.bars_off = p.qf_off + (uint32_t)((qf_bytes + 127) / 128 * 128);
    const size_t smem = (size_t)p.bars_off + ((sizeof(WBars) + 127) / 128) * 128 + 128;
    const double scale = softmax_scale > 0.f ? (double)softmax_scale : 1.0 / std::sqrt((double)d_head);
    p.scale_log2 = (float)(scale * 1.4426950408889634);
    p.status = dev_status;
    p.wait_ns = wait_limit_ns > 0 ? (unsigned long long)wait_limit_ns : 1000000000ull;
    p.flags = flags;

    const bool half = window_frames <= 16;
    WKernel kern = half ? pick_qw<16>(queries_per_window) : pick_qw<32>(queries_per_window);
    int &set = g_smem_set[half][queries_per_window][dev < 64 ? dev : 0];
    if (dev >= 64 || set < (int)smem) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
            return NLE_ERR_CUDA;
        set = (int)smem;
    }
    const long long max_windows = (long long)n_seq + total_frames / window_frames;
    const int grid = (int)(max_windows < di.sm_count ? max_windows : di.sm_count);
    kern<<<grid, kThreads, smem, static_cast<cudaStream_t>(stream)>>>(p);
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
