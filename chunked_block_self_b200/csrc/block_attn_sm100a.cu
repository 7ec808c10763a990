// block_attn_sm100a.cu -- varlen block (chunked) bidirectional
// self-attention on B200 (sm_100a).
//
// Operation (granite-speech-4.1-2b-nar model card, "Model Architecture" (1)
// CTC Speech Encoder: block attention over 4 s blocks = 200 encoder frames
// at 50 Hz; "Usage / Installation": packed sequences, is_causal=False):
// for every block of every packed utterance and every head,
//     O = softmax(scale * Q K^T) V  over the block's L <= B frames.
//
// Design (one persistent CTA per SM, 10 warps):
//   warp 0      TMA producer.  Work item = (block, head).  Q (two boxes:
//               rows 0..127 and 128..B-1), K and V of the item are loaded
//               with 128-byte-swizzled TMA boxes (no multicast) into a ring
//               of QK stages and a ring of two V stages; V lags QK by one
//               item so Q/K run up to (stages) items ahead.
//   warp 1      TMEM owner and MMA issuer (one elected lane):
//                 S_t = Q_t K^T   tcgen05.mma kind::f16, M=128, N=NB (B
//                                 rounded up to 16), K=64 in 4 steps
//                 O_t = P_t V     A operand = P in TMEM, B = V (N-major) in
//                                 smem, M=128, N=64, K=NB in NB/16 steps
//               t = 0 covers block rows 0..127, t = 1 rows 128..B-1.
//   warps 2-5   softmax + epilogue of tile 0; warps 6-9 of tile 1.  Each
//               thread owns one block row (its TMEM lane): pass 1 reads S and
//               takes the row max over the L valid keys; pass 2 forms
//               p = exp2(S*scale*log2e - max*scale*log2e) in fp32, sums it,
//               packs it to bf16 and writes it back into S's TMEM columns as
//               the A operand of PV.  The epilogue reads O, divides by the
//               row sum, rounds to bf16 and stores only rows < L with 16-byte
//               vector stores.
// TMEM (512 columns): tile slot t at column 256*t holds S (NB columns), then
// P (NB/2 columns, over S) and O (64 columns at +128).
//
// Masking and locality: keys >= L get p = 0 by index (never by value); V
// rows L..B-1 of a partial block are zeroed in shared memory before PV, and
// rows B..NB-1 of every V stage are zero, so no value outside the block can
// reach an output, even a NaN or Inf.  Query rows >= L are computed but
// never stored.
//
// Every mbarrier wait is bounded (see nle_device.cuh); on expiry the CTA
// drains its copies and MMAs in flight, frees TMEM and returns.
#include <cmath>

#include "nle.h"
#include "nle_device.cuh"
#include "nle_host.h"

namespace {

using namespace nle;

constexpr int kThreads = 320;
constexpr int kQTile = 128;        // MMA M (rows per tile)
constexpr int kRowBytes = 128;     // one frame of one head: 64 bf16
constexpr int kMaxQK = 4;          // QK ring depth upper bound
constexpr int kSV = 2;             // V ring depth
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSlotCols = 256; // TMEM columns per tile slot
constexpr uint32_t kOCol = 128;     // O offset inside a tile slot

struct Bars {
    uint64_t qk_full[kMaxQK];
    uint64_t qk_empty[kMaxQK];
    uint64_t v_full[kSV];
    uint64_t v_empty[kSV];
    uint64_t s_full[2];
    uint64_t p_full[2];
    uint64_t o_full[2];
    uint64_t tmem_free[2];
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort_flag;
};

struct Params {
    const int32_t *cu;
    int n_seq;
    int total;
    int heads;
    int B;        // block_frames
    int NB;       // B rounded up to 16 (MMA N of S, K extent of PV)
    int q0rows;   // rows of the first Q box (min(B, 128))
    int q1rows;   // rows of the second Q box (B - 128, or 0)
    int sqk;      // QK ring depth
    uint32_t q_bytes;   // Q region of a QK stage
    uint32_t qk_bytes;  // QK stage
    uint32_t v_bytes;   // V stage
    float scale_log2;
    __nv_bfloat16 *out;
    int out_stride;     // elements between output frames (heads * 64)
    int32_t *status;
    unsigned long long wait_ns;
    int flags;
};

__global__ void __launch_bounds__(kThreads, 1)
    block_attn_kernel(const __grid_constant__ CUtensorMap tm_q0, const __grid_constant__ CUtensorMap tm_q1,
                      const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      const Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t qk_base = smem_u32(smem);
    const uint32_t v_off = p.sqk * p.qk_bytes;
    const uint32_t v_base = qk_base + v_off;
    Bars *bars = reinterpret_cast<Bars *>(smem + v_off + kSV * p.v_bytes);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // ------------------------------------------------------------ set-up
    if (threadIdx.x == 0) {
        for (int s = 0; s < p.sqk; ++s) {
            mbar_init(smem_u32(&bars->qk_full[s]), 1);
            mbar_init(smem_u32(&bars->qk_empty[s]), 1);
        }
        for (int s = 0; s < kSV; ++s) {
            mbar_init(smem_u32(&bars->v_full[s]), 1);
            mbar_init(smem_u32(&bars->v_empty[s]), 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(smem_u32(&bars->s_full[t]), 1);
            mbar_init(smem_u32(&bars->p_full[t]), 4);
            mbar_init(smem_u32(&bars->o_full[t]), 1);
            mbar_init(smem_u32(&bars->tmem_free[t]), 4);
        }
        mbar_init(smem_u32(&bars->mma_done), 1);
        bars->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&bars->tmem_base), kTmemCols);
        tmem_relinquish();
    }
    if (threadIdx.x == 32 * 2) {
        tma_prefetch_desc(&tm_q0);
        tma_prefetch_desc(&tm_q1);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    // V rows B..NB-1 (MMA padding) are zero for the whole launch.
    {
        const int pad_chunks = (p.NB - p.B) * (kRowBytes / 16);
        for (int i = threadIdx.x; i < kSV * pad_chunks; i += kThreads) {
            const int s = i / pad_chunks, c = i - s * pad_chunks;
            reinterpret_cast<uint4 *>(smem + v_off + s * p.v_bytes + p.B * kRowBytes)[c] = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    volatile int *abort_flag = &bars->abort_flag;
    const unsigned long long wait_ns = p.wait_ns;

    if (warp == 0) {
        // ======================================================== producer
        PlanWalker w;
        w.init(p.cu, p.n_seq, p.total, p.B, lane);
        const uint64_t pol = policy_evict_first();
        uint32_t qk_issued[kMaxQK] = {0, 0, 0, 0};
        uint32_t v_issued[kSV] = {0, 0};
        int prev_h = 0, prev_f0 = 0;
        long long n = 0;
        bool ok = true;

        auto issue_v = [&](long long m, int h, int f0) -> bool {
            const int sv = (int)(m % kSV);
            const uint32_t uv = (uint32_t)(m / kSV);
            if (uv > 0 && !wait_bar(smem_u32(&bars->v_empty[sv]), (uv - 1) & 1, abort_flag, wait_ns, p.status))
                return false;
            if (lane == 0) {
                const uint32_t bar = smem_u32(&bars->v_full[sv]);
                mbar_arrive_expect_tx(bar, p.B * kRowBytes);
                tma_load_2d(v_base + sv * p.v_bytes, &tm_v, h * 64, f0, bar, pol);
                ++v_issued[sv];
            }
            __syncwarp();
            return true;
        };

        for (long long item = blockIdx.x;; item += gridDim.x, ++n) {
            const long long b = item / p.heads;
            const int h = (int)(item - b * p.heads);
            int f0, L, seq;
            if (!w.find(b, lane, f0, L, seq))
                break;
            const int s = (int)(n % p.sqk);
            const uint32_t u = (uint32_t)(n / p.sqk);
            if (u > 0 &&
                !wait_bar(smem_u32(&bars->qk_empty[s]), (u - 1) & 1, abort_flag, wait_ns, p.status)) {
                ok = false;
                break;
            }
            if (lane == 0 && !((p.flags & NLE_FLAG_TEST_SKIP_FIRST_LOAD) && n == 0)) {
                const bool two = L > kQTile;
                const uint32_t bar = smem_u32(&bars->qk_full[s]);
                const uint32_t bytes = (p.q0rows + (two ? p.q1rows : 0) + p.B) * kRowBytes;
                const uint32_t qdst = qk_base + s * p.qk_bytes;
                mbar_arrive_expect_tx(bar, bytes);
                tma_load_2d(qdst, &tm_q0, h * 64, f0, bar, pol);
                if (two)
                    tma_load_2d(qdst + kQTile * kRowBytes, &tm_q1, h * 64, f0 + kQTile, bar, pol);
                tma_load_2d(qdst + p.q_bytes, &tm_k, h * 64, f0, bar, pol);
                ++qk_issued[s];
            }
            __syncwarp();
            if (n > 0 && !issue_v(n - 1, prev_h, prev_f0)) {
                ok = false;
                break;
            }
            prev_h = h;
            prev_f0 = f0;
        }
        if (ok && n > 0)
            issue_v(n - 1, prev_h, prev_f0);
        if (w.bad && lane == 0)
            report(p.status, NLE_ERR_INVALID_ARG);
        // drain: every issued copy must land before the CTA can exit
        if (lane == 0) {
            for (int s = 0; s < p.sqk; ++s)
                if (qk_issued[s])
                    wait_bar_drain(smem_u32(&bars->qk_full[s]), (qk_issued[s] - 1) & 1, wait_ns);
            for (int s = 0; s < kSV; ++s)
                if (v_issued[s])
                    wait_bar_drain(smem_u32(&bars->v_full[s]), (v_issued[s] - 1) & 1, wait_ns);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ======================================================== MMA issuer
        PlanWalker w;
        w.init(p.cu, p.n_seq, p.total, p.B, lane);
        const uint32_t id_s = idesc_bf16_f32(128, p.NB, false);
        const uint32_t id_pv = idesc_bf16_f32(128, 64, true);
        uint32_t tile_uses[2] = {0, 0};
        long long n = 0;
        for (long long item = blockIdx.x;; item += gridDim.x, ++n) {
            const long long b = item / p.heads;
            int f0, L, seq;
            if (!w.find(b, lane, f0, L, seq))
                break;
            const int s = (int)(n % p.sqk);
            if (!wait_bar(smem_u32(&bars->qk_full[s]), (uint32_t)(n / p.sqk) & 1, abort_flag, wait_ns, p.status))
                break;
            tc_fence_after();
            const int ntiles = L > kQTile ? 2 : 1;
            const uint32_t qaddr = qk_base + s * p.qk_bytes;
            const uint32_t kaddr = qaddr + p.q_bytes;
            bool ok = true;
            for (int t = 0; t < ntiles; ++t) {
                const uint32_t ut = tile_uses[t];
                if (ut > 0 &&
                    !wait_bar(smem_u32(&bars->tmem_free[t]), (ut - 1) & 1, abort_flag, wait_ns, p.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t da = smem_desc_sw128(qaddr + t * kQTile * kRowBytes + kk * 32, 16, 1024);
                        const uint64_t db = smem_desc_sw128(kaddr + kk * 32, 16, 1024);
                        mma_ss(tmem + t * kSlotCols, da, db, id_s, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(smem_u32(&bars->s_full[t]));
                }
                __syncwarp();
            }
            if (!ok)
                break;
            if (lane == 0)
                mma_commit(smem_u32(&bars->qk_empty[s]));
            __syncwarp();
            const int sv = (int)(n % kSV);
            if (!wait_bar(smem_u32(&bars->v_full[sv]), (uint32_t)(n / kSV) & 1, abort_flag, wait_ns, p.status))
                break;
            tc_fence_after();
            const uint32_t vaddr = v_base + sv * p.v_bytes;
            for (int t = 0; t < ntiles; ++t) {
                const uint32_t ut = tile_uses[t];
                if (!wait_bar(smem_u32(&bars->p_full[t]), ut & 1, abort_flag, wait_ns, p.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t slot = tmem + t * kSlotCols;
                    for (int kk = 0; kk < p.NB / 16; ++kk) {
                        // N = 64 is one 128-byte swizzle atom along N, so
                        // the N-direction atom stride (LBO) is never used.
                        const uint64_t db = smem_desc_sw128(vaddr + kk * 16 * kRowBytes, 0, 1024);
                        mma_ts(slot + kOCol, slot + kk * 8, db, id_pv, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(smem_u32(&bars->o_full[t]));
                }
                __syncwarp();
                tile_uses[t] = ut + 1;
            }
            if (!ok)
                break;
            if (lane == 0)
                mma_commit(smem_u32(&bars->v_empty[sv]));
            __syncwarp();
        }
        // every MMA issued so far must finish before TMEM is released
        if (lane == 0) {
            mma_commit(smem_u32(&bars->mma_done));
            wait_bar_drain(smem_u32(&bars->mma_done), 0, wait_ns);
        }
        __syncwarp();
    } else {
        // ======================================================== softmax + epilogue
        const int t = (warp - 2) >> 2;             // tile slot
        const int qq = warp & 3;                   // TMEM lane quarter of this warp
        const uint32_t tS = tmem + ((uint32_t)(qq * 32) << 16) + t * kSlotCols;
        const float sl2 = p.scale_log2;
        PlanWalker w;
        w.init(p.cu, p.n_seq, p.total, p.B, lane);
        uint32_t uses = 0;
        long long n = 0;
        for (long long item = blockIdx.x;; item += gridDim.x, ++n) {
            const long long b = item / p.heads;
            const int h = (int)(item - b * p.heads);
            int f0, L, seq;
            if (!w.find(b, lane, f0, L, seq))
                break;
            if (t == 1 && L <= kQTile)
                continue;
            if (!wait_bar(smem_u32(&bars->s_full[t]), uses & 1, abort_flag, wait_ns, p.status))
                break;
            tc_fence_after();
            const int row0 = t * kQTile + qq * 32;   // first block row of this warp
            const bool active = row0 < L;
            float l = 0.f;
            if (active) {
                // pass 1: row max over the L valid keys
                float m = -INFINITY;
                for (int c0 = 0; c0 < p.NB; c0 += 32) {
                    if (c0 + 32 <= p.NB) {
                        uint32_t r[32];
                        tmem_ld32_sync(tS + c0, r);
                        if (c0 + 32 <= L) {
#pragma unroll
                            for (int j = 0; j < 32; ++j)
                                m = fmaxf(m, __uint_as_float(r[j]));
                        } else {
#pragma unroll
                            for (int j = 0; j < 32; ++j)
                                if (c0 + j < L)
                                    m = fmaxf(m, __uint_as_float(r[j]));
                        }
                    } else {
                        uint32_t r[16];
                        tmem_ld16_sync(tS + c0, r);
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            if (c0 + j < L)
                                m = fmaxf(m, __uint_as_float(r[j]));
                    }
                }
                const float mc = m * sl2;
                // pass 2: p = exp2(s*scale*log2e - m*scale*log2e), bf16 P over S
                for (int c0 = 0; c0 < p.NB; c0 += 32) {
                    if (c0 + 32 <= p.NB) {
                        uint32_t r[32], pk[16];
                        tmem_ld32_sync(tS + c0, r);
                        if (c0 + 32 <= L) {
#pragma unroll
                            for (int j = 0; j < 16; ++j) {
                                const float a = ex2_approx(fmaf(__uint_as_float(r[2 * j]), sl2, -mc));
                                const float c = ex2_approx(fmaf(__uint_as_float(r[2 * j + 1]), sl2, -mc));
                                l += a + c;
                                pk[j] = pack_bf16x2(a, c);
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < 16; ++j) {
                                const float a = (c0 + 2 * j < L)
                                                    ? ex2_approx(fmaf(__uint_as_float(r[2 * j]), sl2, -mc))
                                                    : 0.f;
                                const float c = (c0 + 2 * j + 1 < L)
                                                    ? ex2_approx(fmaf(__uint_as_float(r[2 * j + 1]), sl2, -mc))
                                                    : 0.f;
                                l += a + c;
                                pk[j] = pack_bf16x2(a, c);
                            }
                        }
                        tmem_st16(tS + c0 / 2, pk);
                    } else {
                        uint32_t r[16], pk[8];
                        tmem_ld16_sync(tS + c0, r);
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const float a = (c0 + 2 * j < L)
                                                ? ex2_approx(fmaf(__uint_as_float(r[2 * j]), sl2, -mc))
                                                : 0.f;
                            const float c = (c0 + 2 * j + 1 < L)
                                                ? ex2_approx(fmaf(__uint_as_float(r[2 * j + 1]), sl2, -mc))
                                                : 0.f;
                            l += a + c;
                            pk[j] = pack_bf16x2(a, c);
                        }
                        tmem_st8(tS + c0 / 2, pk);
                    }
                }
                tmem_wait_st();
            }
            if (t == 0 && L < p.B) {
                // partial block: zero V rows L..B-1 so nothing outside the
                // block reaches PV (P is 0 there, and 0 * Inf would be NaN)
                const int sv = (int)(n % kSV);
                if (!wait_bar(smem_u32(&bars->v_full[sv]), (uint32_t)(n / kSV) & 1, abort_flag, wait_ns,
                              p.status))
                    break;
                uint4 *vz = reinterpret_cast<uint4 *>(smem + v_off + sv * p.v_bytes + L * kRowBytes);
                const int chunks = (p.B - L) * (kRowBytes / 16);
                for (int i = (warp - 2) * 32 + lane; i < chunks; i += 128)
                    vz[i] = make_uint4(0, 0, 0, 0);
                fence_proxy_async_smem();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_u32(&bars->p_full[t]));
            if (!wait_bar(smem_u32(&bars->o_full[t]), uses & 1, abort_flag, wait_ns, p.status))
                break;
            tc_fence_after();
            uint32_t o0[32], o1[32];
            if (active) {
                tmem_ld32_sync(tS + kOCol, o0);
                tmem_ld32_sync(tS + kOCol + 32, o1);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_u32(&bars->tmem_free[t]));
            const int r = row0 + lane;
            if (active && r < L) {
                const float inv = 1.f / l;
                uint4 *dst = reinterpret_cast<uint4 *>(p.out + (size_t)(f0 + r) * p.out_stride + h * 64);
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    dst[c] = make_uint4(pack_bf16x2(__uint_as_float(o0[8 * c + 0]) * inv, __uint_as_float(o0[8 * c + 1]) * inv),
                                        pack_bf16x2(__uint_as_float(o0[8 * c + 2]) * inv, __uint_as_float(o0[8 * c + 3]) * inv),
                                        pack_bf16x2(__uint_as_float(o0[8 * c + 4]) * inv, __uint_as_float(o0[8 * c + 5]) * inv),
                                        pack_bf16x2(__uint_as_float(o0[8 * c + 6]) * inv, __uint_as_float(o0[8 * c + 7]) * inv));
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    dst[4 + c] = make_uint4(pack_bf16x2(__uint_as_float(o1[8 * c + 0]) * inv, __uint_as_float(o1[8 * c + 1]) * inv),
                                            pack_bf16x2(__uint_as_float(o1[8 * c + 2]) * inv, __uint_as_float(o1[8 * c + 3]) * inv),
                                            pack_bf16x2(__uint_as_float(o1[8 * c + 4]) * inv, __uint_as_float(o1[8 * c + 5]) * inv),
                                            pack_bf16x2(__uint_as_float(o1[8 * c + 6]) * inv, __uint_as_float(o1[8 * c + 7]) * inv));
            }
            ++uses;
        }
        tmem_wait_st();
    }

    // ------------------------------------------------------------ teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

int g_smem_set[64] = {};   // dynamic smem already opted in, per device

} // namespace

extern "C" int nle_block_attn_fwd_ex(const void *q, const void *k, const void *v, void *out,
                                     const int32_t *cu_seqlens, int n_seq, int64_t total_frames, int heads,
                                     int d_head, int block_frames, float softmax_scale, int64_t row_stride_qkv,
                                     int32_t *dev_status, int flags, int64_t wait_limit_ns, void *stream)
{
    if (n_seq < 0 || total_frames < 0 || heads <= 0 || block_frames <= 0 || wait_limit_ns < 0)
        return NLE_ERR_INVALID_ARG;
    if (d_head != 64 || block_frames > 256 || total_frames > 0x7fffffffLL)
        return NLE_ERR_UNSUPPORTED;
    if (n_seq == 0 || total_frames == 0)
        return NLE_OK;
    if (!q || !k || !v || !out || !cu_seqlens)
        return NLE_ERR_INVALID_ARG;
    const int64_t dense = (int64_t)heads * 64;
    const int64_t stride = row_stride_qkv ? row_stride_qkv : dense;
    if (stride < dense || dense > 0x7fffffffLL)
        return NLE_ERR_INVALID_ARG;
    if (stride % 8 != 0 || !nle::aligned16(q) || !nle::aligned16(k) || !nle::aligned16(v) ||
        !nle::aligned16(out))
        return NLE_ERR_MISALIGNED;

    nle::DeviceInfo di;
    int dev = 0;
    if (!nle::current_device_info(&di, &dev))
        return NLE_ERR_CUDA;
    if (di.cc_major != 10)
        return NLE_ERR_UNSUPPORTED;

    const int B = block_frames;
    const int NB = (B + 15) / 16 * 16;
    const int rows8 = (B + 7) / 8 * 8;
    Params p{};
    p.cu = cu_seqlens;
    p.n_seq = n_seq;
    p.total = (int)total_frames;
    p.heads = heads;
    p.B = B;
    p.NB = NB;
    p.q0rows = B < kQTile ? B : kQTile;
    p.q1rows = B > kQTile ? B - kQTile : 0;
    // The M=128 MMAs read 128 rows from each tile's base: keep >= 128 rows of
    // Q per stage (tile 1 over-reads into the K region, which follows).
    p.q_bytes = (uint32_t)((rows8 > kQTile ? rows8 : kQTile) * kRowBytes);
    p.qk_bytes = p.q_bytes + (uint32_t)(rows8 * kRowBytes);
    p.v_bytes = (uint32_t)(NB * kRowBytes);
    const size_t fixed = (size_t)kSV * p.v_bytes + ((sizeof(Bars) + 127) / 128) * 128 + 1024;
    int sqk = (int)(((size_t)di.smem_optin - fixed) / p.qk_bytes);
    if (sqk > kMaxQK)
        sqk = kMaxQK;
    if (sqk < 2)
        return NLE_ERR_UNSUPPORTED;
    p.sqk = sqk;
    size_t smem = (size_t)sqk * p.qk_bytes + fixed;
    // One CTA per SM: it owns all 512 TMEM columns, so a second resident CTA
    // would only wait in tcgen05.alloc.  Ask for more than half the SM's
    // shared memory to rule that out.
    if (smem <= (size_t)di.smem_optin / 2)
        smem = (size_t)di.smem_optin / 2 + 1024;
    const double scale = softmax_scale > 0.f ? (double)softmax_scale : 1.0 / std::sqrt((double)d_head);
    p.scale_log2 = (float)(scale * 1.4426950408889634);
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.out_stride = (int)dense;
    p.status = dev_status;
    p.wait_ns = wait_limit_ns > 0 ? (unsigned long long)wait_limit_ns : 1000000000ull;
    p.flags = flags;

    CUtensorMap tq0, tq1, tk, tv;
    const uint64_t cols = (uint64_t)dense, rows = (uint64_t)total_frames;
    if (!nle::encode_tmap_bf16_2d(&tq0, q, cols, rows, stride, 64, p.q0rows) ||
        !nle::encode_tmap_bf16_2d(&tq1, q, cols, rows, stride, 64, p.q1rows ? p.q1rows : p.q0rows) ||
        !nle::encode_tmap_bf16_2d(&tk, k, cols, rows, stride, 64, B) ||
        !nle::encode_tmap_bf16_2d(&tv, v, cols, rows, stride, 64, B))
        return NLE_ERR_CUDA;

    if (dev < 64 && g_smem_set[dev] < (int)smem) {
        if (cudaFuncSetAttribute(block_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return NLE_ERR_CUDA;
        g_smem_set[dev] = (int)smem;
    }
    // upper bound on work items: each utterance has at most T/B + 1 blocks
    const long long max_items = ((long long)n_seq + total_frames / B) * heads;
    const int grid = (int)(max_items < di.sm_count ? max_items : di.sm_count);
    block_attn_kernel<<<grid, kThreads, smem, static_cast<cudaStream_t>(stream)>>>(tq0, tq1, tk, tv, p);
    return cudaGetLastError() == cudaSuccess ? NLE_OK : NLE_ERR_CUDA;
}

extern "C" int nle_block_attn_fwd(const void *q, const void *k, const void *v, void *out, const int32_t *cu_seqlens,
                                  int n_seq, int64_t total_frames, int heads, int d_head, int block_frames,
                                  void *stream)
{
    return nle_block_attn_fwd_ex(q, k, v, out, cu_seqlens, n_seq, total_frames, heads, d_head, block_frames, 0.f,
                                 0, nullptr, 0, 0, stream);
}
