// block_attn_sm100a.cu -- varlen block (chunked) bidirectional
// self-attention on B200 (sm_100a).
//
// Operation (granite-speech-4.1-2b-nar model card, "Model Architecture" (1)
// CTC Speech Encoder: block attention over 4 s blocks = 200 encoder frames
// at 50 Hz; "Usage / Installation": packed sequences, is_causal=False):
// for every block of every packed utterance and every head,
//     O = softmax(scale * Q K^T) V  over the block's L <= B frames.
//
// Design (one persistent CTA per SM, three warpgroups):
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
//               Before PV of a partial block it zeroes V rows L..ceil16(L)-1
//               in shared memory (frames outside the block; P is 0 there,
//               but 0 * Inf would be NaN).
//   warps 2-3   idle (they complete warpgroup 0 for setmaxnreg).
//   warps 4-7   softmax + epilogue of tile 0; warps 8-11 of tile 1.  Each
//               thread owns one block row (its TMEM lane) and reads S in
//               register segments of up to 112 columns: segment max, p =
//               exp2(S*scale*log2e - m) in fp32 with an integer running max m
//               (keys >= L are 0 by index, never by value), row sum, bf16
//               pack, P written back over S.  The epilogue reads O, divides by
//               the row sum, rounds to bf16 and stores only rows < L with
//               16-byte vector stores.
// The MMAs of an item stop at ceil16(L) keys, so a partial block costs only
// its own keys.
// TMEM (512 columns): tile slot t at column 256*t holds S (NB columns), then
// P (NB/2 columns, over S) and O (64 columns at +128).
//
// Every mbarrier wait is bounded (see nle_device.cuh); on expiry the CTA
// drains its copies and MMAs in flight, frees TMEM and returns.
#include <cmath>

#include "nle.h"
#include "nle_device.cuh"
#include "nle_host.h"

namespace {

using namespace nle;

// Wide blocks (NB >= 176, the pages' 200-frame blocks among them) run three
// warpgroups with a setmaxnreg split: warpgroup 0 (producer, MMA, two idle
// warps) gives registers to the two softmax warpgroups, whose threads then
// hold 112-column segments of S.  128 x 56 + 256 x 224 equals the launch
// allocation 384 x 168; the host refuses to launch a build whose per-thread
// count differs (a larger request would wait forever).  Narrower blocks run
// ten warps without the split and 64-column segments.
constexpr int kSplitMinNB = 176;
constexpr int kRegsLaunch = 168;
constexpr int kRegsLow = 56;
constexpr int kRegsHigh = 224;
static_assert(128 * kRegsLow + 256 * kRegsHigh == 384 * kRegsLaunch, "register split must match launch");

template <int NB>
struct Shape {
    static constexpr bool split = NB >= kSplitMinNB;
    static constexpr int threads = split ? 384 : 320;
    static constexpr int first_softmax_warp = split ? 4 : 2;
    static constexpr int seg = split ? 112 : 64;
};
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

// Softmax of one TMEM lane quarter of a tile (32 rows, one per lane).
//
// S is read from TMEM in register segments of at most kSeg columns (a
// multiple of 16, so each segment's P covers whole PV K-steps).  The running
// maximum is kept as an integer m in the log2 domain (x = s * scale * log2e,
// m = ceil(max x)), so p = exp2(x - m) <= 1 for the segment that set m.  A
// later segment whose own max exceeds m by at most kSlack keeps m (its p
// may reach 2^kSlack, harmless in fp32 / bf16); otherwise m moves up and the
// P already written is rescaled by 2^(m_old - m_new), an exact power of two.
// The result is the same softmax: every p of a row shares one m.
constexpr float kSlack = 8.f;

template <int W>
__device__ __forceinline__ void seg_load(uint32_t taddr, uint32_t (&s)[W])
{
#pragma unroll
    for (int c = 0; c + 32 <= W; c += 32)
        tmem_ld32_nowait(taddr + c, &s[c]);
    if constexpr (W % 32 == 16)
        tmem_ld16_nowait(taddr + W - 16, &s[W - 16]);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < W; ++i)
        reg_fence(s[i]);
}

template <int W>
__device__ __forceinline__ void seg_store(uint32_t taddr, const uint32_t (&pk)[W / 2])
{
#pragma unroll
    for (int c = 0; c + 32 <= W / 2; c += 32)
        tmem_st32(taddr + c, &pk[c]);
    if constexpr ((W / 2) % 32 >= 16)
        tmem_st16p(taddr + (W / 2) / 32 * 32, &pk[(W / 2) / 32 * 32]);
    if constexpr ((W / 2) % 16 == 8)
        tmem_st8p(taddr + W / 2 - 8, &pk[W / 2 - 8]);
}

// Masks keys >= L (by index) to -inf and returns the segment's max.
template <int W>
__device__ __forceinline__ float seg_mask_max(uint32_t (&s)[W], int c0, int L)
{
#pragma unroll
    for (int g = 0; g < W / 8; ++g) {
        if (c0 + 8 * g + 8 > L) {   // warp-uniform
#pragma unroll
            for (int e = 0; e < 8; ++e)
                if (c0 + 8 * g + e >= L)
                    s[8 * g + e] = __float_as_uint(-INFINITY);
        }
    }
    float mx[8];
#pragma unroll
    for (int e = 0; e < 8; ++e)
        mx[e] = __uint_as_float(s[e]);
#pragma unroll
    for (int i = 8; i < W; ++i)
        mx[i & 7] = fmaxf(mx[i & 7], __uint_as_float(s[i]));
    return fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
}

// p = exp2(s * sl2 - m) for keys < L (0 beyond), summed into l, packed to
// bf16 pairs.
template <int W>
__device__ __forceinline__ void seg_exp(const uint32_t (&s)[W], uint32_t (&pk)[W / 2], int c0, int L, float sl2,
                                        float m, float &l)
{
    float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int g = 0; g < W / 8; ++g) {
        if (c0 + 8 * g < L) {   // warp-uniform; masked keys hold -inf -> 0
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float a = ex2_approx(fmaf(__uint_as_float(s[8 * g + 2 * e]), sl2, -m));
                const float b = ex2_approx(fmaf(__uint_as_float(s[8 * g + 2 * e + 1]), sl2, -m));
                ls[e] += a + b;
                pk[4 * g + e] = pack_bf16x2(a, b);
            }
        } else {
#pragma unroll
            for (int e = 0; e < 4; ++e)
                pk[4 * g + e] = 0u;
        }
    }
    l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
}

// Multiply the bf16 P already in TMEM columns [0, ncols) by f, a power of
// two <= 1 (exact up to underflow); lanes with f = 1 rewrite P unchanged.
// Rare path; must be entered by the whole warp.
__device__ __noinline__ void rescale_p(uint32_t tS, int ncols, float f)
{
    tmem_wait_st();
    for (int c = 0; c < ncols; c += 8) {
        uint32_t r[8];
        tmem_ld8_nowait(tS + c, r);
        tmem_wait_ld();
        uint32_t o[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            reg_fence(r[i]);
            const float a = __uint_as_float(r[i] << 16) * f;
            const float b = __uint_as_float(r[i] & 0xffff0000u) * f;
            o[i] = pack_bf16x2(a, b);
        }
        tmem_st8p(tS + c, o);
        tmem_wait_st();
    }
}

template <int C0, int W>
__device__ __forceinline__ void softmax_segment(uint32_t tS, int L, float sl2, float &m, float &l)
{
    uint32_t s[W];
    seg_load<W>(tS + C0, s);
    const float mk = ceilf(seg_mask_max<W>(s, C0, L) * sl2);
    float f = 1.f;                      // rescale of the earlier segments
    if (C0 == 0) {
        m = mk;
    } else if (mk > m + kSlack) {
        // 2^(m - mk) built from its exponent (m, mk are integers); below the
        // normal range the old terms are negligible and drop to 0
        const int e = (int)(m - mk);
        f = e >= -126 ? __int_as_float((127 + e) << 23) : 0.f;
        l *= f;
        m = mk;
    }
    uint32_t pk[W / 2];
    seg_exp<W>(s, pk, C0, L, sl2, m, l);
    seg_store<W>(tS + C0 / 2, pk);
    if (__any_sync(kFull, f != 1.f))    // after the store: few live registers
        rescale_p(tS, C0 / 2, f);
}

// Returns this lane's row sum; P (bf16) is left over the first NB/2 columns
// of S.  Segments wholly at or past L are skipped (the MMAs stop at
// ceil16(L) keys).
template <int NB, int SEG>
__device__ __forceinline__ float softmax_rows(uint32_t tS, int L, float sl2)
{
    static_assert(SEG % 16 == 0 && NB <= 4 * SEG, "segments");
    float m = 0.f, l = 0.f;
    constexpr int W0 = NB < SEG ? NB : SEG;
    softmax_segment<0, W0>(tS, L, sl2, m, l);
    if constexpr (NB > SEG) {
        constexpr int W1 = NB - SEG < SEG ? NB - SEG : SEG;
        if (L > SEG)
            softmax_segment<SEG, W1>(tS, L, sl2, m, l);
    }
    if constexpr (NB > 2 * SEG) {
        constexpr int W2 = NB - 2 * SEG < SEG ? NB - 2 * SEG : SEG;
        if (L > 2 * SEG)
            softmax_segment<2 * SEG, W2>(tS, L, sl2, m, l);
    }
    if constexpr (NB > 3 * SEG) {
        constexpr int W3 = NB - 3 * SEG;
        if (L > 3 * SEG)
            softmax_segment<3 * SEG, W3>(tS, L, sl2, m, l);
    }
    tmem_wait_st();
    return l;
}

template <int NB>
__global__ void __launch_bounds__(Shape<NB>::threads, 1)
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
    constexpr int kThreads = Shape<NB>::threads;
    constexpr int kSoftmax0 = Shape<NB>::first_softmax_warp;
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
    if (threadIdx.x == 64) {
        tma_prefetch_desc(&tm_q0);
        tma_prefetch_desc(&tm_q1);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    // V rows B..NB-1 (MMA padding) are zero for the whole launch.
    {
        const int pad_chunks = (NB - p.B) * (kRowBytes / 16);
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
    const int H = p.heads;

    if (warp < kSoftmax0) {
        if constexpr (Shape<NB>::split)
            regs_dec<kRegsLow>();
        if (warp == 0) {
            // ==================================================== producer
            PlanWalker w;
            w.init(p.cu, p.n_seq, p.total, p.B, lane);
            const uint64_t pol = policy_evict_first();
            int qk_count = 0, v_count = 0;   // copies issued (stages used round-robin)
            int prev_h = 0, prev_f0 = 0;
            int n = 0;
            bool ok = true;

            auto issue_v = [&](int m, int h, int f0) -> bool {
                const int sv = m % kSV;
                const uint32_t uv = (uint32_t)(m / kSV);
                if (uv > 0 &&
                    !wait_bar(smem_u32(&bars->v_empty[sv]), (uv - 1) & 1, abort_flag, wait_ns, p.status))
                    return false;
                if (lane == 0) {
                    const uint32_t bar = smem_u32(&bars->v_full[sv]);
                    mbar_arrive_expect_tx(bar, p.B * kRowBytes);
                    tma_load_2d(v_base + sv * p.v_bytes, &tm_v, h * 64, f0, bar, pol);
                }
                ++v_count;
                __syncwarp();
                return true;
            };

            for (int item = blockIdx.x;; item += gridDim.x, ++n) {
                const int b = item / H;
                const int h = item - b * H;
                int f0, L, seq;
                if (!w.find(b, lane, f0, L, seq))
                    break;
                const int s = n % p.sqk;
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
                }
                ++qk_count;
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
            // drain: every issued copy must land before the CTA can exit.
            // Copies went to stages round-robin, so the last ones to each
            // stage are those of the final min(count, stages) items.
            if (lane == 0) {
                const bool skipped0 = (p.flags & NLE_FLAG_TEST_SKIP_FIRST_LOAD) != 0;
                for (int m = qk_count - p.sqk; m < qk_count; ++m)
                    if (m >= 0 && !(skipped0 && m == 0))
                        wait_bar_drain(smem_u32(&bars->qk_full[m % p.sqk]), (uint32_t)(m / p.sqk) & 1, wait_ns);
                for (int m = v_count - kSV; m < v_count; ++m)
                    if (m >= 0)
                        wait_bar_drain(smem_u32(&bars->v_full[m % kSV]), (uint32_t)(m / kSV) & 1, wait_ns);
            }
            __syncwarp();
        } else if (warp == 1) {
            // ==================================================== MMA issuer
            PlanWalker w;
            w.init(p.cu, p.n_seq, p.total, p.B, lane);
            const uint32_t id_pv = idesc_bf16_f32(128, 64, true);
            uint32_t tile_uses[2] = {0, 0};
            int n = 0;
            for (int item = blockIdx.x;; item += gridDim.x, ++n) {
                const int b = item / H;
                int f0, L, seq;
                if (!w.find(b, lane, f0, L, seq))
                    break;
                const int s = n % p.sqk;
                if (!wait_bar(smem_u32(&bars->qk_full[s]), (uint32_t)(n / p.sqk) & 1, abort_flag, wait_ns,
                              p.status))
                    break;
                tc_fence_after();
                const int ntiles = L > kQTile ? 2 : 1;
                const int nkeys = (L + 15) & ~15;   // MMA extent over keys
                const uint32_t id_s = idesc_bf16_f32(128, nkeys, false);
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
                        // K steps of 16 elements = 32 bytes inside the
                        // 128-byte swizzle atom: advance the start address
                        const uint64_t da = smem_desc_sw128(qaddr + t * kQTile * kRowBytes, 16, 1024);
                        const uint64_t db = smem_desc_sw128(kaddr, 16, 1024);
#pragma unroll 1
                        for (int kk = 0; kk < 4; ++kk)
                            mma_ss(tmem + t * kSlotCols, da + 2 * kk, db + 2 * kk, id_s, kk > 0 ? 1u : 0u);
                        mma_commit(smem_u32(&bars->s_full[t]));
                    }
                    __syncwarp();
                }
                if (!ok)
                    break;
                if (lane == 0)
                    mma_commit(smem_u32(&bars->qk_empty[s]));
                __syncwarp();
                const int sv = n % kSV;
                if (!wait_bar(smem_u32(&bars->v_full[sv]), (uint32_t)(n / kSV) & 1, abort_flag, wait_ns,
                              p.status))
                    break;
                // PV reads V rows 0..nkeys-1; rows L..nkeys-1 of a partial
                // block hold frames of the next block (or utterance): zero
                // them so nothing outside the block reaches PV (P is 0 there,
                // but 0 * Inf would be NaN).  Rows B..NB-1 are always zero.
                if (L < nkeys && L < p.B) {
                    const int zend = nkeys < p.B ? nkeys : p.B;
                    uint4 *vz = reinterpret_cast<uint4 *>(smem + v_off + sv * p.v_bytes + L * kRowBytes);
                    for (int i = lane; i < (zend - L) * (kRowBytes / 16); i += 32)
                        vz[i] = make_uint4(0, 0, 0, 0);
                    fence_proxy_async_smem();
                    __syncwarp();
                }
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
                        // N = 64 is one 128-byte swizzle atom along N, so the
                        // N-direction atom stride (LBO) is never used; K steps
                        // of 16 rows advance the start address by 2048 bytes.
                        const uint64_t db = smem_desc_sw128(vaddr, 0, 1024);
#pragma unroll 1
                        for (int kk = 0; kk < nkeys / 16; ++kk)
                            mma_ts(slot + kOCol, slot + kk * 8, db + (uint64_t)(kk * (16 * kRowBytes >> 4)), id_pv,
                                   kk > 0 ? 1u : 0u);
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
        }
    } else {
        if constexpr (Shape<NB>::split)
            regs_inc<kRegsHigh>();
        // ======================================================== softmax + epilogue
        const int t = (warp - kSoftmax0) >> 2;     // tile slot
        const int qq = warp & 3;                   // TMEM lane quarter of this warp
        const uint32_t tS = tmem + ((uint32_t)(qq * 32) << 16) + t * kSlotCols;
        const float sl2 = p.scale_log2;
        PlanWalker w;
        w.init(p.cu, p.n_seq, p.total, p.B, lane);
        uint32_t uses = 0;
        for (int item = blockIdx.x;; item += gridDim.x) {
            const int b = item / H;
            const int h = item - b * H;
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
            float l = 1.f;
            if (active)
                l = softmax_rows<NB, Shape<NB>::seg>(tS, L, sl2);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_u32(&bars->p_full[t]));
            if (!wait_bar(smem_u32(&bars->o_full[t]), uses & 1, abort_flag, wait_ns, p.status))
                break;
            tc_fence_after();
            uint32_t o[64];
            if (active) {
                tmem_ld32_nowait(tS + kOCol, &o[0]);
                tmem_ld32_nowait(tS + kOCol + 32, &o[32]);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 64; ++i)
                    reg_fence(o[i]);
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
                for (int c = 0; c < 8; ++c)
                    dst[c] = make_uint4(pack_bf16x2(__uint_as_float(o[8 * c + 0]) * inv, __uint_as_float(o[8 * c + 1]) * inv),
                                        pack_bf16x2(__uint_as_float(o[8 * c + 2]) * inv, __uint_as_float(o[8 * c + 3]) * inv),
                                        pack_bf16x2(__uint_as_float(o[8 * c + 4]) * inv, __uint_as_float(o[8 * c + 5]) * inv),
                                        pack_bf16x2(__uint_as_float(o[8 * c + 6]) * inv, __uint_as_float(o[8 * c + 7]) * inv));
            }
            ++uses;
        }
    }

    // ------------------------------------------------------------ teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

using BlockKernel = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, Params);

struct KernelInfo {
    BlockKernel fn;
    int threads;
    bool split;
};

template <int NB>
KernelInfo kernel_nb()
{
    return {reinterpret_cast<BlockKernel>(block_attn_kernel<NB>), Shape<NB>::threads, Shape<NB>::split};
}

KernelInfo pick_kernel(int nb)
{
    switch (nb) {
    case 16: return kernel_nb<16>();
    case 32: return kernel_nb<32>();
    case 48: return kernel_nb<48>();
    case 64: return kernel_nb<64>();
    case 80: return kernel_nb<80>();
    case 96: return kernel_nb<96>();
    case 112: return kernel_nb<112>();
    case 128: return kernel_nb<128>();
    case 144: return kernel_nb<144>();
    case 160: return kernel_nb<160>();
    case 176: return kernel_nb<176>();
    case 192: return kernel_nb<192>();
    case 208: return kernel_nb<208>();
    case 224: return kernel_nb<224>();
    case 240: return kernel_nb<240>();
    default: return kernel_nb<256>();
    }
}

// Per (NB/16, device): dynamic smem opted in so far, and whether the
// register count of a split build was verified (1 ok, -1 refused).
int g_smem_set[17][64] = {};
int g_regs_ok[17][64] = {};

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
    // upper bound on work items: each utterance has at most T/B + 1 blocks
    const long long max_items = ((long long)n_seq + total_frames / block_frames) * heads;
    if (max_items > 0x7fffffffLL)
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

    const KernelInfo kern = pick_kernel(NB);
    const int slot = dev < 64 ? dev : 0;
    if (kern.split) {
        // setmaxnreg.inc waits until the block's launch allocation can cover
        // the new split; it can only if every thread starts with exactly
        // kRegsLaunch registers.
        int &ok = g_regs_ok[NB / 16][slot];
        if (ok == 0 || dev >= 64) {
            cudaFuncAttributes fa;
            if (cudaFuncGetAttributes(&fa, reinterpret_cast<const void *>(kern.fn)) != cudaSuccess)
                return NLE_ERR_CUDA;
            ok = fa.numRegs == kRegsLaunch ? 1 : -1;
        }
        if (ok != 1)
            return NLE_ERR_UNSUPPORTED;
    }
    int &set = g_smem_set[NB / 16][slot];
    if (dev >= 64 || set < (int)smem) {
        if (cudaFuncSetAttribute(reinterpret_cast<const void *>(kern.fn),
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
            return NLE_ERR_CUDA;
        set = (int)smem;
    }
    const int grid = (int)(max_items < di.sm_count ? max_items : di.sm_count);
    kern.fn<<<grid, kern.threads, smem, static_cast<cudaStream_t>(stream)>>>(tq0, tq1, tk, tv, p);
    return cudaGetLastError() == cudaSuccess ? NLE_OK : NLE_ERR_CUDA;
}

extern "C" int nle_block_attn_fwd(const void *q, const void *k, const void *v, void *out, const int32_t *cu_seqlens,
                                  int n_seq, int64_t total_frames, int heads, int d_head, int block_frames,
                                  void *stream)
{
    return nle_block_attn_fwd_ex(q, k, v, out, cu_seqlens, n_seq, total_frames, heads, d_head, block_frames, 0.f,
                                 0, nullptr, 0, 0, stream);
}
