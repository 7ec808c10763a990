// varlen_attn_sm100a.cu -- full bidirectional self-attention inside each
// packed utterance, any length, on B200 (sm_100a).
//
// Operation (granite-speech-4.1-2b-nar model card, "Model Architecture" (3)
// Bidirectional LLM Editor: the LLM with its causal mask removed; "Usage /
// Installation": packed sequences, is_causal=False): for every utterance of
// the packed batch and every head,
//     O = softmax(scale * Q K^T) V  over all T frames of the utterance.
// The block kernel covers blocks of up to 256 frames in one key tile; here
// the keys of an utterance are walked in tiles of 64 with an online
// softmax, so T is unbounded.
//
// Design (one persistent CTA per SM, 20 warps):
//   warp 0      TMA producer.  Work item = (512 query rows of an utterance,
//               head).  Per item it loads the item's Q (one 128-row box
//               per row tile that has rows) into one of two Q stages, then
//               every key tile of the utterance (K and V boxes of 64 rows)
//               into a ring of KV stages, all 128-byte-swizzled (no
//               multicast).
//   warp 1      owns TMEM (allocates and frees it).
//   warp 2      V fix-up: waits for each KV stage to land and, for the
//               utterance's last, partial key tile, zeroes V rows past the
//               utterance up to the MMA's 16-row granule (their P is 0,
//               but 0 * Inf would be NaN), then releases the stage to the
//               chains.
//   warps 4-19  four chains of four warps; chain c takes query rows
//               128c..128c+127 of the item in TMEM slot c.  All chains walk
//               every key tile of the item, sharing the KV stages; their
//               MMAs and softmaxes interleave, so the exp units always have
//               rows to work on while other chains' MMAs run.  Per key
//               tile j, the chain's first warp issues (one elected lane):
//                 S = Q_c K_j^T  (tcgen05.mma kind::f16, M=128,
//                                N=ceil16(valid keys), K=64 in 4 steps)
//               and, once its four warps have written P,
//                 O += P V_j     (A = P from TMEM, B = V_j N-major, M=128,
//                                N=64, K=ceil16(valid keys)).
//               softmax: p = exp2(S*scale*log2e - m) with the row's running
//               shift m (set from the first 16 keys of the first tile) in
//               32-column register segments; keys past the utterance are 0
//               by index.  If an exponent would exceed 32, m moves up by a
//               whole k and the row's P, running sum and O are scaled by
//               2^-k (exact).  P (bf16) is written over S.
//               After the last tile O is read, divided by the row sum,
//               rounded to bf16 and stored with 16-byte stores, rows of the
//               utterance only.  A chain with no rows in the item only
//               releases the item's stages.
// TMEM (512 columns): slot c at column 128*c holds S (64 columns; P over
// its first 32) and O (64 columns at +64).
//
// Every mbarrier wait is bounded; on expiry the CTA drains its copies and
// MMAs in flight, frees TMEM and returns.
#include <cmath>

#include "attn_softmax.cuh"
#include "nle.h"
#include "nle_device.cuh"
#include "nle_host.h"

namespace {

using namespace nle;

constexpr int kChains = 4;                                  // softmax chains of 128 query rows
constexpr int kChain0 = 4;                                  // first warp of chain 0
constexpr int kThreads = 32 * (kChain0 + 4 * kChains);      // 640
constexpr int kQRows = 128;                                 // query rows per chain (MMA M)
constexpr int kItemRows = kChains * kQRows;                 // query rows per item
constexpr int kKeys = 64;                                   // keys per KV tile (one S/PV round)
constexpr int kRowBytes = 128;                              // one frame of one head: 64 bf16
constexpr uint32_t kQTileBytes = kQRows * kRowBytes;        // 16 KB
constexpr uint32_t kQStageBytes = kChains * kQTileBytes;    // 64 KB
constexpr uint32_t kKVTileBytes = kKeys * kRowBytes;        // 8 KB
constexpr uint32_t kKVStageBytes = 2 * kKVTileBytes;        // K, then V
constexpr int kMaxKV = 12;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSlotCols = 128;                         // per chain: S (64 columns), then O
constexpr uint32_t kOCol = 64;
constexpr int kSeg = 32;                                    // softmax register segment (2 per key tile)
constexpr int kDescRing = 4;                                // item descriptors in flight
constexpr int kDescReaders = 4 * kChains;                   // every chain warp reads every descriptor

// One work item as the producer publishes it to the chain warps (L < 0:
// no further item).
struct ItemDesc {
    int f0, L, T, h;
};

struct Bars {
    uint64_t q_full[2];
    uint64_t q_empty[2];         // kChains arrivals: each chain's last S MMA of the item
    uint64_t kv_full[kMaxKV];
    uint64_t kv_ready[kMaxKV];   // the fix-up warp has checked the stage
    uint64_t kv_empty[kMaxKV];   // kChains arrivals: each chain's PV MMA of the tile
    uint64_t s_full[kChains];
    uint64_t wg_p[kChains];      // 4 arrivals: P of the tile written
    uint64_t o_done[kChains];    // the chain's latest PV MMA has completed
    uint64_t mma_done[kChains];
    uint64_t desc_full[kDescRing];
    uint64_t desc_empty[kDescRing];   // kDescReaders arrivals: every chain warp has read the entry
    ItemDesc desc[kDescRing];
    uint32_t tmem_base;
    int abort_flag;
};

struct Params {
    const int32_t *cu;
    int n_seq;
    int total;
    int heads;
    int nkv;            // KV ring depth
    uint32_t kv_off;    // KV ring, after the two Q stages
    uint32_t bars_off;  // barriers, after the KV ring
    float scale_log2;
    __nv_bfloat16 *out;
    int out_stride;     // elements between output frames (heads * 64)
    int32_t *status;
    unsigned long long wait_ns;
    int flags;
};

// The CTA's items in order: item i = blockIdx.x + n * gridDim.x = u * H + h,
// u = the 512-row query unit of the batch.  Every role walks the same
// sequence.
struct ItemWalk {
    PlanWalker w;
    int b, h, step_b, step_h, H;

    __device__ __forceinline__ void init(const Params &p, int lane)
    {
        w.init(p.cu, p.n_seq, p.total, kItemRows, lane);
        H = p.heads;
        b = (int)(blockIdx.x / H);
        h = (int)(blockIdx.x % H);
        step_b = (int)(gridDim.x / H);
        step_h = (int)(gridDim.x % H);
    }

    // f0, L: the item's query rows; us, T: its utterance; hh: its head.
    __device__ __forceinline__ bool next(const Params &p, int lane, int &f0, int &L, int &us, int &T, int &hh)
    {
        int seq;
        if (!w.find(b, lane, f0, L, seq))
            return false;
        us = __ldg(p.cu + seq);
        T = __ldg(p.cu + seq + 1) - us;
        hh = h;
        b += step_b;
        h += step_h;
        if (h >= H) {
            h -= H;
            ++b;
        }
        return true;
    }
};

// 2-D tiled TMA load (no multicast) with the default L2 policy: K and V
// tiles are read again by every query unit of their utterance.
__device__ __forceinline__ void tma_load_2d_nohint(uint32_t dst, const void *tmap, int32_t x, int32_t y, uint32_t bar)
{
    asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(bar)
                 : "memory");
}

// p = exp2(s * sl2 - m) for the W keys of a segment (masked keys hold -inf
// -> 0), packed to bf16 pairs and stored over S's columns [C0/2, C0/2 +
// W/2) eight at a time: the S values they overwrite are already in
// registers.  Two partial sums and maxima and eight packed registers at a
// time keep the chain warps within their 96 registers.  Returns the
// segment sum; ymax: the largest exponent.
template <int W>
__device__ __forceinline__ float seg_exp_store(uint32_t tP, const uint32_t (&s)[kSeg], float sl2, float m,
                                               float &ymax)
{
    static_assert(W % 16 == 0 && W <= kSeg, "segment width");
    float ls[2] = {0.f, 0.f};
    float ym[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int c = 0; c < W / 2; c += 8) {
        uint32_t pk[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int i = 2 * (c + j);
            const float ya = fmaf(__uint_as_float(s[i]), sl2, -m);
            const float yb = fmaf(__uint_as_float(s[i + 1]), sl2, -m);
            ym[j & 1] = fmax3(ym[j & 1], ya, yb);
            const float pa = ex2_approx(ya);
            const float pb = ex2_approx(yb);
            ls[j & 1] += pa + pb;
            pk[j] = pack_bf16x2(pa, pb);
        }
        tmem_st8p(tP + c, pk);
    }
    ymax = fmaxf(ym[0], ym[1]);
    return ls[0] + ls[1];
}

// One segment of a key tile (whole warp): p for its W keys from the S values
// in `cur` (keys past the tile's valid ones already -inf), with the rare
// shift step of the block kernel's softmax, but done from registers: for a
// row whose exponent went past kYMax, the segment's exact max gives k, m
// moves up by k, the running sum and the product fs of this tile's factors
// take 2^-k, the segment is recomputed (its P stored again over the first
// attempt's) and the P already written in this tile (columns < C0/2) are
// rescaled (other rows: k = 0, unchanged).
template <int W>
__device__ __forceinline__ void tile_segment(uint32_t tS, int C0, uint32_t (&cur)[kSeg], float sl2, float &m,
                                             float &l, float &fs)
{
    float ymax;
    float ls = seg_exp_store<W>(tS + C0 / 2, cur, sl2, m, ymax);
    const bool mine = !(ymax <= kYMax);   // this row's exponent is too large (or NaN)
    if (__any_sync(kFull, mine)) {
        // only the rows that need it move their shift, so a row's result
        // never depends on the other rows of its warp
        const float y = seg_max<W>(cur) * sl2 - m;
        const int k = mine && y > 0.f ? (int)ceilf(y) : 0;
        const float f = k <= 126 ? __int_as_float((127 - k) << 23) : 0.f;
        m += (float)k;
        l *= f;
        fs *= f;
        tmem_wait_st();   // the first attempt's stores complete before they are overwritten
        ls = seg_exp_store<W>(tS + C0 / 2, cur, sl2, m, ymax);
        if (C0 > 0)
            rescale_p(tS, C0 / 2, f);
    }
    l += ls;
}

// Softmax of one key tile for this lane's row: keys [0, nv) of the tile are
// valid (nv >= 1).  first: the item's first tile (m is set here).  Returns
// the factor (a power of two, 1 normally) by which the row's earlier P
// weights changed, i.e. by which O must be scaled before this tile's PV.
__device__ __forceinline__ float softmax_tile(uint32_t tS, int nv, float sl2, float &m, float &l, bool first)
{
    float fs = 1.f;
    uint32_t cur[kSeg];
    seg_issue<kSeg>(tS, cur);
    tmem_wait_ld();
    seg_fence<kSeg>(cur);
    if (nv < kSeg)
        seg_mask<kSeg>(cur, 0, nv);
    if (first) {
        float mx = -INFINITY;
#pragma unroll
        for (int i = 0; i < 16; ++i)
            mx = fmaxf(mx, __uint_as_float(cur[i]));
        m = mx * sl2;
        l = 0.f;
    }
    tile_segment<kSeg>(tS, 0, cur, sl2, m, l, fs);
    if (nv > kSeg) {
        seg_issue<kSeg>(tS + kSeg, cur);
        tmem_wait_ld();
        seg_fence<kSeg>(cur);
        if (nv < 2 * kSeg)
            seg_mask<kSeg>(cur, kSeg, nv);
        tile_segment<kSeg>(tS, kSeg, cur, sl2, m, l, fs);
    }
    tmem_wait_st();
    return fs;
}

// O (64 fp32 columns of this lane's row) *= f.  Whole warp.
__device__ __forceinline__ void rescale_o(uint32_t tO, float f)
{
    for (int c = 0; c < 64; c += 16) {
        uint32_t r[16];
        tmem_ld16_nowait(tO + c, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            reg_fence(r[i]);
            r[i] = __float_as_uint(__uint_as_float(r[i]) * f);
        }
        tmem_st16(tO + c, r);
    }
    tmem_wait_st();
}

__global__ void __launch_bounds__(kThreads, 1)
    varlen_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t q_base = smem_u32(smem);
    const uint32_t kv_base = q_base + p.kv_off;
    Bars *bars = reinterpret_cast<Bars *>(smem + p.bars_off);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int nkv = p.nkv;

    // ------------------------------------------------------------ set-up
    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_u32(&bars->q_full[s]), 1);
            mbar_init(smem_u32(&bars->q_empty[s]), kChains);
        }
        for (int s = 0; s < nkv; ++s) {
            mbar_init(smem_u32(&bars->kv_full[s]), 1);
            mbar_init(smem_u32(&bars->kv_ready[s]), 1);
            mbar_init(smem_u32(&bars->kv_empty[s]), kChains);
        }
        for (int c = 0; c < kChains; ++c) {
            mbar_init(smem_u32(&bars->s_full[c]), 1);
            mbar_init(smem_u32(&bars->wg_p[c]), 4);
            mbar_init(smem_u32(&bars->o_done[c]), 1);
            mbar_init(smem_u32(&bars->mma_done[c]), 1);
        }
        for (int j = 0; j < kDescRing; ++j) {
            mbar_init(smem_u32(&bars->desc_full[j]), 1);
            mbar_init(smem_u32(&bars->desc_empty[j]), kDescReaders);
        }
        bars->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&bars->tmem_base), kTmemCols);
        tmem_relinquish();
    }
    if (threadIdx.x == 64) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    volatile int *abort_flag = &bars->abort_flag;
    const unsigned long long wait_ns = p.wait_ns;

    if (warp == 0) {
        // ======================================================== producer
        ItemWalk it;
        it.init(p, lane);
        const uint64_t pol_q = policy_evict_first();   // Q is read once; K and V by every query unit
        const bool skip0 = (p.flags & NLE_FLAG_TEST_SKIP_FIRST_LOAD) != 0;
        int nq = 0;    // items whose Q stage was claimed (= descriptors published)
        int nkt = 0;   // key tiles whose KV stage was claimed
        bool stop = false;
        // the chain warps learn each item (and the end) from the descriptor
        // ring, so they hold no plan-walking state
        auto publish = [&](const ItemDesc &d) -> bool {
            const int j = nq % kDescRing;
            if (nq >= kDescRing && !wait_bar(smem_u32(&bars->desc_empty[j]), (uint32_t)(nq / kDescRing - 1) & 1,
                                             abort_flag, wait_ns, p.status))
                return false;
            if (lane == 0) {
                bars->desc[j] = d;
                mbar_arrive(smem_u32(&bars->desc_full[j]));
            }
            __syncwarp();
            return true;
        };
        for (;;) {
            int f0, L, us, T, h;
            if (!it.next(p, lane, f0, L, us, T, h))
                break;
            if (!publish(ItemDesc{f0, L, T, h})) {
                stop = true;
                break;
            }
            const int qs = nq & 1;
            if (nq >= 2 && !wait_bar(smem_u32(&bars->q_empty[qs]), (uint32_t)((nq >> 1) - 1) & 1, abort_flag,
                                     wait_ns, p.status))
                break;
            if (lane == 0 && !(skip0 && nq == 0)) {
                const uint32_t bar = smem_u32(&bars->q_full[qs]);
                const uint32_t dst = q_base + qs * kQStageBytes;
                const int boxes = (L + kQRows - 1) / kQRows;   // row tiles with query rows
                mbar_arrive_expect_tx(bar, (uint32_t)boxes * kQTileBytes);
                for (int c = 0; c < boxes; ++c)
                    tma_load_2d(dst + c * kQTileBytes, &tm_q, h * 64, f0 + c * kQRows, bar, pol_q);
            }
            __syncwarp();
            ++nq;
            for (int j = 0; j * kKeys < T; ++j) {
                const int s = nkt % nkv;
                const uint32_t u = (uint32_t)(nkt / nkv);
                if (u > 0 &&
                    !wait_bar(smem_u32(&bars->kv_empty[s]), (u - 1) & 1, abort_flag, wait_ns, p.status)) {
                    stop = true;
                    break;
                }
                if (lane == 0) {
                    const uint32_t bar = smem_u32(&bars->kv_full[s]);
                    const uint32_t dst = kv_base + s * kKVStageBytes;
                    mbar_arrive_expect_tx(bar, kKVStageBytes);
                    tma_load_2d_nohint(dst, &tm_k, h * 64, us + j * kKeys, bar);
                    tma_load_2d_nohint(dst + kKVTileBytes, &tm_v, h * 64, us + j * kKeys, bar);
                }
                __syncwarp();
                ++nkt;
            }
            if (stop)
                break;
        }
        if (it.w.bad && lane == 0)
            report(p.status, NLE_ERR_INVALID_ARG);
        if (!stop)
            publish(ItemDesc{0, -1, 0, 0});   // end marker (its index is nq, not counted as an item)
        // drain: the last copy into each stage must land before exit
        if (lane == 0) {
            for (int m = nq - 2; m < nq; ++m)
                if (m >= 0 && !(skip0 && m == 0))
                    wait_bar_drain(smem_u32(&bars->q_full[m & 1]), (uint32_t)(m >> 1) & 1, wait_ns);
            for (int m = nkt - nkv; m < nkt; ++m)
                if (m >= 0)
                    wait_bar_drain(smem_u32(&bars->kv_full[m % nkv]), (uint32_t)(m / nkv) & 1, wait_ns);
        }
        __syncwarp();
    } else if (warp == 2) {
        // ======================================================== V fix-up
        ItemWalk it;
        it.init(p, lane);
        int nkt = 0;
        bool stop = false;
        for (;;) {
            int f0, L, us, T, h;
            if (!it.next(p, lane, f0, L, us, T, h))
                break;
            for (int j = 0; j * kKeys < T; ++j, ++nkt) {
                const int s = nkt % nkv;
                if (!wait_bar(smem_u32(&bars->kv_full[s]), (uint32_t)(nkt / nkv) & 1, abort_flag, wait_ns,
                              p.status)) {
                    stop = true;
                    break;
                }
                const int nv = T - j * kKeys < kKeys ? T - j * kKeys : kKeys;
                const int nk = (nv + 15) & ~15;
                if (nv < nk) {
                    uint4 *vz = reinterpret_cast<uint4 *>(smem + p.kv_off + s * kKVStageBytes + kKVTileBytes +
                                                          nv * kRowBytes);
                    for (int i = lane; i < (nk - nv) * (kRowBytes / 16); i += 32)
                        vz[i] = make_uint4(0, 0, 0, 0);
                    fence_proxy_async_smem();
                }
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(smem_u32(&bars->kv_ready[s]));
            }
            if (stop)
                break;
        }
    } else if (warp >= kChain0) {
        // ======================================================== chains
        const int c = (warp - kChain0) >> 2;   // chain = TMEM slot = row tile of the item
        const int qq = warp & 3;               // TMEM lane quarter of this warp
        const bool leader = qq == 0;
        const uint32_t slot = tmem + c * kSlotCols;
        const uint32_t tS = slot + ((uint32_t)(qq * 32) << 16);
        const float sl2 = p.scale_log2;
        const uint32_t id_pv = idesc_bf16_f32(128, 64, true);
        int n = 0;           // items
        int nkt = 0;         // key tiles walked (KV stage sequence)
        uint32_t uses = 0;   // S/PV rounds of this chain
        bool ok = true;
        for (;; ++n) {
            const int dj = n % kDescRing;
            if (!wait_bar(smem_u32(&bars->desc_full[dj]), (uint32_t)(n / kDescRing) & 1, abort_flag, wait_ns,
                          p.status)) {
                ok = false;
                break;
            }
            // the entry stays claimed until the item's output is written:
            // its first frame and head are read again there
            const int L = bars->desc[dj].L, T = bars->desc[dj].T;
            if (L < 0) {
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(smem_u32(&bars->desc_empty[dj]));
                break;   // no further item
            }
            const int qs = n & 1;
            const int tiles = (T + kKeys - 1) / kKeys;
            const bool chain_rows = L > c * kQRows;
            const int row0 = c * kQRows + qq * 32;   // first item row of this warp
            const bool active = row0 < L;
            if (leader &&
                !wait_bar(smem_u32(&bars->q_full[qs]), (uint32_t)(n >> 1) & 1, abort_flag, wait_ns, p.status)) {
                ok = false;
                break;
            }
            if (!chain_rows) {
                // no query rows for this chain: release the item's Q and KV
                // stages in order (each only once it holds this item's data)
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(smem_u32(&bars->desc_empty[dj]));
                if (leader) {
                    if (lane == 0)
                        mbar_arrive(smem_u32(&bars->q_empty[qs]));
                    for (int j = 0; j < tiles; ++j) {
                        const int s = (nkt + j) % nkv;
                        if (!wait_bar(smem_u32(&bars->kv_ready[s]), (uint32_t)((nkt + j) / nkv) & 1, abort_flag,
                                      wait_ns, p.status)) {
                            ok = false;
                            break;
                        }
                        if (lane == 0)
                            mbar_arrive(smem_u32(&bars->kv_empty[s]));
                    }
                    __syncwarp();
                }
                nkt += tiles;
                if (!ok)
                    break;
                continue;
            }
            float m = 0.f, l = 0.f;
            const uint32_t qaddr = q_base + qs * kQStageBytes + c * kQTileBytes;
            for (int j = 0; j < tiles; ++j, ++nkt) {
                const int s = nkt % nkv;
                const int nv = T - j * kKeys < kKeys ? T - j * kKeys : kKeys;
                const int nk = (nv + 15) & ~15;
                const uint32_t kaddr = kv_base + s * kKVStageBytes;
                // ---------------------------------------------- S = Q K^T
                if (leader) {
                    if (!wait_bar(smem_u32(&bars->kv_ready[s]), (uint32_t)(nkt / nkv) & 1, abort_flag, wait_ns,
                                  p.status)) {
                        ok = false;
                    } else if (uses > 0 && !wait_bar(smem_u32(&bars->o_done[c]), (uses - 1) & 1, abort_flag,
                                                     wait_ns, p.status)) {
                        // the previous PV still reads P from the S columns
                        ok = false;
                    } else {
                        tc_fence_after();
                        const uint64_t da = smem_desc_sw128(qaddr, 16, 1024);
                        const uint64_t db = smem_desc_sw128(kaddr, 16, 1024);
                        const uint32_t id_s = idesc_bf16_f32(128, nk, false);
                        if (elect_one()) {
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                mma_ss(slot, da + 2 * kk, db + 2 * kk, id_s, kk > 0 ? 1u : 0u);
                            mma_commit(smem_u32(&bars->s_full[c]));
                            if (j == tiles - 1)   // the item's last S: its Q stage can be reused
                                mma_commit(smem_u32(&bars->q_empty[qs]));
                        }
                    }
                    __syncwarp();
                }
                if (!ok)
                    break;
                // ---------------------------------------------- softmax
                if (!wait_bar(smem_u32(&bars->s_full[c]), uses & 1, abort_flag, wait_ns, p.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (active) {
                    const float fs = softmax_tile(tS, nv, sl2, m, l, j == 0);
                    // O holds the earlier tiles' sum (their PV completed
                    // before this tile's S): scale it with the row's P
                    if (j > 0 && __any_sync(kFull, fs != 1.f))
                        rescale_o(tS + kOCol, fs);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(smem_u32(&bars->wg_p[c]));
                // ---------------------------------------------- O += P V
                if (leader) {
                    if (!wait_bar(smem_u32(&bars->wg_p[c]), uses & 1, abort_flag, wait_ns, p.status)) {
                        ok = false;
                    } else {
                        tc_fence_after();
                        // N = 64 is one 128-byte swizzle atom along N; K
                        // steps of 16 rows advance the start by 2048 bytes
                        const uint64_t dv = smem_desc_sw128(kaddr + kKVTileBytes, 0, 1024);
                        if (elect_one()) {
                            for (int kk = 0; kk < nk / 16; ++kk)
                                mma_ts(slot + kOCol, slot + kk * 8, dv + (uint64_t)(kk * (16 * kRowBytes >> 4)), id_pv,
                                       (j > 0 || kk > 0) ? 1u : 0u);
                            mma_commit(smem_u32(&bars->o_done[c]));
                            mma_commit(smem_u32(&bars->kv_empty[s]));
                        }
                    }
                    __syncwarp();
                }
                ++uses;
                if (!ok)
                    break;
            }
            if (!ok)
                break;
            // ---------------------------------------------- output
            if (!wait_bar(smem_u32(&bars->o_done[c]), (uses - 1) & 1, abort_flag, wait_ns, p.status)) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (active) {
                // O in two halves of 32 columns (registers are scarce at 20 warps)
                const float inv = 1.f / l;
                const bool row_ok = row0 + lane < L;
                const int f0 = bars->desc[dj].f0, h = bars->desc[dj].h;
                uint4 *dst = reinterpret_cast<uint4 *>(p.out + (size_t)(f0 + row0 + lane) * p.out_stride + h * 64);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t o[32];
                    tmem_ld32_nowait(tS + kOCol + 32 * half, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        reg_fence(o[i]);
                    if (row_ok) {
#pragma unroll
                        for (int cc = 0; cc < 4; ++cc)
                            dst[4 * half + cc] = make_uint4(
                                pack_bf16x2(__uint_as_float(o[8 * cc]) * inv, __uint_as_float(o[8 * cc + 1]) * inv),
                                pack_bf16x2(__uint_as_float(o[8 * cc + 2]) * inv, __uint_as_float(o[8 * cc + 3]) * inv),
                                pack_bf16x2(__uint_as_float(o[8 * cc + 4]) * inv, __uint_as_float(o[8 * cc + 5]) * inv),
                                pack_bf16x2(__uint_as_float(o[8 * cc + 6]) * inv, __uint_as_float(o[8 * cc + 7]) * inv));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_u32(&bars->desc_empty[dj]));
        }
        // this chain's MMAs must finish before TMEM is released
        if (leader) {
            if (elect_one()) {
                mma_commit(smem_u32(&bars->mma_done[c]));
                wait_bar_drain(smem_u32(&bars->mma_done[c]), 0, wait_ns);
            }
            __syncwarp();
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

} // namespace

extern "C" int nle_varlen_attn_fwd_ex(const void *q, const void *k, const void *v, void *out,
                                      const int32_t *cu_seqlens, int n_seq, int64_t total_frames, int heads,
                                      int d_head, float softmax_scale, int64_t row_stride_qkv, int32_t *dev_status,
                                      int flags, int64_t wait_limit_ns, void *stream)
{
    if (n_seq < 0 || total_frames < 0 || heads <= 0 || wait_limit_ns < 0)
        return NLE_ERR_INVALID_ARG;
    if (d_head != 64 || total_frames > 0x7fffffffLL)
        return NLE_ERR_UNSUPPORTED;
    // upper bound on work items: each utterance has at most T/512 + 1 query units
    const long long max_items = ((long long)n_seq + total_frames / kItemRows) * heads;
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
    // the kernel counts the key tiles a CTA walks in 32 bits
    const long long grid_ll = max_items < di.sm_count ? max_items : di.sm_count;
    if ((max_items / grid_ll + 1) * (total_frames / kKeys + 1) > 0x7fffffffLL)
        return NLE_ERR_UNSUPPORTED;

    Params p{};
    p.cu = cu_seqlens;
    p.n_seq = n_seq;
    p.total = (int)total_frames;
    p.heads = heads;
    // two Q stages, then as many KV stages as fit (up to kMaxKV), then the
    // barriers and alignment slack
    const size_t bars_bytes = ((sizeof(Bars) + 127) / 128) * 128 + 1024;
    const size_t q_bytes = 2 * (size_t)kQStageBytes;
    int nkv = (int)(((size_t)di.smem_optin - q_bytes - bars_bytes) / kKVStageBytes);
    if (nkv > kMaxKV)
        nkv = kMaxKV;
    if (nkv < 2)
        return NLE_ERR_UNSUPPORTED;
    p.nkv = nkv;
    p.kv_off = (uint32_t)q_bytes;
    p.bars_off = (uint32_t)(q_bytes + (size_t)nkv * kKVStageBytes);
    size_t smem = p.bars_off + bars_bytes;
    // one CTA per SM: it owns all 512 TMEM columns
    if (smem <= (size_t)di.smem_optin / 2)
        smem = (size_t)di.smem_optin / 2 + 1024;
    const double scale = softmax_scale > 0.f ? (double)softmax_scale : 1.0 / std::sqrt((double)d_head);
    p.scale_log2 = (float)(scale * 1.4426950408889634);
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.out_stride = (int)dense;
    p.status = dev_status;
    p.wait_ns = wait_limit_ns > 0 ? (unsigned long long)wait_limit_ns : 1000000000ull;
    p.flags = flags;

    CUtensorMap tq, tk, tv;
    const uint64_t cols = (uint64_t)dense, rows = (uint64_t)total_frames;
    if (!nle::encode_tmap_bf16_2d(&tq, q, cols, rows, stride, 64, kQRows) ||
        !nle::encode_tmap_bf16_2d(&tk, k, cols, rows, stride, 64, kKeys) ||
        !nle::encode_tmap_bf16_2d(&tv, v, cols, rows, stride, 64, kKeys))
        return NLE_ERR_CUDA;

    if (!nle::allow_max_dynamic_smem(reinterpret_cast<const void *>(varlen_attn_kernel), dev, di.smem_optin))
        return NLE_ERR_CUDA;
    const int grid = (int)grid_ll;
    varlen_attn_kernel<<<grid, kThreads, smem, static_cast<cudaStream_t>(stream)>>>(tq, tk, tv, p);
    return cudaGetLastError() == cudaSuccess ? NLE_OK : NLE_ERR_CUDA;
}

extern "C" int nle_varlen_attn_fwd(const void *q, const void *k, const void *v, void *out,
                                   const int32_t *cu_seqlens, int n_seq, int64_t total_frames, int heads, int d_head,
                                   void *stream)
{
    return nle_varlen_attn_fwd_ex(q, k, v, out, cu_seqlens, n_seq, total_frames, heads, d_head, 0.f, 0, nullptr, 0,
                                  0, stream);
}
