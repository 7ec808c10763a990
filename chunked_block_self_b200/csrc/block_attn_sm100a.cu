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
//   warps 0, 1  TMA producers.  Work item = (block, head).  Warp 0 loads
//               Q (two boxes: rows 0..127 and 128..B-1) and K of each item
//               into a ring of QK stages, warp 1 loads V into a ring of V
//               stages, all as 128-byte-swizzled TMA boxes (no multicast).
//               Warp 1 also owns TMEM (allocates and frees it).
//   warps 4-7   tile warpgroup 0, TMEM slot 0: the CTA's even items,
//   warps 8-11  tile warpgroup 1, TMEM slot 1: the odd items.  For each of
//               its items a warpgroup computes row tile 0 (block rows
//               0..127) and then, for blocks longer than 128 frames, row
//               tile 1 (rows 128..B-1) in its slot; the two warpgroups run
//               independent chains, so one's MMA and output phases overlap
//               the other's softmax.  The first warp of each warpgroup
//               issues the slot's MMAs (one elected lane, warp-uniform
//               descriptors):
//                 S = Q_x K^T     tcgen05.mma kind::f16, M=128, N=ceil16(L),
//                                 K=64 in 4 steps
//                 O_x = P V       A operand = P in TMEM, B = V (N-major) in
//                                 smem, M=128, N=64, K=ceil16(L) in steps
//                                 of 16
//               Before the first PV of a partial block the warpgroup zeroes
//               V rows L..ceil16(L)-1 in shared memory (frames outside the
//               block; P is 0 there, but 0 * Inf would be NaN).  Each
//               thread owns one block row (its TMEM lane) and reads S in
//               64-column register segments: p = exp2(S*scale*log2e
//               - m) in fp32 with one shift m per row (keys >= L are 0 by
//               index, never by value), row sum, bf16 pack, P written back
//               over S.  The epilogue reads O, divides by the row sum,
//               rounds to bf16 and writes each row < L with 16-byte vector
//               stores, while the warpgroup's next S MMA runs.  Rows past the
//               block end are never written.
//               QK and V rings have even depths, so an item's stages have
//               the parity of its warpgroup and each stage belongs to one
//               warpgroup.
// The MMAs of an item stop at ceil16(L) keys, so a partial block costs only
// its own keys.
// TMEM (512 columns): tile slot t at column 256*t holds S (NB columns), then
// P (NB/2 columns, over S) and O (64 columns at +128).
//
// Every mbarrier wait is bounded (see nle_device.cuh); on expiry the CTA
// drains its copies and MMAs in flight, frees TMEM and returns.
#include <cmath>

#include "nle.h"
#include "attn_softmax.cuh"
#include "nle_device.cuh"
#include "nle_host.h"

// Optional cycle trace of CTA 0 for performance analysis (not built by
// default): NLE_TRACE_AT(role, item, event) stores clock64() into a device
// buffer registered with nle_trace_set().
#ifdef NLE_TRACE
__device__ unsigned long long *g_nle_trace = nullptr;
extern "C" int nle_trace_set(void *p)
{
    return cudaMemcpyToSymbol(g_nle_trace, &p, sizeof(p)) == cudaSuccess ? 0 : -1;
}
#define NLE_TRACE_AT(role, n, ev)                                                                       \
    do {                                                                                                \
        if (blockIdx.x == 0 && g_nle_trace && (n) < 64)                                                 \
            g_nle_trace[((role) * 64 + (n)) * 16 + (ev)] = clock64();                                   \
    } while (0)
#else
#define NLE_TRACE_AT(role, n, ev) \
    do {                          \
    } while (0)
#endif

namespace {

using namespace nle;

// Three warpgroups: warps 0-1 producers (warp 1 also owns TMEM), warps 2-3 idle,
// warps 4-11 the two tile warpgroups (168 registers each; the softmax works
// on 64-column segments of S).
constexpr int kThreads = 384;
constexpr int kSoftmax0 = 4;
constexpr int kSeg = 64;

constexpr int kQTile = 128;        // MMA M (rows per tile)
constexpr int kRowBytes = 128;     // one frame of one head: 64 bf16
constexpr int kMaxQK = 4;          // QK ring depth upper bound
constexpr int kMaxV = 4;           // V ring depth upper bound
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSlotCols = 256; // TMEM columns per tile slot
constexpr uint32_t kOCol = 128;     // O offset inside a tile slot

struct Bars {
    uint64_t qk_full[kMaxQK];
    uint64_t qk_empty[kMaxQK];   // the item's last S MMA has completed
    uint64_t v_full[kMaxV];
    uint64_t v_empty[kMaxV];     // the item's last PV MMA has completed
    uint64_t s_full[2];
    uint64_t wg_p[2];            // 4 arrivals: P of the unit written
    uint64_t o_full[2];
    uint64_t wg_o[2];            // 4 arrivals: O of the unit read from TMEM
    uint64_t mma_done[2];
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
    int nsv;      // V ring depth
    uint32_t q_bytes;   // Q region of a QK stage
    uint32_t qk_bytes;  // QK stage
    uint32_t v_bytes;   // V stage
    uint32_t bars_off;  // barriers, after the QK and V rings
    int split;          // one row tile per work item (batches that do not fill the GPU)
    float scale_log2;
    __nv_bfloat16 *out;
    int out_stride;     // elements between output frames (heads * 64)
    int32_t *status;
    unsigned long long wait_ns;
    int flags;
};

// The CTA's work items in order: raw item i = blockIdx.x + k * gridDim.x.
// Whole items: i = b * H + h, both row tiles of block b, head h.  Split
// items (p.split, for batches too small to fill the GPU): i = (b * H + h) *
// 2 + x, row tile x alone, so the two row tiles of a block run on two
// chains at once; a block of <= 128 frames has no row tile 1, and every
// role skips that item alike.
struct ItemSeq {
    int b, h, x;      // the next raw item: block, head, row tile
    int sb, sh, sx;   // the step gridDim.x in the same digits

    __device__ __forceinline__ void init(const Params &p)
    {
        const int H = p.heads, G = (int)gridDim.x, i = (int)blockIdx.x;
        const int bh = p.split ? i >> 1 : i, sbh = p.split ? G >> 1 : G;
        x = p.split ? i & 1 : 0;
        sx = p.split ? G & 1 : 0;
        b = bh / H;
        h = bh % H;
        sb = sbh / H;
        sh = sbh % H;
    }

    // the next raw item: block b, head h, row tile x (0 for whole items)
    __device__ __forceinline__ void next(const Params &p, int &ob, int &oh, int &ox)
    {
        ob = b;
        oh = h;
        ox = x;
        x += sx;
        const int carry = x >> 1;   // x in {0, 1, 2}
        x &= 1;
        h += sh + carry;
        b += sb;
        if (h >= p.heads) {   // h < 2 H: one wrap at most
            h -= p.heads;
            ++b;
        }
    }
};

template <int NB>
__global__ void __launch_bounds__(kThreads, 1)
    block_attn_kernel(const __grid_constant__ CUtensorMap tm_q0, const __grid_constant__ CUtensorMap tm_q1,
                      const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, const Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t qk_base = smem_u32(smem);
    const uint32_t v_off = p.sqk * p.qk_bytes;
    const uint32_t v_base = qk_base + v_off;
    Bars *bars = reinterpret_cast<Bars *>(smem + p.bars_off);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // ------------------------------------------------------------ set-up
    if (threadIdx.x == 0) {
        for (int s = 0; s < p.sqk; ++s) {
            mbar_init(smem_u32(&bars->qk_full[s]), 1);
            mbar_init(smem_u32(&bars->qk_empty[s]), 1);
        }
        for (int s = 0; s < p.nsv; ++s) {
            mbar_init(smem_u32(&bars->v_full[s]), 1);
            mbar_init(smem_u32(&bars->v_empty[s]), 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(smem_u32(&bars->s_full[t]), 1);
            mbar_init(smem_u32(&bars->wg_p[t]), 4);
            mbar_init(smem_u32(&bars->o_full[t]), 1);
            mbar_init(smem_u32(&bars->wg_o[t]), 4);
            mbar_init(smem_u32(&bars->mma_done[t]), 1);
        }
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
        for (int i = threadIdx.x; i < p.nsv * pad_chunks; i += kThreads) {
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

    if (warp == 0 || warp == 1) {
        // ==================================================== producers
        // Warp 0 loads Q and K of every item, warp 1 loads V; each refills a
        // stage as soon as the stage's last reader has released it (QK: the
        // item's last S MMA; V: its last PV MMA).
        const bool is_v = warp == 1;
        const int nst = is_v ? p.nsv : p.sqk;
        PlanWalker w;
        w.init(p.cu, p.n_seq, p.total, p.B, lane);
        const uint64_t pol = policy_evict_first();
        const bool skip0 = !is_v && (p.flags & NLE_FLAG_TEST_SKIP_FIRST_LOAD) != 0;
        int n = 0;   // items whose copies were issued
        ItemSeq items;
        items.init(p);
        for (;;) {
            int b, h, x, f0, L, seq;
            items.next(p, b, h, x);
            if (!w.find(b, lane, f0, L, seq))
                break;
            if (x == 1 && L <= kQTile)
                continue;   // split items: the block has no row tile 1
            const int s = n % nst;
            const uint32_t u = (uint32_t)(n / nst);
            if (u > 0 && !wait_bar(smem_u32(is_v ? &bars->v_empty[s] : &bars->qk_empty[s]), (u - 1) & 1, abort_flag,
                                   wait_ns, p.status))
                break;
            if (lane == 0) {
                if (is_v) {
                    const uint32_t bar = smem_u32(&bars->v_full[s]);
                    mbar_arrive_expect_tx(bar, p.B * kRowBytes);
                    tma_load_2d(v_base + s * p.v_bytes, &tm_v, h * 64, f0, bar, pol);
                } else if (!(skip0 && n == 0)) {
                    // Q of the item's row tiles (a split item: its one tile), then K
                    const bool t0 = !p.split || x == 0;
                    const bool t1 = p.split ? x == 1 : L > kQTile;
                    const uint32_t bar = smem_u32(&bars->qk_full[s]);
                    const uint32_t bytes = ((t0 ? p.q0rows : 0) + (t1 ? p.q1rows : 0) + p.B) * kRowBytes;
                    const uint32_t qdst = qk_base + s * p.qk_bytes;
                    mbar_arrive_expect_tx(bar, bytes);
                    if (t0)
                        tma_load_2d(qdst, &tm_q0, h * 64, f0, bar, pol);
                    if (t1)
                        tma_load_2d(qdst + kQTile * kRowBytes, &tm_q1, h * 64, f0 + kQTile, bar, pol);
                    tma_load_2d(qdst + p.q_bytes, &tm_k, h * 64, f0, bar, pol);
                }
                NLE_TRACE_AT(0, n, is_v ? 1 : 0);
            }
            __syncwarp();
            ++n;
        }
        if (!is_v && w.bad && lane == 0)
            report(p.status, NLE_ERR_INVALID_ARG);
        // drain: every issued copy must land before the CTA can exit.
        // Copies went to stages round-robin, so the last ones to each stage
        // are those of the final min(n, stages) items.
        if (lane == 0) {
            for (int m = n - nst; m < n; ++m)
                if (m >= 0 && !(skip0 && m == 0))
                    wait_bar_drain(smem_u32(is_v ? &bars->v_full[m % nst] : &bars->qk_full[m % nst]),
                                   (uint32_t)(m / nst) & 1, wait_ns);
        }
        __syncwarp();
    } else if (warp < kSoftmax0) {
        // warps 2, 3: no role
    } else {
        // ======================================================== tile warpgroups
        // Warpgroup t owns TMEM slot t and computes the CTA's items
        // n = t, t + 2, t + 4, ...: for each, row tile 0 (block rows
        // 0..127) and then, for blocks longer than 128 frames, row tile 1
        // (rows 128..B-1), one after the other in its slot.  The two
        // warpgroups thus run independent chains, and one's MMA and output
        // phases overlap the other's softmax.  The first warp's elected lane
        // issues the slot's MMAs; all four warps run softmax and epilogue.
        const int t = (warp - kSoftmax0) >> 2;     // TMEM slot
        const int qq = warp & 3;                   // TMEM lane quarter of this warp
        const bool leader = qq == 0;
        const uint32_t slot = tmem + t * kSlotCols;
        const uint32_t tS = slot + ((uint32_t)(qq * 32) << 16);
        const float sl2 = p.scale_log2;
        const uint32_t id_pv = idesc_bf16_f32(128, 64, true);
        PlanWalker w;
        w.init(p.cu, p.n_seq, p.total, p.B, lane);
        // the CTA's item sequence: item n is blockIdx.x + n * gridDim.x
        ItemSeq items;
        items.init(p);
        int next_n = 0;      // next item of the CTA's sequence (not yet looked at)
        int n = -1;          // current item
        int x = 1;           // current row tile of the item
        bool fresh = false;  // the current unit is its item's first (its stages still to be waited for)
        uint32_t uses = 0;   // units (item, row tile) this slot has computed
        int f0 = 0, L = 0, hcur = 0, nkeys = 16, s = 0, sv = 0;
        bool ok = true;

        // Move to the slot's next unit: row tile 1 of the current item if it
        // has one (whole items), else the first (or, split, the only) row
        // tile of the slot's next item.  The leader then
        // issues the unit's S MMA (after the slot's previous O has been read
        // by all four warps).  False at the end of the work.
        // Both ring depths are even, so the item's stages have the parity of
        // its slot: each stage belongs to one slot, whose items meet its
        // phases one by one, in order (a parity wait is only meaningful on
        // the current phase or the one after it).
        auto advance = [&]() -> bool {
            if (p.split || !(x == 0 && L > kQTile)) {
                // the slot's next item: pass over the other slot's one
                for (;;) {
                    int b, hh, xx, sf0, sL, sseq;
                    items.next(p, b, hh, xx);
                    if (!w.find(b, lane, sf0, sL, sseq))
                        return false;
                    if (xx == 1 && sL <= kQTile)
                        continue;   // split items: the block has no row tile 1
                    const int nn = next_n++;
                    if ((nn & 1) != t)
                        continue;
                    n = nn;
                    f0 = sf0;
                    L = sL;
                    hcur = hh;
                    x = xx;
                    break;
                }
                fresh = true;
                nkeys = (L + 15) & ~15;   // MMA extent over keys
                s = n % p.sqk;
                sv = n % p.nsv;
            } else {
                x = 1;
                fresh = false;
            }
            if (leader) {
                if (lane == 0)
                    NLE_TRACE_AT(1 + t, n * 2 + x, 0);
                if (fresh &&
                    !wait_bar(smem_u32(&bars->qk_full[s]), (uint32_t)(n / p.sqk) & 1, abort_flag, wait_ns, p.status)) {
                    ok = false;
                    return false;
                }
                if (uses > 0 &&
                    !wait_bar(smem_u32(&bars->wg_o[t]), (uses - 1) & 1, abort_flag, wait_ns, p.status)) {
                    ok = false;
                    return false;
                }
                tc_fence_after();
                // K steps of 16 elements = 32 bytes inside the 128-byte
                // swizzle atom: advance the descriptor start address
                const uint32_t qaddr = qk_base + s * p.qk_bytes;
                const uint64_t da = smem_desc_sw128(qaddr + x * kQTile * kRowBytes, 16, 1024);
                const uint64_t db = smem_desc_sw128(qaddr + p.q_bytes, 16, 1024);
                const uint32_t id_s = idesc_bf16_f32(128, nkeys, false);
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ss(slot, da + 2 * kk, db + 2 * kk, id_s, kk > 0 ? 1u : 0u);
                    mma_commit(smem_u32(&bars->s_full[t]));
                    if (p.split || x == 1 || L <= kQTile)   // the item's last S: its QK stage can be reused
                        mma_commit(smem_u32(&bars->qk_empty[s]));
                    NLE_TRACE_AT(1 + t, n * 2 + x, 1);
                }
                __syncwarp();
            }
            return true;
        };

        // Each pass: advance (the leader issues the next unit's S MMA),
        // write the previous unit's output, then compute the current unit.
        uint32_t pk[32];
        bool pending = false;          // pk holds rows of the previous unit
        int ef0 = 0, eL = 0, eh = 0, erow0 = 0;
        for (;;) {
            const bool have = advance();
            if (!ok)
                break;
            if (pending) {
                // rows past the block end are never written
                if (erow0 + lane < eL) {
                    uint4 *dst =
                        reinterpret_cast<uint4 *>(p.out + (size_t)(ef0 + erow0 + lane) * p.out_stride + eh * 64);
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        dst[c] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
                }
                pending = false;
            }
            if (!have)
                break;
            const uint32_t ph_v = (uint32_t)(n / p.nsv) & 1;
            // ---------------------------------------------- softmax
            if (!wait_bar(smem_u32(&bars->s_full[t]), uses & 1, abort_flag, wait_ns, p.status))
                break;
            tc_fence_after();
            if (lane == 0 && qq == 0)
                NLE_TRACE_AT(3 + t, n * 2 + x, 0);
            const int row0 = x * kQTile + qq * 32;   // first block row of this warp
            const bool active = row0 < L;
            float l = 1.f;
            if (active)
                l = block_softmax_rows<NB, kSeg>(tS, L, sl2);
            if (lane == 0 && qq == 0)
                NLE_TRACE_AT(3 + t, n * 2 + x, 1);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_u32(&bars->wg_p[t]));
            // ---------------------------------------------- O = P V
            if (leader) {
                if (!wait_bar(smem_u32(&bars->wg_p[t]), uses & 1, abort_flag, wait_ns, p.status))
                    break;
                if (fresh) {
                    if (!wait_bar(smem_u32(&bars->v_full[sv]), ph_v, abort_flag, wait_ns, p.status))
                        break;
                    if (L < nkeys && L < p.B) {
                        // PV reads V rows 0..nkeys-1; rows L..nkeys-1 of a
                        // partial block hold frames of the next block (or
                        // utterance): zero them so nothing outside the block
                        // reaches PV (P is 0 there, but 0 * Inf would be
                        // NaN).  Rows B..NB-1 are always zero.
                        const int zend = nkeys < p.B ? nkeys : p.B;
                        uint4 *vz = reinterpret_cast<uint4 *>(smem + v_off + sv * p.v_bytes + L * kRowBytes);
                        for (int i = lane; i < (zend - L) * (kRowBytes / 16); i += 32)
                            vz[i] = make_uint4(0, 0, 0, 0);
                        fence_proxy_async_smem();
                        __syncwarp();
                    }
                }
                tc_fence_after();
                if (lane == 0)
                    NLE_TRACE_AT(1 + t, n * 2 + x, 5);
                // N = 64 is one 128-byte swizzle atom along N, so the
                // N-direction atom stride (LBO) is never used; K steps of 16
                // rows advance the start address by 2048 bytes.
                const uint64_t dv = smem_desc_sw128(v_base + sv * p.v_bytes, 0, 1024);
                if (elect_one()) {
                    for (int kk = 0; kk < nkeys / 16; ++kk)
                        mma_ts(slot + kOCol, slot + kk * 8, dv + (uint64_t)(kk * (16 * kRowBytes >> 4)), id_pv,
                               kk > 0 ? 1u : 0u);
                    mma_commit(smem_u32(&bars->o_full[t]));
                    if (p.split || x == 1 || L <= kQTile)   // the item's last PV: its V stage can be reused
                        mma_commit(smem_u32(&bars->v_empty[sv]));
                    NLE_TRACE_AT(1 + t, n * 2 + x, 6);
                }
                __syncwarp();
            }
            // ---------------------------------------------- read O
            if (!wait_bar(smem_u32(&bars->o_full[t]), uses & 1, abort_flag, wait_ns, p.status))
                break;
            tc_fence_after();
            if (lane == 0 && qq == 0)
                NLE_TRACE_AT(3 + t, n * 2 + x, 2);
            if (active) {
                uint32_t o[64];
#pragma unroll
                for (int c = 0; c < 64; c += 16)
                    tmem_ld16_nowait(tS + kOCol + c, &o[c]);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 64; ++i)
                    reg_fence(o[i]);
                const float inv = 1.f / l;
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    pk[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_u32(&bars->wg_o[t]));
            if (lane == 0 && qq == 0)
                NLE_TRACE_AT(3 + t, n * 2 + x, 3);
            ++uses;
            pending = active;
            ef0 = f0;
            eL = L;
            eh = hcur;
            erow0 = row0;
        }
        // this slot's MMAs must finish before TMEM is released
        if (leader) {
            if (elect_one()) {
                mma_commit(smem_u32(&bars->mma_done[t]));
                wait_bar_drain(smem_u32(&bars->mma_done[t]), 0, wait_ns);
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

using BlockKernel = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, Params);

struct KernelInfo {
    BlockKernel fn;
};

template <int NB>
KernelInfo kernel_nb()
{
    return {reinterpret_cast<BlockKernel>(block_attn_kernel<NB>)};
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
    // Shared memory: QK ring and V ring, each of an even depth (the two
    // tile warpgroups take alternate items, so each stage then belongs to
    // one warpgroup), as deep as fits (V first: it is held from the item's
    // first PV to its last), then the barriers and alignment slack.
    const size_t bars_bytes = ((sizeof(Bars) + 127) / 128) * 128 + 1024;
    int sqk = 0, nsv = 0;
    for (const int v : {4, 2}) {
        for (const int q : {4, 2})
            if ((size_t)q * p.qk_bytes + (size_t)v * p.v_bytes + bars_bytes <= (size_t)di.smem_optin) {
                sqk = q;
                nsv = v;
                break;
            }
        if (sqk)
            break;
    }
    if (!sqk)
        return NLE_ERR_UNSUPPORTED;
    p.sqk = sqk;
    p.nsv = nsv;
    p.bars_off = (uint32_t)(sqk * p.qk_bytes + nsv * p.v_bytes);
    const size_t fixed = (size_t)nsv * p.v_bytes + bars_bytes;
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

    // Work split: a batch whose (block, head) items fit one per SM runs each
    // row tile as its own item (two chains per block at once); blocks <=
    // sum ceil(T_i / B) <= (T + n_seq (B - 1)) / B
    const long long items_bound = (total_frames + (long long)n_seq * (B - 1)) / B * heads;
    p.split = B > kQTile && (flags & NLE_FLAG_WHOLE_ITEMS) == 0 &&
              ((flags & NLE_FLAG_SPLIT_ITEMS) != 0 || items_bound <= di.sm_count);
    const long long work = p.split ? 2 * items_bound : max_items;
    if (p.split && 2 * items_bound > 0x7fffffffLL)
        return NLE_ERR_UNSUPPORTED;
    const KernelInfo kern = pick_kernel(NB);
    if (!nle::allow_max_dynamic_smem(reinterpret_cast<const void *>(kern.fn), dev, di.smem_optin))
        return NLE_ERR_CUDA;
    const int grid = (int)(work < di.sm_count ? work : di.sm_count);
    kern.fn<<<grid, kThreads, smem, static_cast<cudaStream_t>(stream)>>>(tq0, tq1, tk, tv, p);
    return cudaGetLastError() == cudaSuccess ? NLE_OK : NLE_ERR_CUDA;
}

extern "C" int nle_block_attn_fwd(const void *q, const void *k, const void *v, void *out, const int32_t *cu_seqlens,
                                  int n_seq, int64_t total_frames, int heads, int d_head, int block_frames,
                                  void *stream)
{
    return nle_block_attn_fwd_ex(q, k, v, out, cu_seqlens, n_seq, total_frames, heads, d_head, block_frames, 0.f,
                                 0, nullptr, 0, 0, stream);
}
