// qkv_attn_sm100a.cu -- the QKV projection fused with varlen block
// self-attention on B200 (sm_100a).
//
// Operation (granite-speech-4.1-2b-nar model card, "Model Architecture" (1)
// CTC Speech Encoder: each conformer layer's self-attention projects its
// hidden states to queries, keys and values and attends within 4 s blocks of
// 200 encoder frames; "Usage / Installation": packed sequences,
// is_causal=False).  For every block of every packed utterance and every
// head h:
//     [Q_h | K_h | V_h] = bf16( X_blk W_h^T + b_h )      (fp32 accumulation)
//     O_blk,h = softmax(scale * Q_h K_h^T) V_h           (the block kernel)
// where W_h stacks rows h*64.., H*64 + h*64.. and 2*H*64 + h*64.. (64 each)
// of the linear layer's weight W [3*H*64][D] (output features x input
// features), and b the optional bias.  Q, K and V never leave the SM.
//
// Work split: the (head, frame) positions h * T + f are cut into one equal
// range per CTA; a CTA takes the (block, head) items whose first position
// lies in its range, so its items form runs of consecutive blocks of one
// head (one run, two where the range crosses a head).  The blocks of a run
// cover consecutive frames, so the run's projection is a plain row range of
// X: it is computed in tiles of 128 consecutive frames, whatever the block
// boundaries, and only the last tile of a run is ragged.
//
// Design (one persistent CTA per SM, 12 warps):
//   warp 0      walks the CTA's items, writes each block's descriptor into
//               one ring and each projection tile's into another, and
//               streams the projection operands in stages of 64 input
//               features: the tile's X box (128 frames x 64) and the head's
//               three 64-row W boxes (192 x 64), 128-byte swizzled, no
//               multicast.
//   warp 1      owns TMEM and issues the projection MMAs (lane 0):
//               D[128 x 192] += X_tile W_h^T, tcgen05.mma kind::f16, M=128,
//               N=192, K=16 x 4 per stage, fp32 accumulator in TMEM
//               columns 0..191.
//   warps 4-7   projection epilogue: each lane reads its frame's 192 columns
//               of D (+ bias), rounds them to bf16 in registers and releases
//               D at once, so the next tile's projection starts; it then
//               writes the row's q, k and v into the shared-memory buffers
//               of the block the frame belongs to (K-major Q and K, N-major
//               V, 128-byte swizzle), and hands a block to the attention
//               when its last frame is written.
//   warps 8-11  attention, as one tile warpgroup of the block kernel, on
//               TMEM columns 256..511: S = Q_x K^T (M=128, N=ceil16(L)), fp32
//               register softmax with one shift per row, P (bf16) over S,
//               O = P V (P from TMEM), O / rowsum rounded to bf16 and written
//               with 16-byte stores; rows past the block end are never
//               written.
// There is one Q/K buffer and two V buffers: the epilogue stores the q and
// k rows of a block once the previous block's last S MMA has completed, and
// its v rows once the last PV of the block two before has completed (blocks
// alternate between the V buffers); V rows L..ceil16(L)-1 (read by the PV
// MMA, weighted by zeros) are cleared.  Shared memory: Q (max(ceil16(B),
// 128) rows), K and two V buffers (ceil16(B) rows each) and three 40 KB
// stages for B = 200.
//
// Every mbarrier wait is bounded (see nle_device.cuh); on expiry the CTA
// drains its copies and MMAs in flight, frees TMEM and returns.
#include <cmath>

#include "nle.h"
#include "attn_softmax.cuh"
#include "nle_device.cuh"
#include "nle_host.h"

namespace {

using namespace nle;

constexpr int kThreads = 384;
constexpr int kEpi0 = 4;           // warps 4-7: projection epilogue
constexpr int kAttn0 = 8;          // warps 8-11: attention
constexpr int kSeg = 64;
constexpr int kQTile = 128;        // attention row tile
constexpr int kPTile = 128;        // projection tile: consecutive frames
constexpr int kRowBytes = 128;     // one frame of one head: 64 bf16
constexpr uint32_t kXBytes = 128 * 128;          // X box: 128 rows x 64 features
constexpr uint32_t kWBytes = 192 * 128;          // W boxes: 192 rows x 64 features
constexpr uint32_t kStageBytes = kXBytes + kWBytes;
constexpr int kMaxStages = 4;
constexpr int kDescRing = 8;
constexpr uint32_t kBlockReaders = 8;            // epilogue and attention warps
constexpr uint32_t kTileReaders = 5;             // warp 1 and the epilogue warps
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kDCol = 0;      // projection accumulator, 192 columns
constexpr uint32_t kSCol = 256;    // attention: S (<= 256 columns), P over S, O at +128
constexpr uint32_t kOCol = 128;

// A block (f0, L, head, run) or a projection tile (first frame, 1, head,
// run); L < 0 ends a ring.
struct Desc {
    int f0, L, h, run;
};

struct Bars {
    uint64_t st_full[kMaxStages];
    uint64_t st_empty[kMaxStages];   // the stage's MMAs have completed
    uint64_t d_full;                 // the tile's projection has completed
    uint64_t d_empty;                // 4 arrivals: the epilogue has read D
    uint64_t qkv_ready;              // 4 arrivals: a block's Q, K, V are in shared memory
    uint64_t qk_free;                // the block's last S MMA has completed (Q and K read)
    uint64_t v_free[2];              // per V buffer: a block's last PV MMA has completed (V read)
    uint64_t blk_full[kDescRing];
    uint64_t blk_empty[kDescRing];   // every reader has read the entry
    uint64_t tile_full[kDescRing];
    uint64_t tile_empty[kDescRing];
    uint64_t s_full, wg_p, o_full, wg_o;
    uint64_t mma_done[2];
    Desc blk[kDescRing];
    Desc tile[kDescRing];
    // the q, k and v bias rows of a run's head, by run parity: every
    // epilogue warp writes the copy of a run before its first tile (the same
    // values) and reads it through the run; the warps are less than one
    // tile apart, so no warp still reads a copy when it is rewritten
    uint4 bias[2][24];
    uint32_t tmem_base;
    int abort_flag;
};

struct Params {
    const int32_t *cu;
    int n_seq;
    int total;
    int heads;
    int B;            // block_frames
    int ksteps;       // input features / 64
    int nst;          // stage ring depth
    uint32_t k_off, v_off, v_size, st_off, bars_off;   // Q at 0, then K, V0, V1, stages, barriers
    const __nv_bfloat16 *bias;   // nullable, [3 * heads * 64]
    float scale_log2;
    __nv_bfloat16 *out;
    int out_stride;
    int32_t *status;
    unsigned long long wait_ns;
    int flags;
};

__device__ __forceinline__ uint64_t policy_evict_last()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t policy_evict_normal()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// The first unit whose first frame is >= F (units tile the utterances'
// frames in order; utterances flagged invalid by the walker hold none), or
// the number of units when there is none.  Queries must not decrease.
__device__ __forceinline__ long long first_unit_from(PlanWalker &w, int F, int lane)
{
    for (;;) {
        const bool in = w.base + lane < w.n_seq && w.len > 0 && w.start + w.len > F;
        const unsigned m = __ballot_sync(kFull, in);
        if (m) {
            const int src = __ffs(m) - 1;
            const int incl_s = __shfl_sync(kFull, w.incl, src);
            const int st = __shfl_sync(kFull, w.start, src);
            const int nb = __shfl_sync(kFull, w.units, src);
            const int j = F <= st ? 0 : (F - st + w.unit - 1) / w.unit;   // may be nb: the next utterance
            return (long long)w.before + (incl_s - nb) + j;
        }
        if (w.base + 32 >= w.n_seq)
            return (long long)w.before + w.group_units;
        w.before += w.group_units;
        w.base += 32;
        w.load_group(lane);
    }
}

// 64 fp32 accumulator columns of this lane's row (+ bias), rounded to bf16
// pairs in `pk`.  The TMEM loads are warp-collective: every lane of the warp
// calls this.
__device__ __forceinline__ void epi_load(uint32_t taddr, const uint4 *bias, uint32_t (&pk)[32])
{
    uint32_t v[64];
    tmem_ld32_nowait(taddr, &v[0]);
    tmem_ld32_nowait(taddr + 32, &v[32]);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 64; ++i)
        reg_fence(v[i]);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        float b[8];
        if (bias) {
            const uint4 bw = bias[c];
            const uint32_t bb[4] = {bw.x, bw.y, bw.z, bw.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                b[2 * e] = __uint_as_float(bb[e] << 16);
                b[2 * e + 1] = __uint_as_float(bb[e] & 0xffff0000u);
            }
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e)
                b[e] = 0.f;
        }
#pragma unroll
        for (int e = 0; e < 4; ++e)
            pk[4 * c + e] = pack_bf16x2(__uint_as_float(v[8 * c + 2 * e]) + b[2 * e],
                                        __uint_as_float(v[8 * c + 2 * e + 1]) + b[2 * e + 1]);
    }
}

// One 128-byte row of a 128-byte-swizzled operand buffer: the 16-byte chunk
// c of row r sits at chunk position c ^ (r & 7).
__device__ __forceinline__ void epi_store(const uint32_t (&pk)[32], uint8_t *row_dst, int r)
{
#pragma unroll
    for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4 *>(row_dst + ((c ^ (r & 7)) << 4)) =
            make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
}

template <int NB>
__global__ void __launch_bounds__(kThreads, 1)
    qkv_attn_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                    const Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t q_base = smem_u32(smem);
    const uint32_t k_base = q_base + p.k_off;
    const uint32_t v_base = q_base + p.v_off;
    const uint32_t st_base = q_base + p.st_off;
    Bars *bars = reinterpret_cast<Bars *>(smem + p.bars_off);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // ------------------------------------------------------------ set-up
    if (threadIdx.x == 0) {
        for (int s = 0; s < p.nst; ++s) {
            mbar_init(smem_u32(&bars->st_full[s]), 1);
            mbar_init(smem_u32(&bars->st_empty[s]), 1);
        }
        mbar_init(smem_u32(&bars->d_full), 1);
        mbar_init(smem_u32(&bars->d_empty), 4);
        mbar_init(smem_u32(&bars->qkv_ready), 4);
        mbar_init(smem_u32(&bars->qk_free), 1);
        mbar_init(smem_u32(&bars->v_free[0]), 1);
        mbar_init(smem_u32(&bars->v_free[1]), 1);
        for (int j = 0; j < kDescRing; ++j) {
            mbar_init(smem_u32(&bars->blk_full[j]), 1);
            mbar_init(smem_u32(&bars->blk_empty[j]), kBlockReaders);
            mbar_init(smem_u32(&bars->tile_full[j]), 1);
            mbar_init(smem_u32(&bars->tile_empty[j]), kTileReaders);
        }
        mbar_init(smem_u32(&bars->s_full), 1);
        mbar_init(smem_u32(&bars->wg_p), 4);
        mbar_init(smem_u32(&bars->o_full), 1);
        mbar_init(smem_u32(&bars->wg_o), 4);
        mbar_init(smem_u32(&bars->mma_done[0]), 1);
        mbar_init(smem_u32(&bars->mma_done[1]), 1);
        bars->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&bars->tmem_base), kTmemCols);
        tmem_relinquish();
    }
    if (threadIdx.x == 64) {
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_w);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    volatile int *abort_flag = &bars->abort_flag;
    const unsigned long long wait_ns = p.wait_ns;
    const int H = p.heads;
    const int KS = p.ksteps;

    // every reader of a descriptor ring: entry n, then release it
    auto read_ring = [&](uint64_t *full, uint64_t *empty, const Desc *ring, int n, Desc &d) -> bool {
        const int j = n % kDescRing;
        if (!wait_bar(smem_u32(&full[j]), (uint32_t)(n / kDescRing) & 1, abort_flag, wait_ns, p.status))
            return false;
        d = ring[j];
        __syncwarp();
        if (lane == 0)
            mbar_arrive(smem_u32(&empty[j]));
        return true;
    };

    if (warp == 0) {
        // ==================================================== producer
        const uint64_t pol_x = policy_evict_normal();   // X rows: read by the CTAs of every head
        const uint64_t pol_w = policy_evict_last();     // W: read by every tile
        const bool skip0 = (p.flags & NLE_FLAG_TEST_SKIP_FIRST_LOAD) != 0;
        uint32_t g = 0;        // stages issued
        int nblk = 0, ntile = 0;
        bool ok = true;
        auto publish = [&](uint64_t *full, uint64_t *empty, Desc *ring, int &n, const Desc &d) -> bool {
            const int j = n % kDescRing;
            if (n >= kDescRing && !wait_bar(smem_u32(&empty[j]), (uint32_t)(n / kDescRing - 1) & 1, abort_flag,
                                            wait_ns, p.status))
                return false;
            if (lane == 0) {
                ring[j] = d;
                mbar_arrive(smem_u32(&full[j]));
            }
            __syncwarp();
            ++n;
            return true;
        };
        // one projection tile: its descriptor, then its KS stages
        auto issue_tile = [&](int t0, int h, int run) -> bool {
            if (!publish(bars->tile_full, bars->tile_empty, bars->tile, ntile, Desc{t0, 1, h, run}))
                return false;
            for (int kb = 0; kb < KS; ++kb, ++g) {
                const int s = (int)(g % (uint32_t)p.nst);
                const uint32_t u = g / (uint32_t)p.nst;
                if (u > 0 && !wait_bar(smem_u32(&bars->st_empty[s]), (u - 1) & 1, abort_flag, wait_ns, p.status))
                    return false;
                if (lane == 0 && !(skip0 && g == 0)) {
                    const uint32_t bar = smem_u32(&bars->st_full[s]);
                    const uint32_t dst = st_base + (uint32_t)s * kStageBytes;
                    mbar_arrive_expect_tx(bar, kStageBytes);
                    tma_load_2d(dst, &tm_x, kb * 64, t0, bar, pol_x);
                    tma_load_2d(dst + kXBytes, &tm_w, kb * 64, h * 64, bar, pol_w);
                    tma_load_2d(dst + kXBytes + 8192, &tm_w, kb * 64, (H + h) * 64, bar, pol_w);
                    tma_load_2d(dst + kXBytes + 16384, &tm_w, kb * 64, (2 * H + h) * 64, bar, pol_w);
                }
                __syncwarp();
            }
            return true;
        };

        // this CTA's positions [lo, hi) of the H * total (head, frame) positions
        const long long HT = (long long)H * p.total;
        const long long lo = HT * (long long)blockIdx.x / (long long)gridDim.x;
        const long long hi = HT * ((long long)blockIdx.x + 1) / (long long)gridDim.x;
        int bad = 0;
        if (lo < hi) {
            int h = (int)(lo / p.total);
            PlanWalker w;
            w.init(p.cu, p.n_seq, p.total, p.B, lane);
            long long u = first_unit_from(w, (int)(lo % p.total), lane);
            int run = -1, run_h = -1, run_end = 0, next_t = 0;
            for (;;) {
                int f0, L, seq;
                if (!w.find(u, lane, f0, L, seq)) {
                    // past the last block of head h: the next head from its first block
                    bad |= w.bad;
                    if (++h >= H || (long long)h * p.total >= hi)
                        break;
                    w.init(p.cu, p.n_seq, p.total, p.B, lane);
                    u = 0;
                    continue;
                }
                if ((long long)h * p.total + f0 >= hi)
                    break;
                // a run: consecutive blocks of one head over consecutive frames
                if (h != run_h || f0 != run_end) {
                    ++run;
                    run_h = h;
                    next_t = f0;
                }
                run_end = f0 + L;
                if (!publish(bars->blk_full, bars->blk_empty, bars->blk, nblk, Desc{f0, L, h, run})) {
                    ok = false;
                    break;
                }
                // the tiles that hold this block's frames
                for (; next_t < run_end; next_t += kPTile)
                    if (!issue_tile(next_t, h, run)) {
                        ok = false;
                        break;
                    }
                if (!ok)
                    break;
                ++u;
            }
            bad |= w.bad;
        }
        if (bad && lane == 0)
            report(p.status, NLE_ERR_INVALID_ARG);
        if (ok) {   // end markers
            publish(bars->blk_full, bars->blk_empty, bars->blk, nblk, Desc{0, -1, 0, -1});
            publish(bars->tile_full, bars->tile_empty, bars->tile, ntile, Desc{0, -1, 0, -1});
        }
        // drain: the last copies of every stage must land before the CTA exits
        if (lane == 0) {
            const uint32_t nst = (uint32_t)p.nst;
            for (uint32_t m = g > nst ? g - nst : 0; m < g; ++m)
                if (!(skip0 && m == 0))
                    wait_bar_drain(smem_u32(&bars->st_full[m % nst]), (m / nst) & 1, wait_ns);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ==================================================== projection MMAs
        const uint32_t id_p = idesc_bf16_f32(128, 192, false);
        uint32_t g = 0, tiles_done = 0;
        for (int n = 0;; ++n) {
            Desc d;
            if (!read_ring(bars->tile_full, bars->tile_empty, bars->tile, n, d) || d.L < 0)
                break;
            if (tiles_done > 0 &&
                !wait_bar(smem_u32(&bars->d_empty), (tiles_done - 1) & 1, abort_flag, wait_ns, p.status))
                break;
            tc_fence_after();
            bool ok = true;
            for (int kb = 0; kb < KS; ++kb, ++g) {
                const int s = (int)(g % (uint32_t)p.nst);
                if (!wait_bar(smem_u32(&bars->st_full[s]), (g / (uint32_t)p.nst) & 1, abort_flag, wait_ns,
                              p.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a = st_base + (uint32_t)s * kStageBytes;
                const uint64_t da = smem_desc_sw128(a, 16, 1024);
                const uint64_t db = smem_desc_sw128(a + kXBytes, 16, 1024);
                if (lane == 0) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ss(tmem + kDCol, da + 2 * kk, db + 2 * kk, id_p, (kb | kk) ? 1u : 0u);
                    mma_commit(smem_u32(&bars->st_empty[s]));
                    if (kb == KS - 1)
                        mma_commit(smem_u32(&bars->d_full));
                }
                __syncwarp();
            }
            if (!ok)
                break;
            ++tiles_done;
        }
        if (lane == 0) {
            mma_commit(smem_u32(&bars->mma_done[0]));
            wait_bar_drain(smem_u32(&bars->mma_done[0]), 0, wait_ns);
        }
        __syncwarp();
    } else if (warp >= kEpi0 && warp < kAttn0) {
        // ==================================================== projection epilogue
        const int qq = warp & 3;
        const uint32_t tD = tmem + kDCol + ((uint32_t)(qq * 32) << 16);
        uint32_t tiles_done = 0;
        int bias_run = -1;
        int nb = 0;              // blocks handed to the attention
        int tn = 0, bn = 0;      // descriptors read
        Desc cb{0, -1, 0, -1};   // the block being filled
        bool have = false, claimed = false;
        bool ok = true;
        for (;;) {
            Desc td;
            if (!read_ring(bars->tile_full, bars->tile_empty, bars->tile, tn++, td)) {
                ok = false;
                break;
            }
            if (td.L < 0)
                break;
            if (!wait_bar(smem_u32(&bars->d_full), tiles_done & 1, abort_flag, wait_ns, p.status))
                break;
            tc_fence_after();
            // this lane's frame of the tile: its q, k and v, then D is free
            uint32_t pq[32], pk[32], pv[32];
            uint4 *rbias = bars->bias[td.run & 1];
            if (p.bias && td.run != bias_run) {
                if (lane < 24)
                    rbias[lane] = __ldg(reinterpret_cast<const uint4 *>(p.bias + (size_t)((lane >> 3) * H + td.h) * 64) +
                                        (lane & 7));
                __syncwarp();
                bias_run = td.run;
            }
            epi_load(tD, p.bias ? rbias : nullptr, pq);
            epi_load(tD + 64, p.bias ? rbias + 8 : nullptr, pk);
            epi_load(tD + 128, p.bias ? rbias + 16 : nullptr, pv);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_u32(&bars->d_empty));
            ++tiles_done;
            const int f = td.f0 + qq * 32 + lane;
            // the blocks of this run that hold frames of the tile, in order
            for (;;) {
                if (!have) {
                    if (!read_ring(bars->blk_full, bars->blk_empty, bars->blk, bn++, cb)) {
                        ok = false;
                        break;
                    }
                    have = true;
                    claimed = false;
                }
                if (cb.L < 0 || cb.run != td.run || cb.f0 >= td.f0 + kPTile)
                    break;   // it starts in a later tile
                const int r = f - cb.f0;
                const bool mine = r >= 0 && r < cb.L;
                // the previous block's attention must be done with the buffers
                if (!claimed && nb > 0 &&
                    !wait_bar(smem_u32(&bars->qk_free), (uint32_t)(nb - 1) & 1, abort_flag, wait_ns, p.status)) {
                    ok = false;
                    break;
                }
                if (mine) {
                    epi_store(pq, smem + (size_t)r * kRowBytes, r);
                    epi_store(pk, smem + p.k_off + (size_t)r * kRowBytes, r);
                }
                // V buffer nb & 1: the block two before must be done with it
                const uint32_t vb = (uint32_t)nb & 1;
                if (!claimed && nb > 1 &&
                    !wait_bar(smem_u32(&bars->v_free[vb]), (uint32_t)((nb >> 1) - 1) & 1, abort_flag, wait_ns,
                              p.status)) {
                    ok = false;
                    break;
                }
                claimed = true;
                uint8_t *vbuf = smem + p.v_off + vb * p.v_size;
                if (mine)
                    epi_store(pv, vbuf + (size_t)r * kRowBytes, r);
                if (cb.f0 + cb.L > td.f0 + kPTile)
                    break;   // the block goes on in the next tile
                // complete: clear V rows L..ceil16(L)-1, hand the block over
                const int zr = cb.L + qq * 32 + lane;
                if (zr < ((cb.L + 15) & ~15)) {
                    uint4 *z = reinterpret_cast<uint4 *>(vbuf + (size_t)zr * kRowBytes);
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        z[c] = make_uint4(0u, 0u, 0u, 0u);
                }
                fence_proxy_async_smem();   // the rows are read by the async proxy (MMAs)
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(smem_u32(&bars->qkv_ready));
                ++nb;
                have = false;
            }
            if (!ok)
                break;
        }
    } else if (warp >= kAttn0) {
        // ==================================================== attention
        const int qq = warp & 3;
        const bool leader = qq == 0;
        const uint32_t slot = tmem + kSCol;
        const uint32_t tS = slot + ((uint32_t)(qq * 32) << 16);
        const float sl2 = p.scale_log2;
        const uint32_t id_pv = idesc_bf16_f32(128, 64, true);
        int n = -1, x = 1, L = 0, f0 = 0, hcur = 0, nkeys = 16;
        uint32_t uses = 0;
        bool ok = true;

        // Next unit: row tile 1 of the block if it has one, else row tile 0
        // of the next block; the leader issues the unit's S MMA once the
        // previous unit's O has been read and, for a new block, its Q, K and
        // V are in shared memory.
        auto advance = [&]() -> bool {
            if (!(x == 0 && L > kQTile)) {
                ++n;
                Desc d;
                if (!read_ring(bars->blk_full, bars->blk_empty, bars->blk, n, d)) {
                    ok = false;
                    return false;
                }
                if (d.L < 0)
                    return false;
                f0 = d.f0;
                L = d.L;
                hcur = d.h;
                x = 0;
                nkeys = (L + 15) & ~15;
            } else {
                x = 1;
            }
            if (leader) {
                if (uses > 0 && !wait_bar(smem_u32(&bars->wg_o), (uses - 1) & 1, abort_flag, wait_ns, p.status)) {
                    ok = false;
                    return false;
                }
                if (x == 0 && !wait_bar(smem_u32(&bars->qkv_ready), (uint32_t)n & 1, abort_flag, wait_ns, p.status)) {
                    ok = false;
                    return false;
                }
                tc_fence_after();
                // A = Q rows of the row tile, B = K, both from shared memory
                const uint64_t da = smem_desc_sw128(q_base + (uint32_t)(x * kQTile * kRowBytes), 16, 1024);
                const uint64_t db = smem_desc_sw128(k_base, 16, 1024);
                const uint32_t id_s = idesc_bf16_f32(128, nkeys, false);
                if (lane == 0) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ss(slot, da + 2 * kk, db + 2 * kk, id_s, kk > 0 ? 1u : 0u);
                    mma_commit(smem_u32(&bars->s_full));
                    if (x == 1 || L <= kQTile)   // the block's last S: Q and K may be overwritten
                        mma_commit(smem_u32(&bars->qk_free));
                }
                __syncwarp();
            }
            return true;
        };

        uint32_t pk[32];
        bool pending = false;
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
            // ---------------------------------------------- softmax
            if (!wait_bar(smem_u32(&bars->s_full), uses & 1, abort_flag, wait_ns, p.status))
                break;
            tc_fence_after();
            const int row0 = x * kQTile + qq * 32;
            const bool active = row0 < L;
            float l = 1.f;
            if (active)
                l = block_softmax_rows<NB, kSeg>(tS, L, sl2);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_u32(&bars->wg_p));
            // ---------------------------------------------- O = P V
            if (leader) {
                if (!wait_bar(smem_u32(&bars->wg_p), uses & 1, abort_flag, wait_ns, p.status))
                    break;
                tc_fence_after();
                // V rows L..nkeys-1 are zeros (cleared by the epilogue)
                const uint64_t dv = smem_desc_sw128(v_base + ((uint32_t)n & 1) * p.v_size, 0, 1024);
                if (lane == 0) {
                    const int ksteps = nkeys / 16;
#pragma unroll
                    for (int kk = 0; kk < NB / 16; ++kk)
                        if (kk < ksteps)
                            mma_ts(slot + kOCol, slot + kk * 8, dv + (uint64_t)(kk * (16 * kRowBytes >> 4)), id_pv,
                                   kk > 0 ? 1u : 0u);
                    mma_commit(smem_u32(&bars->o_full));
                    if (x == 1 || L <= kQTile)   // the block's last PV: its V buffer may be overwritten
                        mma_commit(smem_u32(&bars->v_free[n & 1]));
                }
                __syncwarp();
            }
            // ---------------------------------------------- read O
            if (!wait_bar(smem_u32(&bars->o_full), uses & 1, abort_flag, wait_ns, p.status))
                break;
            tc_fence_after();
            if (active) {
                uint32_t o[64];
                tmem_ld32_nowait(tS + kOCol, &o[0]);
                tmem_ld32_nowait(tS + kOCol + 32, &o[32]);
                tmem_wait_ld();
                const float inv = 1.f / l;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    reg_fence(o[2 * i]);
                    reg_fence(o[2 * i + 1]);
                    pk[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_u32(&bars->wg_o));
            ++uses;
            pending = active;
            ef0 = f0;
            eL = L;
            eh = hcur;
            erow0 = row0;
        }
        if (leader) {
            if (lane == 0) {
                mma_commit(smem_u32(&bars->mma_done[1]));
                wait_bar_drain(smem_u32(&bars->mma_done[1]), 0, wait_ns);
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
using QkvKernel = void (*)(CUtensorMap, CUtensorMap, Params);

template <int NB>
QkvKernel qkv_kernel_nb()
{
    return reinterpret_cast<QkvKernel>(qkv_attn_kernel<NB>);
}

QkvKernel pick_qkv_kernel(int nb)
{
    switch (nb) {
    case 16: return qkv_kernel_nb<16>();
    case 32: return qkv_kernel_nb<32>();
    case 48: return qkv_kernel_nb<48>();
    case 64: return qkv_kernel_nb<64>();
    case 80: return qkv_kernel_nb<80>();
    case 96: return qkv_kernel_nb<96>();
    case 112: return qkv_kernel_nb<112>();
    case 128: return qkv_kernel_nb<128>();
    case 144: return qkv_kernel_nb<144>();
    case 160: return qkv_kernel_nb<160>();
    case 176: return qkv_kernel_nb<176>();
    case 192: return qkv_kernel_nb<192>();
    case 208: return qkv_kernel_nb<208>();
    case 224: return qkv_kernel_nb<224>();
    case 240: return qkv_kernel_nb<240>();
    default: return qkv_kernel_nb<256>();
    }
}

} // namespace

extern "C" int nle_block_attn_qkv_fwd_ex(const void *x, const void *w_qkv, const void *bias, void *out,
                                         const int32_t *cu_seqlens, int n_seq, int64_t total_frames, int d_model,
                                         int heads, int d_head, int block_frames, float softmax_scale,
                                         int32_t *dev_status, int flags, int64_t wait_limit_ns, void *stream)
{
    if (n_seq < 0 || total_frames < 0 || heads <= 0 || block_frames <= 0 || d_model <= 0 || wait_limit_ns < 0)
        return NLE_ERR_INVALID_ARG;
    if (d_head != 64 || block_frames > 256 || d_model % 64 != 0 || d_model > 16384 ||
        total_frames > 0x7fffffffLL || (int64_t)3 * heads * 64 > 0x7fffffffLL)
        return NLE_ERR_UNSUPPORTED;
    const long long max_items = ((long long)n_seq + total_frames / block_frames) * heads;
    if (max_items > 0x7fffffffLL)
        return NLE_ERR_UNSUPPORTED;
    if (n_seq == 0 || total_frames == 0)
        return NLE_OK;
    if (!x || !w_qkv || !out || !cu_seqlens)
        return NLE_ERR_INVALID_ARG;
    if (!nle::aligned16(x) || !nle::aligned16(w_qkv) || !nle::aligned16(out) || (bias && !nle::aligned16(bias)))
        return NLE_ERR_MISALIGNED;

    nle::DeviceInfo di;
    int dev = 0;
    if (!nle::current_device_info(&di, &dev))
        return NLE_ERR_CUDA;
    if (di.cc_major != 10)
        return NLE_ERR_UNSUPPORTED;

    const double scale = softmax_scale > 0.f ? (double)softmax_scale : 1.0 / std::sqrt((double)d_head);
    const unsigned long long wns = wait_limit_ns > 0 ? (unsigned long long)wait_limit_ns : 1000000000ull;
    const int B = block_frames;
    const int NB = (B + 15) / 16 * 16;
    Params p{};
    p.cu = cu_seqlens;
    p.n_seq = n_seq;
    p.total = (int)total_frames;
    p.heads = heads;
    p.B = B;
    p.ksteps = d_model / 64;
    // shared memory: Q (NB rows, at least the 128 an S MMA reads; the S MMA
    // of row tile 1 reads rows up to 255, past NB into K, whose results
    // belong to rows past the block end and are never written), K (NB rows),
    // two V buffers (NB rows each), the stage ring, the barriers
    const uint32_t q_bytes = (uint32_t)(NB > kQTile ? NB : kQTile) * kRowBytes;
    const uint32_t kv_bytes = (uint32_t)NB * kRowBytes;
    p.k_off = q_bytes;
    p.v_off = q_bytes + kv_bytes;
    p.v_size = kv_bytes;
    p.st_off = (q_bytes + 3 * kv_bytes + 1023) & ~1023u;
    const size_t bars_round = ((sizeof(Bars) + 127) / 128) * 128;
    int nst = 0;
    for (int s = kMaxStages; s >= 2; --s)
        if ((size_t)p.st_off + (size_t)s * kStageBytes + bars_round + 1024 <= (size_t)di.smem_optin) {
            nst = s;
            break;
        }
    if (!nst)
        return NLE_ERR_UNSUPPORTED;
    p.nst = nst;
    p.bars_off = p.st_off + (uint32_t)nst * kStageBytes;
    size_t smem = (size_t)p.bars_off + bars_round + 1024;
    // one CTA per SM: it owns all 512 TMEM columns
    if (smem <= (size_t)di.smem_optin / 2)
        smem = (size_t)di.smem_optin / 2 + 1024;
    p.bias = static_cast<const __nv_bfloat16 *>(bias);
    p.scale_log2 = (float)(scale * 1.4426950408889634);
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.out_stride = heads * 64;
    p.status = dev_status;
    p.wait_ns = wns;
    p.flags = flags;

    CUtensorMap tx, tw;
    if (!nle::encode_tmap_bf16_2d(&tx, x, (uint64_t)d_model, (uint64_t)total_frames, (uint64_t)d_model, 64, 128) ||
        !nle::encode_tmap_bf16_2d(&tw, w_qkv, (uint64_t)d_model, (uint64_t)3 * heads * 64, (uint64_t)d_model, 64,
                                  64))
        return NLE_ERR_CUDA;

    const QkvKernel kern = pick_qkv_kernel(NB);
    if (!nle::allow_max_dynamic_smem(reinterpret_cast<const void *>(kern), dev, di.smem_optin))
        return NLE_ERR_CUDA;
    const int grid = (int)(max_items < di.sm_count ? max_items : di.sm_count);
    kern<<<grid, kThreads, smem, static_cast<cudaStream_t>(stream)>>>(tx, tw, p);
    return cudaGetLastError() == cudaSuccess ? NLE_OK : NLE_ERR_CUDA;
}

extern "C" int nle_block_attn_qkv_fwd(const void *x, const void *w_qkv, const void *bias, void *out,
                                      const int32_t *cu_seqlens, int n_seq, int64_t total_frames, int d_model,
                                      int heads, int d_head, int block_frames, void *stream)
{
    return nle_block_attn_qkv_fwd_ex(x, w_qkv, bias, out, cu_seqlens, n_seq, total_frames, d_model, heads, d_head,
                                     block_frames, 0.f, nullptr, 0, 0, stream);
}
