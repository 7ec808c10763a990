// attn_softmax.cuh -- register-segment softmax pieces shared by the block
// and full-utterance attention kernels (sm_100a): S is read from TMEM in
// segments of W columns (one fp32 per key, one row per lane), turned into
// p = exp2(S * scale * log2e - m) for a per-row shift m, packed to bf16 and
// written back over S's first columns as the A operand of the PV MMA.
#pragma once

#include "nle_device.cuh"

namespace nle {

// Softmax of one TMEM lane quarter of a tile (32 rows, one per lane).
//
// In the log2 domain (x = s * scale * log2e) every p of a row is
// exp2(x - m) for one shift m per row; softmax does not depend on m, which
// only has to keep p in range.  m starts as the max of the row's first 16
// keys, so the row's largest p is usually a small power above 1 (and exactly
// 1 for a one-key block).  While p is formed, the largest exponent x - m of
// the segment is tracked next to the exp; if any lane sees one above kYMax
// (or a NaN), the warp takes the rare path: m moves up by a whole number k so
// that the segment's max maps to 0, the segment is recomputed from the
// registers that still hold it, and the P already written are rescaled by
// 2^-k, an exact power of two.
//
// S is read from TMEM in register segments of SEG columns (a multiple of
// 16, so each segment's P covers whole PV K-steps); each segment's exps are
// one straight-line block.  P (bf16 pairs) is written back over S's first
// columns.
constexpr float kYMax = 32.f;

template <int W, int N>
__device__ __forceinline__ void seg_issue(uint32_t taddr, uint32_t (&s)[N])
{
    static_assert(W <= N && W % 16 == 0, "segment width");
#pragma unroll
    for (int c = 0; c + 32 <= W; c += 32)
        tmem_ld32_nowait(taddr + c, &s[c]);
    if constexpr (W % 32 == 16)
        tmem_ld16_nowait(taddr + W - 16, &s[W - 16]);
}

template <int W, int N>
__device__ __forceinline__ void seg_fence(uint32_t (&s)[N])
{
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

// Keys >= L (by index) -> -inf, branch-free (selects); only called for the
// segment that holds L.
template <int W, int N>
__device__ __forceinline__ void seg_mask(uint32_t (&s)[N], int c0, int L)
{
#pragma unroll
    for (int i = 0; i < W; ++i)
        s[i] = c0 + i < L ? s[i] : __float_as_uint(-INFINITY);
}

// Exact max of the first W values (rare path and the initial shift).
template <int W, int N>
__device__ __forceinline__ float seg_max(const uint32_t (&s)[N])
{
    float mx[8];
#pragma unroll
    for (int e = 0; e < 8; ++e)
        mx[e] = fmaxf(__uint_as_float(s[e]), __uint_as_float(s[8 + e]));
#pragma unroll
    for (int i = 16; i + 16 <= W; i += 16)
#pragma unroll
        for (int e = 0; e < 8; ++e)
            mx[e] = fmax3(mx[e], __uint_as_float(s[i + e]), __uint_as_float(s[i + 8 + e]));
    return fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
}

// p = exp2(s * sl2 - m) for the W keys (masked keys hold -inf -> 0), packed
// to bf16 pairs; returns the segment sum, and the largest exponent in ymax.
// Straight-line code: one basic block per segment keeps the exps of the
// whole segment in flight.
template <int W, int N>
__device__ __forceinline__ float seg_exp(const uint32_t (&s)[N], uint32_t (&pk)[W / 2], float sl2, float m,
                                         float &ymax)
{
    float ls[4] = {0.f, 0.f, 0.f, 0.f};
    float ym[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int j = 0; j < W / 2; ++j) {
        const float ya = fmaf(__uint_as_float(s[2 * j]), sl2, -m);
        const float yb = fmaf(__uint_as_float(s[2 * j + 1]), sl2, -m);
        ym[j & 3] = fmax3(ym[j & 3], ya, yb);
        const float a = ex2_approx(ya);
        const float b = ex2_approx(yb);
        ls[j & 3] += a + b;
        pk[j] = pack_bf16x2(a, b);
    }
    ymax = fmaxf(fmaxf(ym[0], ym[1]), fmaxf(ym[2], ym[3]));
    return (ls[0] + ls[1]) + (ls[2] + ls[3]);
}

// Multiply the bf16 P already in TMEM columns [0, ncols) by f, a power of
// two <= 1 (exact up to underflow); lanes with f = 1 rewrite P unchanged.
// Rare path; must be entered by the whole warp.
__device__ __forceinline__ void rescale_p(uint32_t tS, int ncols, float f)
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

// ------------------------------------------------------------ one-tile rows
// Rare path of one segment (whole warp): S of the segment is still intact
// in TMEM (its P has not been stored yet), so it is streamed again in
// 16-column chunks: first its max, then m moves up by a whole k so that max
// maps to <= 0, the segment's P is recomputed and stored, and the P already
// written (columns < C0/2) are rescaled by 2^-k.  A chunk's P (columns
// (C0+c)/2..+8) only overwrites S columns that have already been read.
template <int W>
__device__ __forceinline__ void softmax_rare(uint32_t tS, int C0, int L, float sl2, float &m, float &l)
{
    tmem_wait_ld();   // also completes a prefetch of the next segment
    float mx = -INFINITY;
#pragma unroll 1
    for (int c = 0; c < W; c += 16) {
        uint32_t r[16];
        tmem_ld16_nowait(tS + C0 + c, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            reg_fence(r[i]);
            if (C0 + c + i < L)
                mx = fmaxf(mx, __uint_as_float(r[i]));
        }
    }
    const float y = mx * sl2 - m;
    const int k = y > 0.f ? (int)ceilf(y) : 0;
    const float f = k <= 126 ? __int_as_float((127 - k) << 23) : 0.f;
    m += (float)k;
    l *= f;
#pragma unroll 1
    for (int c = 0; c < W; c += 16) {
        uint32_t r[16], pk[8];
        tmem_ld16_nowait(tS + C0 + c, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            reg_fence(r[2 * i]);
            reg_fence(r[2 * i + 1]);
            const float a = C0 + c + 2 * i < L ? ex2_approx(fmaf(__uint_as_float(r[2 * i]), sl2, -m)) : 0.f;
            const float b = C0 + c + 2 * i + 1 < L ? ex2_approx(fmaf(__uint_as_float(r[2 * i + 1]), sl2, -m)) : 0.f;
            l += a + b;
            pk[i] = pack_bf16x2(a, b);
        }
        tmem_st8p(tS + (C0 + c) / 2, pk);
        tmem_wait_st();
    }
    if (C0 > 0)
        rescale_p(tS, C0 / 2, f);
}

template <int NB, int SEG, int K>
__device__ __forceinline__ void softmax_step(uint32_t tS, int L, float sl2, float &m, float &l, uint32_t (&cur)[SEG])
{
    constexpr int C0 = K * SEG;
    constexpr int W = NB - C0 < SEG ? NB - C0 : SEG;
    constexpr int C1 = C0 + SEG;
    if (K > 0) {
        seg_issue<W>(tS + C0, cur);
        tmem_wait_ld();
        seg_fence<W>(cur);
    }
    if (C0 + W > L)   // warp-uniform
        seg_mask<W>(cur, C0, L);
    uint32_t pk[W / 2];
    float ymax;
    const float ls = seg_exp<W>(cur, pk, sl2, m, ymax);
    if (__any_sync(kFull, !(ymax <= kYMax))) {
        softmax_rare<W>(tS, C0, L, sl2, m, l);
    } else {
        l += ls;
        seg_store<W>(tS + C0 / 2, pk);
    }
    if constexpr (C1 < NB) {
        if (L > C1)
            softmax_step<NB, SEG, K + 1>(tS, L, sl2, m, l, cur);
    }
}

// Softmax of a whole row tile whose keys fit one S of NB <= 256 columns
// (the block kernels).  Returns this lane's row sum; P (bf16) is left over
// the first NB/2 columns of S.  Segments wholly at or past L are skipped (the MMAs stop at
// ceil16(L) keys).
template <int NB, int SEG>
__device__ __forceinline__ float block_softmax_rows(uint32_t tS, int L, float sl2)
{
    static_assert(SEG % 16 == 0 && SEG >= 16, "segments");
    constexpr int W0 = NB < SEG ? NB : SEG;
    uint32_t buf[SEG];
    seg_issue<W0>(tS, buf);
    tmem_wait_ld();
    seg_fence<W0>(buf);
    // first shift: max of the first 16 keys (keys >= L masked first)
    if (W0 > L)
        seg_mask<W0>(buf, 0, L);
    float m = fmax3(fmax3(__uint_as_float(buf[0]), __uint_as_float(buf[1]), __uint_as_float(buf[2])),
                    fmax3(__uint_as_float(buf[3]), __uint_as_float(buf[4]), __uint_as_float(buf[5])),
                    fmax3(__uint_as_float(buf[6]), __uint_as_float(buf[7]), __uint_as_float(buf[8])));
    m = fmax3(m, fmax3(__uint_as_float(buf[9]), __uint_as_float(buf[10]), __uint_as_float(buf[11])),
              fmax3(fmax3(__uint_as_float(buf[12]), __uint_as_float(buf[13]), __uint_as_float(buf[14])),
                    __uint_as_float(buf[15]), -INFINITY));
    m *= sl2;
    float l = 0.f;
    softmax_step<NB, SEG, 0>(tS, L, sl2, m, l, buf);
    tmem_wait_st();
    return l;
}

} // namespace nle
