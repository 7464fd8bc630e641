// Large-M block-scaled FP4 GEMM kernels (tcgen05 + TMEM + TMA) with the
// per-segment global-scale epilogue; see gemm_common.cuh for the product they
// compute.
#pragma once

#include "gemm_common.cuh"
#include "quant.cuh"

namespace nvfp4 {

// ===========================================================================
// Large-M kernel (one CTA per SM, 128 x 256 tiles, 256-deep K stages)
//
// Warp roles (16 warps):
//   0      TMA producer: A/B tiles and the stage's scale atoms into a 4-stage ring
//   1      MMA issuer: tcgen05 block-scaled MMAs (M=128, N=256, K=64)
//   2      owns the TMEM allocation (with the activation quantisation fused
//          in, 2..3 quantise A in the background, and 2..15 its first bands)
//   4..11  epilogue: drain the accumulator, scale by s_ga * s_gw[segment],
//          convert and store 16 x 32 chunks through shared memory with TMA
//   12..15 scale staging: read each stage's scale atoms from shared memory and
//          write them into TMEM with tcgen05.st (one warp per 32-lane quadrant,
//          every quadrant receiving the full atom), keeping the tensor pipe free
//          for MMAs
//
// TMEM (512 columns): two 256-column accumulators overlapping by 96 columns,
// ACC0 = [0, 256) and ACC1 = [160, 416), and two 48-column scale slots at
// [416, 512).  Consecutive tiles alternate accumulators; the epilogue drains
// the shared columns first and releases them, so the next tile's MMAs start
// while the rest of the previous tile is still being drained.  (A larger
// overlap with more scale slots, [64, 320) and four slots, measured slower:
// the longer drain before the next tile's first MMA costs more than the
// deeper scale staging gains.)
// ===========================================================================
// Overlap plan for accumulators ACC0 = [0, 256) and ACC1 = [A1, A1 + 256)
// (A1 a multiple of 32): the 32-column chunks of each epilogue warp's
// 128-column half that the other accumulator also uses.  They are drained
// first, starting at chunk rot(b, h); after count(b, h) of them the warp
// releases the overlap (count 0: the warp holds none).
template <int A1>
struct Overlap {
    static constexpr int b0_from = A1 / 32;          // ACC0 chunks >= b0_from are shared
    static constexpr int b1_to = (256 - A1) / 32;    // ACC1 chunks < b1_to are shared
    __host__ __device__ static constexpr int clamp4(int x) { return x < 0 ? 0 : (x > 4 ? 4 : x); }
    __host__ __device__ static constexpr int count(int b, int h)
    {
        return b == 0 ? clamp4(4 * h + 4 - (b0_from > 4 * h ? b0_from : 4 * h))
                      : clamp4((b1_to < 4 * h + 4 ? b1_to : 4 * h + 4) - 4 * h);
    }
    __host__ __device__ static constexpr int rot(int b, int h)
    {
        return (b == 0 && count(0, h) > 0 && b0_from > 4 * h) ? (b0_from - 4 * h) & 3 : 0;
    }
    // warps that release the overlap per tile (the same for both accumulators)
    __host__ __device__ static constexpr int warps() { return 4 * ((count(0, 0) > 0) + (count(0, 1) > 0)); }
    static_assert(A1 % 32 == 0 && A1 > 0 && A1 < 256, "overlap");
    static_assert(4 * ((count(0, 0) > 0) + (count(0, 1) > 0)) == 4 * ((count(1, 0) > 0) + (count(1, 1) > 0)),
                  "both accumulators release through the same number of warps");
};

// Scale and pack one 32-column chunk J of a warp's accumulator slice into
// BF16 pairs.
template <int J>
__device__ __forceinline__ void convert_chunk(const uint32_t (&v)[32], int ncol0, float s_ga, const GemmParams& p,
                                              uint32_t (&packed)[4][16])
{
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int col = ncol0 + J * 32 + h * 16;
        const float alpha = __fmul_rn(s_ga, segment_scale(p.segs, col < p.n ? col : p.n - 1));
#pragma unroll
        for (int e = 0; e < 8; ++e)
            packed[J][h * 8 + e] = pack_bf16x2(__fmul_rn(__uint_as_float(v[h * 16 + 2 * e]), alpha),
                                               __fmul_rn(__uint_as_float(v[h * 16 + 2 * e + 1]), alpha));
    }
}

// Drain one warp's 32 x 128 slice of an accumulator into scaled BF16 pairs,
// 32 columns at a time starting with chunk ROT (compile-time so the results
// stay in registers).  The first AFTER chunks (0: none) are the columns the
// other accumulator shares: the next tile's MMAs wait for them, so they are
// loaded together with one wait, then the warp calls `release()`, and only
// then are they converted.  (Loading and converting them one at a time kept
// the tensor pipe idle ~6 % longer at every tile boundary.)
template <int ROT, int AFTER, typename Release>
__device__ __forceinline__ void drain_bf16(uint32_t taddr, int ncol0, float s_ga, const GemmParams& p,
                                           Release release, int lane, uint32_t (&packed)[4][16])
{
    static_assert(AFTER == 0 || AFTER == 3, "overlap plans drain 0 or 3 shared chunks");
    constexpr int J0 = ROT & 3, J1 = (ROT + 1) & 3, J2 = (ROT + 2) & 3, J3 = (ROT + 3) & 3;
    uint32_t v0[32], v1[32], v2[32];
    if constexpr (AFTER == 3) {
        tmem_ld_32x32b_x32(taddr + J0 * 32, v0);
        tmem_ld_32x32b_x32(taddr + J1 * 32, v1);
        tmem_ld_32x32b_x32(taddr + J2 * 32, v2);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) release();
    } else {
        tmem_ld_32x32b_x32(taddr + J0 * 32, v0);
        tmem_ld_32x32b_x32(taddr + J1 * 32, v1);
        tmem_ld_32x32b_x32(taddr + J2 * 32, v2);
        tmem_ld_wait();
    }
    convert_chunk<J0>(v0, ncol0, s_ga, p, packed);
    convert_chunk<J1>(v1, ncol0, s_ga, p, packed);
    convert_chunk<J2>(v2, ncol0, s_ga, p, packed);
    tmem_ld_32x32b_x32(taddr + J3 * 32, v0);
    tmem_ld_wait();
    convert_chunk<J3>(v0, ncol0, s_ga, p, packed);
}

// Dispatch drain_bf16 on the (accumulator, half) overlap plan.
template <int A1, typename Release>
__device__ __forceinline__ void drain_bf16_plan(int b, int half, uint32_t taddr, int ncol0, float s_ga,
                                                const GemmParams& p, Release release, int lane,
                                                uint32_t (&packed)[4][16])
{
    using OV = Overlap<A1>;
    if (b == 0) {
        if (half == 0)
            drain_bf16<OV::rot(0, 0), OV::count(0, 0)>(taddr, ncol0, s_ga, p, release, lane, packed);
        else
            drain_bf16<OV::rot(0, 1), OV::count(0, 1)>(taddr, ncol0, s_ga, p, release, lane, packed);
    } else {
        if (half == 0)
            drain_bf16<OV::rot(1, 0), OV::count(1, 0)>(taddr, ncol0, s_ga, p, release, lane, packed);
        else
            drain_bf16<OV::rot(1, 1), OV::count(1, 1)>(taddr, ncol0, s_ga, p, release, lane, packed);
    }
}

// Gated DeltaNet gates of the warp's 32 x 128 slice, after its stores: the
// chunks holding gate columns go through the staging buffer once more (j
// picked at run time; each switch arm indexes `packed` with constants, so it
// stays in registers) and gdn_chunk reads them there.  One copy of the gate
// code per kernel, outside the unrolled store loop.
template <int J>
__device__ __forceinline__ void stage_chunk_row(uint8_t* cbuf, const uint32_t (&packed)[4][16], int r)
{
#pragma unroll
    for (int u = 0; u < 4; ++u)
        *reinterpret_cast<uint4*>(cbuf + r * 64 + ((u ^ ((r >> 1) & 3)) << 4)) =
            make_uint4(packed[J][4 * u], packed[J][4 * u + 1], packed[J][4 * u + 2], packed[J][4 * u + 3]);
}

__device__ __forceinline__ void gdn_pass(const GemmParams& p, uint8_t* cbuf, const uint32_t (&packed)[4][16], int row0,
                                         int ncol0, int lane)
{
    if (lane == 0) bulk_wait_group_read<0>();  // the last TMA store has read the buffer
    __syncwarp();
#pragma unroll 1
    for (int q = 0; q < 8; ++q) {
        const int j = q >> 1, hr = q & 1;
        if (!gdn_touches(p, ncol0 + j * 32, 32)) continue;
        if ((lane >> 4) == hr) {
            const int r = lane & 15;
            switch (j) {
                case 0: stage_chunk_row<0>(cbuf, packed, r); break;
                case 1: stage_chunk_row<1>(cbuf, packed, r); break;
                case 2: stage_chunk_row<2>(cbuf, packed, r); break;
                default: stage_chunk_row<3>(cbuf, packed, r); break;
            }
        }
        __syncwarp();
        gdn_chunk(p, cbuf, row0 + 16 * hr, ncol0 + j * 32, lane);
        __syncwarp();
    }
}

// Stage unit (chunk j, row half hr) of `packed` into a 16 x 32 buffer: the
// 16 lanes of that half each write their row.
__device__ __forceinline__ void stage_unit(uint8_t* buf, const uint32_t (&packed)[4][16], int j, int hr, int lane)
{
    if ((lane >> 4) != hr) return;
    const int r = lane & 15;
    switch (j) {
        case 0: stage_chunk_row<0>(buf, packed, r); break;
        case 1: stage_chunk_row<1>(buf, packed, r); break;
        case 2: stage_chunk_row<2>(buf, packed, r); break;
        default: stage_chunk_row<3>(buf, packed, r); break;
    }
}

// The gate pass when only one half of a tile (owner_half) holds gate columns:
// the two epilogue warps of the quadrant share it.  The owner holds the
// values; unit by unit (16 rows x 32 columns) it stages one unit into its
// own 1 KB buffer and the next into its partner's, and each warp computes the
// gates of the unit in its buffer (named barrier 10 + quad between the two
// warps).  In the fused GDN in-proj the gate columns all fall in one half of
// the last tile column, whose other half lies past N, so this halves the gate
// work per warp.
__device__ __forceinline__ void gdn_pass_shared(const GemmParams& p, uint8_t* cbase, int c_warp,
                                                const uint32_t (&packed)[4][16], int row0, int nb0, int quad,
                                                int half, int owner_half, int lane)
{
    uint8_t* own_buf = cbase + (owner_half * 4 + quad) * c_warp;
    uint8_t* help_buf = cbase + ((1 - owner_half) * 4 + quad) * c_warp;
    const int ncol0 = nb0 + owner_half * 128;
    const bool is_owner = half == owner_half;
    const int bar = 10 + quad;
    if (lane == 0) bulk_wait_group_read<0>();  // this warp's last TMA store has read its buffer
    __syncwarp();
    named_barrier_sync(bar, 64);               // both buffers are free
    int k = 0, pj = -1, phr = 0;
#pragma unroll 1
    for (int q = 0; q < 8; ++q) {
        const int j = q >> 1, hr = q & 1;
        if (!gdn_touches(p, ncol0 + j * 32, 32)) continue;
        if ((k & 1) == 0) {
            if (is_owner) stage_unit(own_buf, packed, j, hr, lane);
            pj = j;
            phr = hr;
        } else {
            if (is_owner) stage_unit(help_buf, packed, j, hr, lane);
            named_barrier_sync(bar, 64);       // staged
            if (is_owner) gdn_chunk(p, own_buf, row0 + 16 * phr, ncol0 + pj * 32, lane);
            else gdn_chunk(p, help_buf, row0 + 16 * hr, ncol0 + j * 32, lane);
            named_barrier_sync(bar, 64);       // read: the buffers may be restaged
            pj = -1;
        }
        ++k;
    }
    if (pj >= 0) {
        named_barrier_sync(bar, 64);
        if (is_owner) gdn_chunk(p, own_buf, row0 + 16 * phr, ncol0 + pj * 32, lane);
        named_barrier_sync(bar, 64);
    }
}

namespace large {
constexpr int BM = 128, BN = 256, BK_BYTES = 128;  // BK = 256 FP4 values per stage
constexpr int STAGES = 4;
constexpr int KSTEPS = 4;                          // MMAs (K = 64) per stage
constexpr int A_STAGE = BM * BK_BYTES;             // 16 KB
constexpr int B_STAGE = BN * BK_BYTES;             // 32 KB
constexpr int SFA_STAGE = 4 * 512;                 // 4 atoms of 128 rows
constexpr int SFB_STAGE = 2 * 4 * 512;             // 2 row blocks x 4 atoms
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + STAGES * A_STAGE;
constexpr int OFF_SFA = OFF_B + STAGES * B_STAGE;
constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_STAGE;
constexpr int OFF_C = OFF_SFB + STAGES * SFB_STAGE;
constexpr int C_WARP = 1024;                       // per epilogue warp: one 16 x 32 BF16 chunk
constexpr int OFF_BAR = OFF_C + 8 * C_WARP;
constexpr int SF_SLOTS = 2;
// full[S], empty[S], sf_ready[SLOTS], acc_full[2], acc_empty[2], ovl_free, drain
constexpr int NUM_BARS = 2 * STAGES + SF_SLOTS + 2 + 2 + 1 + 1;
constexpr int OFF_TMEM_PTR = OFF_BAR + NUM_BARS * 8;
constexpr int SMEM_BYTES = OFF_TMEM_PTR + 16 + 1024;  // + alignment slack
constexpr int THREADS = 512;
constexpr int TMEM_COLS = 512;
constexpr int ACC1_COL = 160;                         // ACC0 at 0; overlap [160, 256)
constexpr int SF_COL = 416;                           // two scale slots of 48 columns
constexpr int SF_SLOT = 48;                           // 16 (A: 4 k-steps x 4) + 32 (B: 4 x 8)
static_assert(ACC1_COL + BN <= SF_COL && SF_COL + SF_SLOTS * SF_SLOT <= TMEM_COLS, "TMEM budget");
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
}  // namespace large

// ---------------------------------------------------------------------------
// Activation quantisation fused into the large-M kernel (QA): one launch
// quantises the raw BF16 activations and multiplies them.  The tiles run in
// bands of qa::BAND m-blocks (column-major inside a band), so the first wave
// of tiles needs only the first m-blocks of A.  Those are quantised before the
// mainloop by every warp but the producer and the MMA issuer, across all
// CTAs; warps 2 and 3 then quantise the remaining m-blocks, in order, while
// the MMAs run.  Each CTA counts itself into m-block j's ready word once its
// share of j is stored; a producer loads rows of A only from m-blocks whose
// word shows every CTA (the word carries a per-call tag that grows from call
// to call; the workspace is zeroed once before its first use).  The
// quantisation is quantize_kernel's, item for item, so
// codes, scales and the GEMM output are bit-identical to the two launches.
// ---------------------------------------------------------------------------
namespace qa {
constexpr int BAND = 8;            // m-blocks per band of the tile order
constexpr int FIRST_ITEMS = 2;     // warp-chunks of 32 items in flight per lane, warps 2..15
constexpr int BG_ITEMS = 4;        // the same, warps 2..3 (more bytes in flight for fewer warps)
constexpr int FIRST_WARPS = 14;    // warps 2..15 quantise the first m-blocks
constexpr int BG_WARPS = 2;        // warps 2..3 quantise the rest, a band at a time
constexpr int BAR_FIRST = 8, BAR_BG = 9;  // named barriers
}  // namespace qa

// Tile t of the persistent schedule -> (m-block, n-block).
template <bool QA>
__device__ __forceinline__ void tile_mn(int t, const GemmParams& p, int& mb, int& nb)
{
    if (!QA) {
        mb = t % p.m_tiles;
        nb = t / p.m_tiles;
        return;
    }
    const int band_tiles = qa::BAND * p.n_tiles;
    const int band = t / band_tiles;
    const int r = t - band * band_tiles;
    const int bsz = min(qa::BAND, p.m_tiles - band * qa::BAND);
    nb = r / bsz;
    mb = band * qa::BAND + (r - nb * bsz);
}

// Quantise this warp's chunks of m-blocks [mb0, mb1): chunk c covers the 32
// items (row, block pair) 32c' .. 32c' + 31 of m-block mb0 + c / (4 pairs),
// c' = c mod (4 pairs), numbered row-major over its 128 rows x pairs (2 *
// katoms) as in quantize_kernel, one item per lane.  The warp takes chunks c0,
// c0 + stride, ..., ITEMS of them at a time with all their loads issued first.
// Every lane fences its stores for the async proxy.
template <int ITEMS>
__device__ __forceinline__ void qa_quantize_range(const GemmParams& p, const QuantParams& qp, const QuantLaunch& ql,
                                                  int mb0, int mb1, int c0, int stride, int lane, float s_g)
{
    const uint32_t pairs = ql.pairs;
    const int per_mb = (int)(4u * pairs);    // 128 rows x pairs items / 32
    const int chunks = (mb1 - mb0) * per_mb;
    const int64_t nb16 = p.k >> 4;
    for (int c = c0; c < chunks; c += stride * ITEMS) {
        uint4 u[ITEMS][4];
        bool have[ITEMS], live0[ITEMS], live1[ITEMS];
        uint32_t pr[ITEMS];
        int64_t r[ITEMS], kb0[ITEMS];
#pragma unroll
        for (int i = 0; i < ITEMS; ++i) {
            const int ci = c + i * stride;
            have[i] = ci < chunks;               // the same for every lane
            const int cc = have[i] ? ci : 0;
            const int mbi = cc / per_mb;
            const uint32_t item = (uint32_t)(cc - mbi * per_mb) * 32u + (uint32_t)lane;
            const uint32_t rl = item / pairs;
            pr[i] = item - rl * pairs;
            r[i] = (int64_t)(mb0 + mbi) * 128 + rl;
            kb0[i] = (int64_t)pr[i] * 2;
            const bool row_live = have[i] && r[i] < p.m;
            live0[i] = row_live && kb0[i] < nb16;
            live1[i] = row_live && kb0[i] + 1 < nb16;
            const uint4* src =
                reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.a_in) + r[i] * p.lda + kb0[i] * 16);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                u[i][j] = ((j < 2) ? live0[i] : live1[i]) ? __ldcs(src + j) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int i = 0; i < ITEMS; ++i) {
            if (!have[i]) continue;
            float v0[16], v1[16];
            unpack_bf16x8(u[i][0], v0);
            unpack_bf16x8(u[i][1], v0 + 8);
            unpack_bf16x8(u[i][2], v1);
            unpack_bf16x8(u[i][3], v1 + 8);
            quantize_pair_store(qp, ql, true, pr[i], r[i], kb0[i], live0[i], live1[i], s_g, v0, v1);
        }
    }
    fence_proxy_async_global();
}

// Count this CTA into m-block mb's ready word: the call tag in the high half
// (raised to this call's by the maximum: tags grow from call to call and the
// workspace starts at zero), CTAs done in the low half.  Two atomics, no
// retry loop, so 148 CTAs marking one word cost 296 serialised updates.  The
// caller has synchronised with every thread that stored part of this CTA's
// share.
__device__ __forceinline__ void qa_mark_ready(const GemmParams& p, int mb)
{
    unsigned long long* w = p.qa_ready + mb;
    __threadfence();
    atomicMax(w, (unsigned long long)(uint32_t)p.epoch << 32);
    atomicAdd(w, 1ull);
}

// Warp-collective: wait (bounded) until m-blocks [ready_below, mb] are ready,
// advancing ready_below over every ready m-block found (32 per look).  Then
// the TMA loads this warp issues see the quantised rows.
__device__ __forceinline__ bool qa_wait_ready(const GemmParams& p, int& ready_below, int mb, int lane)
{
    const unsigned long long want = ((unsigned long long)(uint32_t)p.epoch << 32) | gridDim.x;
    const long long t0 = clock64();
    while (ready_below <= mb) {
        const int j = ready_below + lane;
        const bool ok = j >= p.m_tiles || ld_volatile_u64(p.qa_ready + j) == want;
        const unsigned bad = __ballot_sync(0xffffffffu, !ok);
        ready_below = min(ready_below + (bad ? __ffs(bad) - 1 : 32), p.m_tiles);
        if (ready_below > mb) break;
        if (clock64() - t0 > kWaitCycles) {
            if (lane == 0) record_status(kStatusTimeoutQuant);
            return false;
        }
        __nanosleep(256);   // back off: 148 producers poll the same few words
    }
    __threadfence();
    fence_proxy_async_global();
    return true;
}

// SwiGLU epilogue, first half: the warp's two gate chunks and two up chunks
// (items 0, 1: gate g2 = 0, 1 = chunks 2 HALF + g2; items 2, 3: up = those + 4)
// as the BF16 values the unfused GEMM would store, packed in pairs.  The
// chunks the other accumulator shares (ACC0: chunk >= 5, ACC1: chunk <= 2)
// are loaded first, together, and released before anything else, so the next
// tile's MMAs do not wait for this warp's arithmetic; then the rest, one at a
// time, and the accumulator is released.
template <int B, int HALF, typename Release, typename Done>
__device__ __forceinline__ void swiglu_load(uint32_t tacc, int hcol0, float s_ga, const GemmParams& p, int lane,
                                            Release release, Done done, uint32_t (&gp)[2][16], uint32_t (&up)[2][16])
{
    auto chunk = [](int it) { return 2 * HALF + (it & 1) + (it >= 2 ? 4 : 0); };
    auto shared = [&](int it) { return B ? chunk(it) <= 2 : chunk(it) >= 5; };
    auto to_bf16 = [&](const uint32_t (&v)[32], int it, uint32_t (&o)[16]) {
        const int col = (it >= 2 ? p.swiglu_f : 0) + hcol0 + 32 * (it & 1);
        const float a0 = __fmul_rn(s_ga, segment_scale(p.segs, col));
        const float a1 = __fmul_rn(s_ga, segment_scale(p.segs, col + 16));
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            o[e] = pack_bf16x2(__fmul_rn(__uint_as_float(v[2 * e]), a0), __fmul_rn(__uint_as_float(v[2 * e + 1]), a0));
            o[8 + e] = pack_bf16x2(__fmul_rn(__uint_as_float(v[16 + 2 * e]), a1),
                                   __fmul_rn(__uint_as_float(v[16 + 2 * e + 1]), a1));
        }
    };
    auto dst = [&](int it) -> uint32_t(&)[16] { return it >= 2 ? up[it & 1] : gp[it & 1]; };
    // the shared items (one or two; every warp holds at least one)
    constexpr int S0 = (B ? (2 * HALF + 0 <= 2) : false) ? 0 : (B ? (2 * HALF + 1 <= 2 ? 1 : -1) : (2 * HALF + 4 >= 5 ? 2 : 3));
    static_assert(S0 >= 0, "every epilogue warp holds a shared chunk");
    constexpr int S1 = B ? ((S0 == 0 && 2 * HALF + 1 <= 2) ? 1 : -1) : ((S0 == 2) ? 3 : -1);
    {
        uint32_t va[32], vb[32];
        tmem_ld_32x32b_x32(tacc + chunk(S0) * 32, va);
        if constexpr (S1 >= 0) tmem_ld_32x32b_x32(tacc + chunk(S1) * 32, vb);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) release();
        to_bf16(va, S0, dst(S0));
        if constexpr (S1 >= 0) to_bf16(vb, S1, dst(S1));
    }
#pragma unroll
    for (int it = 0; it < 4; ++it) {
        if (it == S0 || it == S1) continue;
        uint32_t v[32];
        tmem_ld_32x32b_x32(tacc + chunk(it) * 32, v);
        tmem_ld_wait();
        to_bf16(v, it, dst(it));
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) done();
}

// SWIGLU: the gate/up GEMM of a gated MLP with its glue fused into the
// epilogue.  Each 128 x 256 tile holds 128 gate columns (accumulator columns
// 0..127) and the matching 128 up columns (128..255), loaded as two 128-row
// boxes of the [gate; up] weight; the epilogue forms
// h = bf16(silu(bf16(g)) * bf16(u)) exactly as the unfused GEMM (BF16 output)
// followed by silu_mul_quantize_kernel would, and quantises it with the
// static scale h_scale, writing codes and tiled scales instead of C.
template <bool SWIGLU, bool QA = false>
__global__ void __launch_bounds__(large::THREADS, 1)
    gemm_large_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_w,
                      const __grid_constant__ CUtensorMap tmap_c, const __grid_constant__ GemmParams p)
{
    using namespace large;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
    uint64_t* empty = full + STAGES;
    uint64_t* sf_ready = empty + STAGES;
    uint64_t* acc_full = sf_ready + SF_SLOTS;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* ovl_free = acc_empty + 2;
    uint64_t* drain = ovl_free + 1;
    uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + OFF_TMEM_PTR);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int num_tiles = p.m_tiles * p.n_tiles;

    if (warp == 0 && lane == 0) {
        prefetch_tensor_map(&tmap_a);
        prefetch_tensor_map(&tmap_w);
        prefetch_tensor_map(&tmap_c);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < SF_SLOTS; ++i) {
            mbar_init(&sf_ready[i], 4);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], 8);
        }
        // SWIGLU: every epilogue warp reads gate and up columns; all release after their drain
        mbar_init(ovl_free, SWIGLU ? 8 : Overlap<ACC1_COL>::warps());
        mbar_init(drain, 1);
        fence_mbarrier_init();
    }
    if (warp == 2) {
        tmem_alloc(tmem_ptr, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_ptr;

    if (QA && warp >= 2) {
        // ------------------------------------------------------------ fused quantisation
        const float s_g = *p.act_scale;
        QuantParams qp = {};
        qp.q = p.qa_q;
        qp.sf = p.qa_sf;
        qp.k = p.k;
        QuantLaunch ql = {};
        ql.pairs = 2u * (uint32_t)p.katoms;
        // the first m-blocks, before the mainloop, by warps 2..15 of every CTA
        qa_quantize_range<qa::FIRST_ITEMS>(p, qp, ql, 0, p.qa_first, blockIdx.x * qa::FIRST_WARPS + (warp - 2),
                                           gridDim.x * qa::FIRST_WARPS, lane, s_g);
        named_barrier_sync(qa::BAR_FIRST, qa::FIRST_WARPS * 32);
        if (warp == 2)
            for (int mb = lane; mb < p.qa_first; mb += 32) qa_mark_ready(p, mb);
        // the rest, a band at a time in order, by warps 2 and 3 while the MMAs run
        if (warp < 4) {
            for (int mb0 = p.qa_first; mb0 < p.m_tiles; mb0 += qa::BAND) {
                const int mb1 = min(mb0 + qa::BAND, p.m_tiles);
                qa_quantize_range<qa::BG_ITEMS>(p, qp, ql, mb0, mb1, blockIdx.x * qa::BG_WARPS + (warp - 2),
                                                gridDim.x * qa::BG_WARPS, lane, s_g);
                named_barrier_sync(qa::BAR_BG, qa::BG_WARPS * 32);
                if (warp == 2 && mb0 + lane < mb1) qa_mark_ready(p, mb0 + lane);
            }
        }
    }

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        // (the whole warp walks the tiles, for the ready check of QA; lane 0
        // issues the copies)
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        int ready_below = 0;
        for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
            const int t = tile + p.tile_shift - (tile + p.tile_shift >= num_tiles ? num_tiles : 0);
            int mb, nb;
            tile_mn<QA>(t, p, mb, nb);
            if (QA && mb >= ready_below) ok = qa_wait_ready(p, ready_below, mb, lane);
            if (lane == 0 && ok) {
                for (int kt = 0; kt < p.k_tiles; ++kt) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, kStatusTimeoutEmpty)) {
                        ok = false;
                        break;
                    }
                    const int nks = min(KSTEPS, p.katoms - kt * KSTEPS);
                    const uint32_t sf_bytes = (uint32_t)nks * 512u;
                    // weight row blocks of the tile's two 128-row halves
                    const int rb0 = SWIGLU ? nb : 2 * nb;
                    const int rb1 = SWIGLU ? p.swiglu_f / 128 + nb : 2 * nb + 1;
                    const bool w_rb1 = rb1 < p.w_rowblocks;
                    const uint32_t bytes = A_STAGE + B_STAGE + sf_bytes * (w_rb1 ? 3u : 2u);
                    mbar_arrive_expect_tx(&full[stage], bytes);
                    tma_load_2d(smem + OFF_A + stage * A_STAGE, &tmap_a, &full[stage], kt * BK_BYTES, mb * BM);
                    if (SWIGLU) {
                        tma_load_2d(smem + OFF_B + stage * B_STAGE, &tmap_w, &full[stage], kt * BK_BYTES, rb0 * 128);
                        tma_load_2d(smem + OFF_B + stage * B_STAGE + 128 * BK_BYTES, &tmap_w, &full[stage],
                                    kt * BK_BYTES, rb1 * 128);
                    } else {
                        tma_load_2d(smem + OFF_B + stage * B_STAGE, &tmap_w, &full[stage], kt * BK_BYTES, nb * BN);
                    }
                    bulk_load(smem + OFF_SFA + stage * SFA_STAGE,
                              p.a_sf + ((int64_t)mb * p.katoms + kt * KSTEPS) * 512, sf_bytes, &full[stage]);
                    bulk_load(smem + OFF_SFB + stage * SFB_STAGE,
                              p.w_sf + ((int64_t)rb0 * p.katoms + kt * KSTEPS) * 512, sf_bytes, &full[stage]);
                    if (w_rb1)
                        bulk_load(smem + OFF_SFB + stage * SFB_STAGE + 2048,
                                  p.w_sf + ((int64_t)rb1 * p.katoms + kt * KSTEPS) * 512, sf_bytes, &full[stage]);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
        }
        if (lane == 0 && !ok) {
            // Give the copies already issued a bounded time to land before the
            // CTA can leave (they need nothing else to complete).
            const long long t0 = clock64();
            while (clock64() - t0 < kWaitCycles / 64) {
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_nvf4(BM, BN);
            const uint64_t adesc0 = desc_kmajor_sw128(smem + OFF_A);
            const uint64_t bdesc0 = desc_kmajor_sw128(smem + OFF_B);
            int stage = 0, slot = 0;
            uint32_t slot_phase = 0;
            bool ok = true;
            int i = 0;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++i) {
                const int b = i & 1;
                // This accumulator's previous tile (i - 2) is fully drained, and
                // the columns it shares with the other one are free (tile i - 1).
                if (!mbar_wait(&acc_empty[b], ((i >> 1) & 1) ^ 1, kStatusTimeoutAccum) ||
                    (i > 0 && !mbar_wait(ovl_free, (i - 1) & 1, kStatusTimeoutAccum))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t acc = tmem_base + (b ? ACC1_COL : 0);
                for (int kt = 0; kt < p.k_tiles; ++kt) {
                    if (!mbar_wait(&sf_ready[slot], slot_phase, kStatusTimeoutFull)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sf_col = tmem_base + SF_COL + slot * SF_SLOT;
                    // stage buffers are 1 KB aligned: advance the descriptors' address fields
                    const uint64_t adesc = adesc0 + (uint64_t)(stage * (A_STAGE >> 4));
                    const uint64_t bdesc = bdesc0 + (uint64_t)(stage * (B_STAGE >> 4));
                    // 64 FP4 values = 32 bytes along K: +2 in the descriptor's 16-byte units.
                    if (kt + 1 < p.k_tiles || p.katoms % KSTEPS == 0) {
#pragma unroll
                        for (int ks = 0; ks < KSTEPS; ++ks)
                            mma_nvf4(acc, adesc + 2 * ks, bdesc + 2 * ks, idesc, (kt | ks) != 0, sf_col + 4 * ks,
                                     sf_col + 16 + 8 * ks);
                    } else {
                        const int nks = p.katoms - kt * KSTEPS;
                        for (int ks = 0; ks < nks; ++ks)
                            mma_nvf4(acc, adesc + 2 * ks, bdesc + 2 * ks, idesc, (kt | ks) != 0, sf_col + 4 * ks,
                                     sf_col + 16 + 8 * ks);
                    }
                    // one commit frees the stage for the producer and, for the
                    // scale warps, the scale slot these MMAs read
                    mma_commit(&empty[stage]);
                    if (++stage == STAGES) stage = 0;
                    if (++slot == SF_SLOTS) {
                        slot = 0;
                        slot_phase ^= 1;
                    }
                }
                mma_commit(&acc_full[b]);
            }
            if (!ok) {
                // After an abort, wait (bounded) until every MMA issued so far has
                // finished before the CTA can free TMEM and leave.
                mma_commit(drain);
                mbar_wait(drain, 0, kStatusTimeoutDrain, kWaitCycles / 8);
            }
        }
        __syncwarp();
    } else if (warp >= 12) {
        // ------------------------------------------------------------ scale staging
        // Quadrant q writes lanes 32q..32q+31; each lane l receives row l of every
        // atom (16 bytes = the scales of rows l, l+32, l+64, l+96), which is the
        // layout block-scaled MMAs read for both operands.
        // The slot of stage k was last read by the MMAs of stage k - SF_SLOTS;
        // their completion is the commit on that stage's empty barrier (which
        // cannot run a phase ahead: stage k + SF_SLOTS needs this slot first).
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        int stage = 0, slot = 0;
        uint32_t phase = 0;
        long long kglob = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
            for (int kt = 0; kt < p.k_tiles; ++kt, ++kglob) {
                const long long kprev = kglob - SF_SLOTS;
                if (!mbar_wait(&full[stage], phase, kStatusTimeoutFull) ||
                    (kprev >= 0 && !mbar_wait(&empty[kprev % STAGES], (uint32_t)((kprev / STAGES) & 1),
                                              kStatusTimeoutFull))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint8_t* sfa = smem + OFF_SFA + stage * SFA_STAGE + lane * 16;
                const uint8_t* sfb = smem + OFF_SFB + stage * SFB_STAGE + lane * 16;
                uint32_t ra[16], rb[16], rc[16];
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint4 a = *reinterpret_cast<const uint4*>(sfa + ks * 512);
                    ra[4 * ks] = a.x;
                    ra[4 * ks + 1] = a.y;
                    ra[4 * ks + 2] = a.z;
                    ra[4 * ks + 3] = a.w;
                    const uint4 b0 = *reinterpret_cast<const uint4*>(sfb + ks * 512);
                    const uint4 b1 = *reinterpret_cast<const uint4*>(sfb + 2048 + ks * 512);
                    uint32_t* d = ks < 2 ? rb : rc;
                    const int o = (ks & 1) * 8;
                    d[o] = b0.x;
                    d[o + 1] = b0.y;
                    d[o + 2] = b0.z;
                    d[o + 3] = b0.w;
                    d[o + 4] = b1.x;
                    d[o + 5] = b1.y;
                    d[o + 6] = b1.z;
                    d[o + 7] = b1.w;
                }
                const uint32_t col = tmem_base + lane_base + SF_COL + slot * SF_SLOT;
                tmem_st_32x32b_x16(col, ra);        // A: k-step ks at columns 4ks .. 4ks+3
                tmem_st_32x32b_x16(col + 16, rb);   // B: k-step ks at columns 16+8ks .. 16+8ks+7
                tmem_st_32x32b_x16(col + 32, rc);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sf_ready[slot]);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
                if (++slot == SF_SLOTS) slot = 0;
            }
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ epilogue
        const int ew = warp - 4;
        const int quad = warp & 3;  // TMEM lanes this warp may access
        const int half = ew >> 2;   // which 128 accumulator columns
        const float s_ga = *p.act_scale;
        int i = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++i) {
            const int b = i & 1;
            const int t = tile + p.tile_shift - (tile + p.tile_shift >= num_tiles ? num_tiles : 0);
            int mb, nb;
            tile_mn<QA>(t, p, mb, nb);
            if (!mbar_wait(&acc_full[b], (i >> 1) & 1, kStatusTimeoutAccum)) break;
            tc_fence_after();
            const int row = mb * BM + quad * 32 + lane;
            const int ncol0 = nb * BN + half * 128;
            const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + (b ? ACC1_COL : 0) + half * 128;
            // The columns shared with the other accumulator are drained first
            // and released (Overlap<ACC1_COL>).
            using OV = Overlap<ACC1_COL>;
            const int ov_rot = OV::rot(b, half), ov_count = OV::count(b, half);
            if (SWIGLU) {
                // warp (quad, half): gate chunks 2 half, 2 half + 1 with the up
                // chunks 4 columns-of-32 to the right; 64 h columns per row.
                // Each chunk is first turned into the BF16 values the unfused
                // GEMM would store (g, u); the chunks the other accumulator
                // shares are loaded first and released before the rest (chunk
                // c of ACC0 is shared when c >= 5, of ACC1 when c <= 2), so the
                // next tile's MMAs do not wait for the SiLU arithmetic.
                const uint32_t tacc = tmem_base + ((uint32_t)(quad * 32) << 16) + (b ? ACC1_COL : 0);
                const float s_h = *p.h_scale;
                const int hcol0 = nb * 128 + half * 64;             // first h column of this warp
                uint32_t gpk[2][16], upk[2][16];                    // BF16 pairs of g and u
                auto rel = [&] { mbar_arrive(ovl_free); };
                auto done = [&] { mbar_arrive(&acc_empty[b]); };
                if (b == 0) {
                    if (half == 0) swiglu_load<0, 0>(tacc, hcol0, s_ga, p, lane, rel, done, gpk, upk);
                    else swiglu_load<0, 1>(tacc, hcol0, s_ga, p, lane, rel, done, gpk, upk);
                } else {
                    if (half == 0) swiglu_load<1, 0>(tacc, hcol0, s_ga, p, lane, rel, done, gpk, upk);
                    else swiglu_load<1, 1>(tacc, hcol0, s_ga, p, lane, rel, done, gpk, upk);
                }
                uint32_t sfw = 0;
                const bool live = row < p.m;
#pragma unroll
                for (int g2 = 0; g2 < 2; ++g2) {
                    const int gcol = hcol0 + 32 * g2;                // gate column in the fused weight
                    const uint32_t(&gp)[16] = gpk[g2];
                    const uint32_t(&up)[16] = upk[g2];
                    float h0[16], h1[16];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float g0l = __uint_as_float(gp[e] << 16), g0h = __uint_as_float(gp[e] & 0xFFFF0000u);
                        const float u0l = __uint_as_float(up[e] << 16), u0h = __uint_as_float(up[e] & 0xFFFF0000u);
                        const float g1l = __uint_as_float(gp[8 + e] << 16), g1h = __uint_as_float(gp[8 + e] & 0xFFFF0000u);
                        const float u1l = __uint_as_float(up[8 + e] << 16), u1h = __uint_as_float(up[8 + e] & 0xFFFF0000u);
                        h0[2 * e] = silu_mul_bf16(g0l, u0l);
                        h0[2 * e + 1] = silu_mul_bf16(g0h, u0h);
                        h1[2 * e] = silu_mul_bf16(g1l, u1l);
                        h1[2 * e + 1] = silu_mul_bf16(g1h, u1h);
                    }
                    uint32_t sb0, sb1;
                    uint2 q0, q1;
                    quantize_block16(h0, s_h, live, sb0, q0);
                    quantize_block16(h1, s_h, live, sb1, q1);
                    if (live)
                        *reinterpret_cast<uint4*>(p.h_q + (int64_t)row * (p.swiglu_f >> 1) + (gcol >> 1)) =
                            make_uint4(q0.x, q0.y, q1.x, q1.y);
                    sfw |= (sb0 | (sb1 << 8)) << (16 * g2);
                }
                // four consecutive 16-column blocks of h: one word of the row's atom
                // (zero on the padding rows, which the tiled layout requires)
                *reinterpret_cast<uint32_t*>(p.h_sf + sf_tiled_offset(row, hcol0 >> 4, p.swiglu_f >> 6)) = sfw;
            } else if (!p.out_fp32) {
                uint32_t packed[4][16];
                drain_bf16_plan<ACC1_COL>(b, half, taddr, ncol0, s_ga, p, [&] { mbar_arrive(ovl_free); }, lane,
                                          packed);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[b]);
                // Store through this warp's 1 KB buffer: 16 rows x 32 BF16 columns
                // (64-byte rows in the 64-byte swizzle the C tensor map uses); the
                // copy engine clips rows and columns past the matrix.
                uint8_t* cbuf = smem + OFF_C + ew * C_WARP;
                const int row0 = mb * BM + quad * 32;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
#pragma unroll
                    for (int hr = 0; hr < 2; ++hr) {
                        if (lane == 0) bulk_wait_group_read<0>();
                        __syncwarp();
                        if ((lane >> 4) == hr) {
                            const int r = lane & 15;
#pragma unroll
                            for (int u = 0; u < 4; ++u)
                                *reinterpret_cast<uint4*>(cbuf + r * 64 + ((u ^ ((r >> 1) & 3)) << 4)) =
                                    make_uint4(packed[j][4 * u], packed[j][4 * u + 1], packed[j][4 * u + 2],
                                               packed[j][4 * u + 3]);
                        }
                        fence_proxy_async_shared();
                        __syncwarp();
                        if (lane == 0 && row0 + 16 * hr < p.m && ncol0 + j * 32 < p.n) {
                            tma_store_2d(&tmap_c, cbuf, ncol0 + j * 32, row0 + 16 * hr);
                            bulk_commit_group();
                        }
                    }
                }
                {
                    // gates: a warp pass over its own columns, or shared by the
                    // quadrant's two warps when only one half holds gate columns
                    const int nb0 = nb * BN;
                    const bool g0 = gdn_touches(p, nb0, 128), g1 = gdn_touches(p, nb0 + 128, 128);
                    if (g0 != g1)
                        gdn_pass_shared(p, smem + OFF_C, C_WARP, packed, row0, nb0, quad, half, g1 ? 1 : 0, lane);
                    else if (g0)
                        gdn_pass(p, cbuf, packed, row0, ncol0, lane);
                }
            } else {
                for (int jj = 0; jj < 4; ++jj) {
                    const int j = (ov_rot + jj) & 3;
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(taddr + j * 32, v);
                    tmem_ld_wait();
                    if (jj + 1 == ov_count) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(ovl_free);
                    }
                    if (jj == 3) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&acc_empty[b]);
                    }
                    const int col0 = ncol0 + j * 32;
                    if (row < p.m && col0 < p.n) {
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            const int col = col0 + 8 * g;
                            if (col < p.n) {
                                const float alpha = __fmul_rn(s_ga, segment_scale(p.segs, col));
                                float o[8];
#pragma unroll
                                for (int e = 0; e < 8; ++e) o[e] = __fmul_rn(__uint_as_float(v[8 * g + e]), alpha);
                                store8(p.c, p.ldc, 1, row, col, o);
                            }
                        }
                    }
                }
            }
        }
    }

    if (warp >= 4 && warp < 12) {
        if (lane == 0) bulk_wait_group<0>();
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// ===========================================================================
// Large-M kernel on CTA pairs (cta_group::2): a cluster of two CTAs on two SMs
// computes a 256 x 256 tile with M = 256 MMAs issued by the even CTA.  Each CTA
// stages its own 128 rows of A and its own 128 of the tile's 256 B rows, so per
// FLOP an SM pulls 2/3 of the operand bytes of the single-CTA kernel through
// L2 -> shared memory (the bound of that kernel).  The rest follows
// gemm_large_kernel: scale staging with tcgen05.st in each CTA (its own A
// scales and the full 256 rows of B scales, which its half of the MMA reads
// from its own TMEM), overlapped accumulators, TMA-store epilogue on each
// CTA's own 128 rows.  Each CTA's loads complete on its own barrier; the even
// CTA learns that both halves of a stage are ready from the scale warps of
// both CTAs (8 arrivals on its sf_ready), and its commits reach both CTAs.
// ===========================================================================
namespace pairk {
constexpr int CTA_ROWS = 128, BN = 256, BK_BYTES = 128;
constexpr int STAGES = 5;
constexpr int KSTEPS = 4;
constexpr int A_STAGE = CTA_ROWS * BK_BYTES;        // 16 KB: this CTA's 128 of the 256 A rows
constexpr int B_STAGE = (BN / 2) * BK_BYTES;        // 16 KB: this CTA's 128 of the 256 B rows
constexpr int SFA_STAGE = 4 * 512;                  // 4 atoms of this CTA's 128 A rows
constexpr int SFB_STAGE = 2 * 4 * 512;              // all 256 B rows: 2 row blocks x 4 atoms
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + STAGES * A_STAGE;
constexpr int OFF_SFA = OFF_B + STAGES * B_STAGE;
constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_STAGE;
constexpr int OFF_C = OFF_SFB + STAGES * SFB_STAGE;
constexpr int C_WARP = 2048;                        // per epilogue warp: one 32 x 32 BF16 chunk
constexpr int OFF_BAR = OFF_C + 8 * C_WARP;
constexpr int SF_SLOTS = 2;
// full[S], empty[S], sf_ready[SLOTS], acc_full[2], acc_empty[2], ovl_free, drain
constexpr int NUM_BARS = 2 * STAGES + SF_SLOTS + 2 + 2 + 1 + 1;
constexpr int OFF_TMEM_PTR = OFF_BAR + NUM_BARS * 8;
constexpr int SMEM_BYTES = OFF_TMEM_PTR + 16 + 1024;
constexpr int THREADS = 512;
constexpr int TMEM_COLS = 512;
constexpr int ACC1_COL = 160;
constexpr int SF_COL = 416;
constexpr int SF_SLOT = 48;
static_assert(ACC1_COL + BN <= SF_COL && SF_COL + SF_SLOTS * SF_SLOT <= TMEM_COLS, "TMEM budget");
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
}  // namespace pairk

__global__ void __launch_bounds__(pairk::THREADS, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_w,
                     const __grid_constant__ CUtensorMap tmap_c, const __grid_constant__ GemmParams p)
{
    using namespace pairk;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
    uint64_t* empty = full + STAGES;
    uint64_t* sf_ready = empty + STAGES;
    uint64_t* acc_full = sf_ready + SF_SLOTS;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* ovl_free = acc_empty + 2;
    uint64_t* drain = ovl_free + 1;
    uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + OFF_TMEM_PTR);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();     // 0: issues the pair's MMAs
    const int pair = blockIdx.x >> 1;
    const int npairs = gridDim.x >> 1;
    const int num_tiles = p.m_tiles * p.n_tiles;  // m_tiles counts 256-row tiles here

    if (warp == 0 && lane == 0) {
        prefetch_tensor_map(&tmap_a);
        prefetch_tensor_map(&tmap_w);
        prefetch_tensor_map(&tmap_c);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < SF_SLOTS; ++i) {
            mbar_init(&sf_ready[i], 8);     // 4 scale warps in each CTA
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], 16);   // 8 epilogue warps in each CTA
        }
        mbar_init(ovl_free, 2 * Overlap<ACC1_COL>::warps());
        mbar_init(drain, 1);
        fence_mbarrier_init();
    }
    if (warp == 2) {
        tmem_alloc_pair(tmem_ptr, TMEM_COLS);
        tmem_relinquish_pair();
    }
    // Both CTAs' barriers exist before either CTA may signal the other's.
    tc_fence_before();
    cluster_arrive_release();
    cluster_wait_acquire();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_ptr;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = pair; tile < num_tiles && ok; tile += npairs) {
                const int mb = tile % p.m_tiles, nb = tile / p.m_tiles;
                const int a_rb = 2 * mb + (int)rank;              // this CTA's 128-row block of A
                const bool a_live = a_rb < p.a_rowblocks;
                for (int kt = 0; kt < p.k_tiles; ++kt) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, kStatusTimeoutEmpty)) {
                        ok = false;
                        break;
                    }
                    const int nks = min(KSTEPS, p.katoms - kt * KSTEPS);
                    const uint32_t sf_bytes = (uint32_t)nks * 512u;
                    const bool w_rb1 = 2 * nb + 1 < p.w_rowblocks;
                    const uint32_t bytes =
                        A_STAGE + B_STAGE + sf_bytes * ((a_live ? 1u : 0u) + 1u + (w_rb1 ? 1u : 0u));
                    mbar_arrive_expect_tx(&full[stage], bytes);
                    tma_load_2d(smem + OFF_A + stage * A_STAGE, &tmap_a, &full[stage], kt * BK_BYTES,
                                a_rb * CTA_ROWS);
                    tma_load_2d(smem + OFF_B + stage * B_STAGE, &tmap_w, &full[stage], kt * BK_BYTES,
                                nb * BN + (int)rank * (BN / 2));
                    if (a_live)
                        bulk_load(smem + OFF_SFA + stage * SFA_STAGE,
                                  p.a_sf + ((int64_t)a_rb * p.katoms + kt * KSTEPS) * 512, sf_bytes, &full[stage]);
                    bulk_load(smem + OFF_SFB + stage * SFB_STAGE,
                              p.w_sf + ((int64_t)(2 * nb) * p.katoms + kt * KSTEPS) * 512, sf_bytes, &full[stage]);
                    if (w_rb1)
                        bulk_load(smem + OFF_SFB + stage * SFB_STAGE + 2048,
                                  p.w_sf + ((int64_t)(2 * nb + 1) * p.katoms + kt * KSTEPS) * 512, sf_bytes,
                                  &full[stage]);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            if (!ok) {
                const long long t0 = clock64();
                while (clock64() - t0 < kWaitCycles / 64) {
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (even CTA)
        if (lane == 0 && rank == 0) {
            const uint32_t idesc = idesc_nvf4(2 * CTA_ROWS, BN);
            const uint64_t adesc0 = desc_kmajor_sw128(smem + OFF_A);
            const uint64_t bdesc0 = desc_kmajor_sw128(smem + OFF_B);
            int stage = 0, slot = 0;
            uint32_t slot_phase = 0;
            bool ok = true;
            int i = 0;
            for (int tile = pair; tile < num_tiles && ok; tile += npairs, ++i) {
                const int b = i & 1;
                if (!mbar_wait(&acc_empty[b], ((i >> 1) & 1) ^ 1, kStatusTimeoutAccum) ||
                    (i > 0 && !mbar_wait(ovl_free, (i - 1) & 1, kStatusTimeoutAccum))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t acc = tmem_base + (b ? ACC1_COL : 0);
                for (int kt = 0; kt < p.k_tiles; ++kt) {
                    // both CTAs' stage has landed and its scales are in both TMEMs
                    if (!mbar_wait(&sf_ready[slot], slot_phase, kStatusTimeoutFull)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sf_col = tmem_base + SF_COL + slot * SF_SLOT;
                    const uint64_t adesc = adesc0 + (uint64_t)(stage * (A_STAGE >> 4));
                    const uint64_t bdesc = bdesc0 + (uint64_t)(stage * (B_STAGE >> 4));
                    if (kt + 1 < p.k_tiles || p.katoms % KSTEPS == 0) {
#pragma unroll
                        for (int ks = 0; ks < KSTEPS; ++ks)
                            mma_nvf4_pair(acc, adesc + 2 * ks, bdesc + 2 * ks, idesc, (kt | ks) != 0,
                                          sf_col + 4 * ks, sf_col + 16 + 8 * ks);
                    } else {
                        const int nks = p.katoms - kt * KSTEPS;
                        for (int ks = 0; ks < nks; ++ks)
                            mma_nvf4_pair(acc, adesc + 2 * ks, bdesc + 2 * ks, idesc, (kt | ks) != 0,
                                          sf_col + 4 * ks, sf_col + 16 + 8 * ks);
                    }
                    // frees the stage in both CTAs and, for their scale warps, the slot
                    mma_commit_pair(&empty[stage], 0x3);
                    if (++stage == STAGES) stage = 0;
                    if (++slot == SF_SLOTS) {
                        slot = 0;
                        slot_phase ^= 1;
                    }
                }
                mma_commit_pair(&acc_full[b], 0x3);
            }
            if (!ok) {
                mma_commit_pair(drain, 0x1);
                mbar_wait(drain, 0, kStatusTimeoutDrain, kWaitCycles / 8);
            }
        }
        __syncwarp();
    } else if (warp >= 12) {
        // ------------------------------------------------------------ scale staging (both CTAs)
        // The slot of stage k was last read by the MMAs of stage k - SF_SLOTS,
        // whose completion the even CTA commits to this CTA's empty barrier.
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        int stage = 0, slot = 0;
        uint32_t phase = 0;
        long long kglob = 0;
        bool ok = true;
        for (int tile = pair; tile < num_tiles && ok; tile += npairs) {
            for (int kt = 0; kt < p.k_tiles; ++kt, ++kglob) {
                const long long kprev = kglob - SF_SLOTS;
                if (!mbar_wait(&full[stage], phase, kStatusTimeoutFull) ||
                    (kprev >= 0 && !mbar_wait(&empty[kprev % STAGES], (uint32_t)((kprev / STAGES) & 1),
                                              kStatusTimeoutFull))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint8_t* sfa = smem + OFF_SFA + stage * SFA_STAGE + lane * 16;
                const uint8_t* sfb = smem + OFF_SFB + stage * SFB_STAGE + lane * 16;
                uint32_t ra[16], rb[16], rc[16];
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint4 a = *reinterpret_cast<const uint4*>(sfa + ks * 512);
                    ra[4 * ks] = a.x;
                    ra[4 * ks + 1] = a.y;
                    ra[4 * ks + 2] = a.z;
                    ra[4 * ks + 3] = a.w;
                    const uint4 b0 = *reinterpret_cast<const uint4*>(sfb + ks * 512);
                    const uint4 b1 = *reinterpret_cast<const uint4*>(sfb + 2048 + ks * 512);
                    uint32_t* d = ks < 2 ? rb : rc;
                    const int o = (ks & 1) * 8;
                    d[o] = b0.x;
                    d[o + 1] = b0.y;
                    d[o + 2] = b0.z;
                    d[o + 3] = b0.w;
                    d[o + 4] = b1.x;
                    d[o + 5] = b1.y;
                    d[o + 6] = b1.z;
                    d[o + 7] = b1.w;
                }
                const uint32_t col = tmem_base + lane_base + SF_COL + slot * SF_SLOT;
                tmem_st_32x32b_x16(col, ra);
                tmem_st_32x32b_x16(col + 16, rb);
                tmem_st_32x32b_x16(col + 32, rc);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(map_shared_rank(smem_u32(&sf_ready[slot]), 0));
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
                if (++slot == SF_SLOTS) slot = 0;
            }
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int ew = warp - 4;
        const int quad = warp & 3;
        const int half = ew >> 2;
        const float s_ga = *p.act_scale;
        const uint32_t ovl0 = map_shared_rank(smem_u32(ovl_free), 0);
        int i = 0;
        for (int tile = pair; tile < num_tiles; tile += npairs, ++i) {
            const int b = i & 1;
            const int mb = tile % p.m_tiles, nb = tile / p.m_tiles;
            if (!mbar_wait(&acc_full[b], (i >> 1) & 1, kStatusTimeoutAccum)) break;
            tc_fence_after();
            const int row0 = mb * 2 * CTA_ROWS + (int)rank * CTA_ROWS + quad * 32;
            const int row = row0 + lane;
            const int ncol0 = nb * BN + half * 128;
            const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + (b ? ACC1_COL : 0) + half * 128;
            using OV = Overlap<ACC1_COL>;
            const int ov_rot = OV::rot(b, half), ov_count = OV::count(b, half);
            if (!p.out_fp32) {
                uint32_t packed[4][16];
                drain_bf16_plan<ACC1_COL>(b, half, taddr, ncol0, s_ga, p, [&] { mbar_arrive_remote(ovl0); }, lane,
                                          packed);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(map_shared_rank(smem_u32(&acc_empty[b]), 0));
                uint8_t* cbuf = smem + OFF_C + ew * C_WARP;
                // One 32 x 32 BF16 chunk per TMA store (this kernel has the shared
                // memory for a 2 KB buffer per warp; half as many stores as
                // 16-row chunks, which measured ~1.5 % faster).
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    if (lane == 0) bulk_wait_group_read<0>();
                    __syncwarp();
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        *reinterpret_cast<uint4*>(cbuf + lane * 64 + ((u ^ ((lane >> 1) & 3)) << 4)) =
                            make_uint4(packed[j][4 * u], packed[j][4 * u + 1], packed[j][4 * u + 2], packed[j][4 * u + 3]);
                    fence_proxy_async_shared();
                    __syncwarp();
                    if (lane == 0 && row0 < p.m && ncol0 + j * 32 < p.n) {
                        tma_store_2d(&tmap_c, cbuf, ncol0 + j * 32, row0);
                        bulk_commit_group();
                    }
                }
                if (gdn_touches(p, ncol0, 128)) gdn_pass(p, cbuf, packed, row0, ncol0, lane);
            } else {
                for (int jj = 0; jj < 4; ++jj) {
                    const int j = (ov_rot + jj) & 3;
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(taddr + j * 32, v);
                    tmem_ld_wait();
                    if (jj + 1 == ov_count) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive_remote(ovl0);
                    }
                    if (jj == 3) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive_remote(map_shared_rank(smem_u32(&acc_empty[b]), 0));
                    }
                    const int col0 = ncol0 + j * 32;
                    if (row < p.m && col0 < p.n) {
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            const int col = col0 + 8 * g;
                            if (col < p.n) {
                                const float alpha = __fmul_rn(s_ga, segment_scale(p.segs, col));
                                float o[8];
#pragma unroll
                                for (int e = 0; e < 8; ++e) o[e] = __fmul_rn(__uint_as_float(v[8 * g + e]), alpha);
                                store8(p.c, p.ldc, 1, row, col, o);
                            }
                        }
                    }
                }
            }
        }
    }

    if (warp >= 4 && warp < 12) {
        if (lane == 0) bulk_wait_group<0>();
        __syncwarp();
    }
    // Neither CTA leaves (or frees TMEM) while the other may still signal it.
    tc_fence_before();
    cluster_arrive_release();
    cluster_wait_acquire();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
}

}  // namespace nvfp4
