// Block-scaled FP4 GEMM on the 5th-generation tensor cores (tcgen05), with the
// per-module global-scale epilogue.
//
//   C[m, n] = cvt( acc[m, n] * (s_ga * s_gw[seg(n)]) )
//   acc[m, n] = sum_kb sa[m, kb] sw[n, kb] sum_{k in kb} e2m1(qa[m, k]) e2m1(qw[n, k])
//
// The pages ("Why Gated DeltaNet Survives 4-Bit Quantization": page summary
// "Background" item 1; abstract, last sentence; news article "Risks and
// caveats") fix the operands (NVFP4 on both sides, native 4-bit tensor-core
// GEMMs) and the requirement that per-module-calibrated weights served as one
// fused GEMM keep their own global scales.  Here the fix is a segment table:
// each output-column range carries its module's FP32 weight global scale and
// the epilogue multiplies each column by the activation scale times the scale
// of the segment the column belongs to.
//
// Two kernels:
//  * gemm_large_kernel: persistent (one CTA per SM), warp-specialised:
//    warp 0 issues TMA loads into a 4-stage shared-memory ring, warp 1 copies
//    the stage's scale factors into TMEM and issues tcgen05 block-scaled MMAs
//    (M=128, N=256, K=64 per instruction) into a TMEM accumulator, warp 2 owns
//    the TMEM allocation, warps 4..11 drain the accumulator and apply the
//    segment scales.
//  * gemm_decode_kernel: small M (<= 64 tokens).  Swap-AB (128 weight rows
//    fill the MMA's M, the tokens its N) and split-K over a thread-block
//    cluster; the partial accumulators are summed in a fixed rank order through
//    distributed shared memory, so the result is deterministic.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "ptx.cuh"

namespace nvfp4 {

constexpr int kMaxSegments = 16;

struct SegTable {
    int count;
    int end[kMaxSegments];      // exclusive column end of segment s; segment s begins at end[s-1] (0 for s = 0)
    float scale[kMaxSegments];  // FP32 weight global (decode) scale of segment s
};

struct GemmParams {
    int m, n, k;
    const uint8_t* a_sf;        // tiled scales of A (rows m)
    const uint8_t* w_sf;        // tiled scales of W (rows n)
    const float* act_scale;     // device: s_ga
    void* c;
    int64_t ldc;
    int out_fp32;
    SegTable segs;
    int m_tiles, n_tiles, k_tiles, katoms;
    int a_rowblocks, w_rowblocks;
    int splits;                 // decode kernel: K-splits (= cluster size)
};

__device__ __forceinline__ float segment_scale(const SegTable& t, int col)
{
    float s = t.scale[0];
#pragma unroll 1
    for (int i = 0; i < t.count; ++i) {
        s = t.scale[i];
        if (col < t.end[i]) break;
    }
    return s;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}

// Store 8 consecutive output columns of one row.
__device__ __forceinline__ void store8(void* c, int64_t ldc, int out_fp32, int row, int col, const float (&v)[8])
{
    if (out_fp32) {
        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(c) + (int64_t)row * ldc + col);
        dst[0] = make_float4(v[0], v[1], v[2], v[3]);
        dst[1] = make_float4(v[4], v[5], v[6], v[7]);
    } else {
        uint4 w;
        w.x = pack_bf16x2(v[0], v[1]);
        w.y = pack_bf16x2(v[2], v[3]);
        w.z = pack_bf16x2(v[4], v[5]);
        w.w = pack_bf16x2(v[6], v[7]);
        *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(c) + (int64_t)row * ldc + col) = w;
    }
}

// ===========================================================================
// Large-M kernel
// ===========================================================================
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
constexpr int OFF_BAR = OFF_SFB + STAGES * SFB_STAGE;
constexpr int NUM_BARS = 2 * STAGES + 3;
constexpr int OFF_TMEM_PTR = OFF_BAR + NUM_BARS * 8;
constexpr int SMEM_BYTES = OFF_TMEM_PTR + 16 + 1024;  // + alignment slack
constexpr int THREADS = 384;                          // 4 control warps + 8 epilogue warps
constexpr int TMEM_COLS = 512;
constexpr int TMEM_SF = 256;                          // scale ring after the 256 accumulator columns
constexpr int TMEM_SF_STAGE = 48;                     // 16 (A) + 32 (B) columns per stage
}  // namespace large

__global__ void __launch_bounds__(large::THREADS, 1)
    gemm_large_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_w,
                      const __grid_constant__ GemmParams p)
{
    using namespace large;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
    uint64_t* empty = full + STAGES;
    uint64_t* tmem_full = empty + STAGES;
    uint64_t* tmem_empty = tmem_full + 1;
    uint64_t* drain = tmem_empty + 1;
    uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + OFF_TMEM_PTR);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int num_tiles = p.m_tiles * p.n_tiles;

    if (warp == 0 && lane == 0) {
        prefetch_tensor_map(&tmap_a);
        prefetch_tensor_map(&tmap_w);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(tmem_full, 1);
        mbar_init(tmem_empty, 8);
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

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                const int mb = tile % p.m_tiles, nb = tile / p.m_tiles;
                for (int kt = 0; kt < p.k_tiles; ++kt) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, kStatusTimeoutEmpty)) {
                        ok = false;
                        break;
                    }
                    const int nks = min(KSTEPS, p.katoms - kt * KSTEPS);
                    const uint32_t sf_bytes = (uint32_t)nks * 512u;
                    const bool w_rb1 = 2 * nb + 1 < p.w_rowblocks;
                    const uint32_t bytes = A_STAGE + B_STAGE + sf_bytes * (w_rb1 ? 3u : 2u);
                    mbar_arrive_expect_tx(&full[stage], bytes);
                    tma_load_2d(smem + OFF_A + stage * A_STAGE, &tmap_a, &full[stage], kt * BK_BYTES, mb * BM);
                    tma_load_2d(smem + OFF_B + stage * B_STAGE, &tmap_w, &full[stage], kt * BK_BYTES, nb * BN);
                    bulk_load(smem + OFF_SFA + stage * SFA_STAGE,
                              p.a_sf + ((int64_t)mb * p.katoms + kt * KSTEPS) * 512, sf_bytes, &full[stage]);
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
                // Give the copies already issued a bounded time to land before the
                // CTA can leave (they need nothing else to complete).
                const long long t0 = clock64();
                while (clock64() - t0 < kWaitCycles / 64) {
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_nvf4(BM, BN);
            int stage = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                if (!mbar_wait(tmem_empty, acc_phase ^ 1, kStatusTimeoutAccum)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int kt = 0; kt < p.k_tiles; ++kt) {
                    if (!mbar_wait(&full[stage], phase, kStatusTimeoutFull)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int nks = min(KSTEPS, p.katoms - kt * KSTEPS);
                    const uint32_t sf_col = tmem_base + TMEM_SF + stage * TMEM_SF_STAGE;
                    const uint8_t* sfa = smem + OFF_SFA + stage * SFA_STAGE;
                    const uint8_t* sfb = smem + OFF_SFB + stage * SFB_STAGE;
                    for (int ks = 0; ks < nks; ++ks) {
                        tmem_cp_32x128b_x4(sf_col + 4 * ks, desc_sf_atom(sfa + ks * 512));
                        tmem_cp_32x128b_x4(sf_col + 16 + 8 * ks, desc_sf_atom(sfb + ks * 512));
                        tmem_cp_32x128b_x4(sf_col + 16 + 8 * ks + 4, desc_sf_atom(sfb + 2048 + ks * 512));
                    }
                    const uint64_t adesc = desc_kmajor_sw128(smem + OFF_A + stage * A_STAGE);
                    const uint64_t bdesc = desc_kmajor_sw128(smem + OFF_B + stage * B_STAGE);
                    for (int ks = 0; ks < nks; ++ks) {
                        // 64 FP4 values = 32 bytes along K: +2 in the descriptor's 16-byte units.
                        mma_nvf4(tmem_base, adesc + 2 * ks, bdesc + 2 * ks, idesc, (kt | ks) != 0,
                                 sf_col + 4 * ks, sf_col + 16 + 8 * ks);
                    }
                    mma_commit(&empty[stage]);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                mma_commit(tmem_full);
                acc_phase ^= 1;
            }
            if (!ok) {
                // After an abort, wait (bounded) until every MMA issued so far has
                // finished before the CTA can free TMEM and leave.
                mma_commit(drain);
                mbar_wait(drain, 0, kStatusTimeoutDrain, kWaitCycles / 8);
            }
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ------------------------------------------------------------ epilogue
        const int ew = warp - 4;
        const int quad = warp & 3;  // TMEM lanes this warp may access
        const int half = ew >> 2;   // which 128 accumulator columns
        uint32_t acc_phase = 0;
        const float s_ga = *p.act_scale;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
            const int mb = tile % p.m_tiles, nb = tile / p.m_tiles;
            if (!mbar_wait(tmem_full, acc_phase, kStatusTimeoutAccum)) break;
            tc_fence_after();
            const int row = mb * BM + quad * 32 + lane;
            for (int j = 0; j < 4; ++j) {
                const int lcol = half * 128 + j * 32;
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(quad * 32) << 16) + lcol, v);
                tmem_ld_wait();
                if (j == 3) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(tmem_empty);
                }
                const int col0 = nb * BN + lcol;
                if (row < p.m && col0 < p.n) {
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const int col = col0 + 8 * g;
                        if (col < p.n) {
                            const float alpha = __fmul_rn(s_ga, segment_scale(p.segs, col));
                            float o[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) o[e] = __fmul_rn(__uint_as_float(v[8 * g + e]), alpha);
                            store8(p.c, p.ldc, p.out_fp32, row, col, o);
                        }
                    }
                }
            }
            acc_phase ^= 1;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// ===========================================================================
// Decode kernel: swap-AB, split-K over a cluster, DSMEM reduction.
// ===========================================================================
namespace decode {
constexpr int BW = 128;                      // weight rows per CTA (the MMA's M)
constexpr int BK_BYTES = 128;
constexpr int KSTEPS = 4;
constexpr int THREADS = 256;                 // 4 control warps + 4 epilogue warps
constexpr int W_STAGE = BW * BK_BYTES;       // 16 KB
constexpr int SF_STAGE = 4 * 512;            // 4 atoms (weights) / 4 atoms (tokens)
constexpr int TMEM_SF_STAGE = 32;            // 16 (weights) + 16 (tokens)

template <int BT>
struct Layout {
    static constexpr int STAGES = BT >= 64 ? 3 : 4;
    static constexpr int T_STAGE = BT * BK_BYTES;
    static constexpr int OFF_W = 0;
    static constexpr int OFF_T = OFF_W + STAGES * W_STAGE;
    static constexpr int OFF_SFW = OFF_T + STAGES * (T_STAGE < 1024 ? 1024 : T_STAGE);
    static constexpr int OFF_SFT = OFF_SFW + STAGES * SF_STAGE;
    static constexpr int OFF_BAR = OFF_SFT + STAGES * SF_STAGE;
    static constexpr int NUM_BARS = 2 * STAGES + 1;
    static constexpr int OFF_TMEM_PTR = OFF_BAR + NUM_BARS * 8;
    static constexpr int SMEM_BYTES = OFF_TMEM_PTR + 16 + 1024;
    static constexpr int RED_BYTES = BW * BT * 4;  // partial sums, reuses the operand ring
    static constexpr int TMEM_COLS = 256;
    static constexpr int TMEM_SF = BT;             // scale ring after the accumulator
    static_assert(RED_BYTES <= OFF_BAR, "reduction buffer must fit in the operand ring");
    static_assert(BT + STAGES * TMEM_SF_STAGE <= TMEM_COLS, "TMEM budget");
};
}  // namespace decode

template <int BT>
__global__ void __launch_bounds__(decode::THREADS, 2)
    gemm_decode_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_w,
                       const __grid_constant__ GemmParams p)
{
    using namespace decode;
    using L = Layout<BT>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
    uint64_t* empty = full + L::STAGES;
    uint64_t* tmem_full = empty + L::STAGES;
    uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + L::OFF_TMEM_PTR);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int wt = blockIdx.x;               // weight-row tile
    const int split = blockIdx.y;            // K split = rank in the cluster
    const int kt_per = (p.k_tiles + p.splits - 1) / p.splits;
    const int kt0 = min(split * kt_per, p.k_tiles);
    const int kt1 = min(kt0 + kt_per, p.k_tiles);

    if (warp == 0 && lane == 0) {
        prefetch_tensor_map(&tmap_a);
        prefetch_tensor_map(&tmap_w);
        for (int s = 0; s < L::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(tmem_full, 1);
        fence_mbarrier_init();
    }
    if (warp == 2) {
        tmem_alloc(tmem_ptr, L::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_ptr;

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            for (int kt = kt0; kt < kt1; ++kt) {
                if (!mbar_wait(&empty[stage], phase ^ 1, kStatusTimeoutEmpty)) break;
                const int nks = min(KSTEPS, p.katoms - kt * KSTEPS);
                const uint32_t sf_bytes = (uint32_t)nks * 512u;
                mbar_arrive_expect_tx(&full[stage], W_STAGE + L::T_STAGE + 2 * sf_bytes);
                tma_load_2d(smem + L::OFF_W + stage * W_STAGE, &tmap_w, &full[stage], kt * BK_BYTES, wt * BW);
                tma_load_2d(smem + L::OFF_T + stage * (L::T_STAGE < 1024 ? 1024 : L::T_STAGE), &tmap_a, &full[stage],
                            kt * BK_BYTES, 0);
                bulk_load(smem + L::OFF_SFW + stage * SF_STAGE, p.w_sf + ((int64_t)wt * p.katoms + kt * KSTEPS) * 512,
                          sf_bytes, &full[stage]);
                bulk_load(smem + L::OFF_SFT + stage * SF_STAGE, p.a_sf + ((int64_t)kt * KSTEPS) * 512, sf_bytes,
                          &full[stage]);
                ++issued;
                if (++stage == L::STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            (void)issued;
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_nvf4(BW, BT);
            int stage = 0;
            uint32_t phase = 0;
            for (int kt = kt0; kt < kt1; ++kt) {
                if (!mbar_wait(&full[stage], phase, kStatusTimeoutFull)) break;
                tc_fence_after();
                const int nks = min(KSTEPS, p.katoms - kt * KSTEPS);
                const uint32_t sf_col = tmem_base + L::TMEM_SF + stage * TMEM_SF_STAGE;
                const uint8_t* sfw = smem + L::OFF_SFW + stage * SF_STAGE;
                const uint8_t* sft = smem + L::OFF_SFT + stage * SF_STAGE;
                for (int ks = 0; ks < nks; ++ks) {
                    tmem_cp_32x128b_x4(sf_col + 4 * ks, desc_sf_atom(sfw + ks * 512));
                    tmem_cp_32x128b_x4(sf_col + 16 + 4 * ks, desc_sf_atom(sft + ks * 512));
                }
                const uint64_t wdesc = desc_kmajor_sw128(smem + L::OFF_W + stage * W_STAGE);
                const uint64_t tdesc =
                    desc_kmajor_sw128(smem + L::OFF_T + stage * (L::T_STAGE < 1024 ? 1024 : L::T_STAGE));
                for (int ks = 0; ks < nks; ++ks)
                    mma_nvf4(tmem_base, wdesc + 2 * ks, tdesc + 2 * ks, idesc, (kt != kt0) || (ks != 0),
                             sf_col + 4 * ks, sf_col + 16 + 4 * ks);
                mma_commit(&empty[stage]);
                if (++stage == L::STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            mma_commit(tmem_full);
        }
        __syncwarp();
    }

    // ---------------------------------------------------------------- partials
    // Epilogue warps 4..7: weight row = 32*(warp%4) + lane; BT token columns.
    float* red = reinterpret_cast<float*>(smem);  // [BT][BW], reuses the operand ring
    const bool have_k = kt1 > kt0;
    if (warp >= 4) {
        const int quad = warp & 3;
        const int wrow = quad * 32 + lane;
        bool ok = true;
        if (have_k) ok = mbar_wait(tmem_full, 0, kStatusTimeoutAccum);
        if (ok && have_k) tc_fence_after();
#pragma unroll
        for (int c = 0; c < BT; c += 16) {
            uint32_t v[16];
            if (have_k && ok) {
                tmem_ld_32x32b_x16(tmem_base + ((uint32_t)(quad * 32) << 16) + c, v);
                tmem_ld_wait();
            } else {
#pragma unroll
                for (int e = 0; e < 16; ++e) v[e] = 0u;
            }
            if (p.splits == 1) {
                const int n = wt * BW + wrow;
                if (n < p.n) {
                    const float alpha = __fmul_rn(*p.act_scale, segment_scale(p.segs, n));
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int t = c + e;
                        if (t < p.m) {
                            const float o = __fmul_rn(__uint_as_float(v[e]), alpha);
                            if (p.out_fp32)
                                static_cast<float*>(p.c)[(int64_t)t * p.ldc + n] = o;
                            else
                                static_cast<__nv_bfloat16*>(p.c)[(int64_t)t * p.ldc + n] = __float2bfloat16_rn(o);
                        }
                    }
                }
            } else {
#pragma unroll
                for (int e = 0; e < 16; ++e) red[(c + e) * BW + wrow] = __uint_as_float(v[e]);
            }
        }
    }

    if (p.splits > 1) {
        // All CTAs of the cluster hold their partials in shared memory now.
        cluster_arrive_release();
        cluster_wait_acquire();
        // Rank r sums its slice of the BT x BW partial tile over ranks 0..S-1 in
        // order, scales, converts and stores.
        const uint32_t red_addr = smem_u32(red);
        constexpr int kVec = BT * BW / 4;
        const int per = (kVec + p.splits - 1) / p.splits;
        const int v0 = split * per, v1 = min(v0 + per, kVec);
        const float s_ga = *p.act_scale;
        for (int i = v0 + (int)threadIdx.x; i < v1; i += THREADS) {
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int r = 0; r < p.splits; ++r) {
                const float4 x = ld_shared_cluster_f4(map_shared_rank(red_addr + 16u * (uint32_t)i, (uint32_t)r));
                acc.x = __fadd_rn(acc.x, x.x);
                acc.y = __fadd_rn(acc.y, x.y);
                acc.z = __fadd_rn(acc.z, x.z);
                acc.w = __fadd_rn(acc.w, x.w);
            }
            const int t = (4 * i) / BW;
            const int wrow = (4 * i) % BW;
            const int n = wt * BW + wrow;
            if (t < p.m && n < p.n) {
                // n % 4 == 0 and n < p.n with p.n % 16 == 0: the 4 columns stay inside one 16-column group.
                const float alpha = __fmul_rn(s_ga, segment_scale(p.segs, n));
                const float o0 = __fmul_rn(acc.x, alpha), o1 = __fmul_rn(acc.y, alpha);
                const float o2 = __fmul_rn(acc.z, alpha), o3 = __fmul_rn(acc.w, alpha);
                if (p.out_fp32) {
                    *reinterpret_cast<float4*>(static_cast<float*>(p.c) + (int64_t)t * p.ldc + n) =
                        make_float4(o0, o1, o2, o3);
                } else {
                    uint2 w;
                    w.x = pack_bf16x2(o0, o1);
                    w.y = pack_bf16x2(o2, o3);
                    *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.c) + (int64_t)t * p.ldc + n) = w;
                }
            }
        }
        // Nobody leaves while a peer may still read its shared memory.
        cluster_arrive_release();
        cluster_wait_acquire();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem_base, L::TMEM_COLS);
    }
}

// Deliberately waits on an mbarrier that nothing arrives at, with a short
// limit, to exercise the timeout path: records kStatusTimeoutSelftest and
// returns.  One thread, no memory traffic.
__global__ void selftest_wait_timeout_kernel(long long limit_cycles)
{
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbarrier_init();
        mbar_wait(&bar, 0, kStatusTimeoutSelftest, limit_cycles);
    }
}

}  // namespace nvfp4
