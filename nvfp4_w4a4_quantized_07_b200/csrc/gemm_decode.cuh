// Decode (small-M) block-scaled FP4 GEMM kernel and the bounded-wait self-test
// kernel; see gemm_common.cuh for the product computed.
#pragma once

#include "gemm_common.cuh"
#include "quant.cuh"

namespace nvfp4 {

// ===========================================================================
// Decode kernel (M <= 64): stream-K over 256-column output tiles.
//
// Small M is pure weight streaming, and on this hardware every TMA / bulk
// copy instruction and every block-scaled MMA has a fixed issue cost (~150
// cycles) whatever its size.  So the kernel keeps both large: the tokens are
// the MMA's M side (a 128-row operand of which only the first M rows are
// loaded and stored -- the rest is never read back), 256 weight rows its N
// side, 32 KB weight tiles per stage.  The (256-column tile, 256-deep k-tile)
// work units are split evenly over exactly one CTA per SM (a cooperative
// launch keeps them all resident).  A tile whose k-tiles span several CTAs is
// finished by the CTA holding its first k-tile: the others reach their part of
// it first, leave FP32 partials in the workspace and publish them with this
// call's epoch value; the owner adds them in CTA order, so the result does not
// depend on timing.
//
// Warp roles: 0 TMA producer, 1 MMA issuer, 2 TMEM allocation, 4..7
// epilogue (TMEM quadrants 0-3 = token rows 0..127), 8..11 scale staging.
// TMEM: accumulator [0, 256), four 48-column scale slots [256, 448).
// ===========================================================================
namespace decode {
constexpr int BN = 256;                      // output columns (weight rows) per tile = the MMA's N
constexpr int BK_BYTES = 128;
constexpr int KSTEPS = 4;
constexpr int THREADS = 384;
constexpr int B_STAGE = BN * BK_BYTES;       // 32 KB of weights
constexpr int SFA_STAGE = 4 * 512;           // token scale atoms (one 128-row block)
constexpr int SFB_STAGE = 2 * 4 * 512;       // weight scale atoms (two 128-row blocks)
constexpr int SF_SLOTS = 4;
constexpr int ACC_PITCH = BN + 4;            // floats per staged accumulator row: float4 access is conflict-free
constexpr int TMEM_COLS = 512;
constexpr int SF_COL = 256;
constexpr int SF_SLOT = 48;                  // 16 (tokens: 4 k-steps x 4) + 32 (weights: 4 x 8)
constexpr int MAX_CTAS = 256;
constexpr int FLAGS_BYTES = MAX_CTAS * 8;
static_assert(SF_COL + SF_SLOTS * SF_SLOT <= TMEM_COLS, "TMEM budget");

// Shared-memory plan for BT token rows.  The A stage holds only the BT loaded
// rows; the M = 128 MMA reads 16 KB from its start, running on into the next
// buffers, and the accumulator rows that come from those bytes are never read.
template <int BT>
struct Cfg {
    static constexpr int STAGES = BT >= 64 ? 3 : (BT >= 32 ? 4 : 5);
    static constexpr int A_STAGE = BT * BK_BYTES;
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + STAGES * A_STAGE;
    static constexpr int OFF_SFA = OFF_B + STAGES * B_STAGE;
    static constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_STAGE;
    static constexpr int OFF_ACC = OFF_SFB + STAGES * SFB_STAGE;
    static constexpr int OFF_BAR = OFF_ACC + BT * ACC_PITCH * 4;
    // full[S], empty[S], sf_ready[SLOTS], sf_free[SLOTS], acc_full, acc_empty, drain, sga_ready
    static constexpr int NUM_BARS = 2 * STAGES + 2 * SF_SLOTS + 4;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;     // TMEM base, verdicts, s_ga, amax partials
    static constexpr int SMEM_BYTES = OFF_MISC + 32 + 1024;
    static_assert(A_STAGE % 1024 == 0, "SW128 stages are 1 KB aligned");
    static_assert(OFF_A + (STAGES - 1) * A_STAGE + 128 * BK_BYTES <= OFF_MISC, "MMA A reads stay in the buffer");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// Which CTA's range holds unit u when `units` are split over `ctas`:
// CTA c owns [floor(c U / G), floor((c+1) U / G)).
__device__ __forceinline__ int cta_of_unit(int64_t u, int units, int ctas)
{
    return (int)(((u + 1) * ctas + units - 1) / units) - 1;
}
}  // namespace decode

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p)
{
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_u64(unsigned long long* p, unsigned long long v)
{
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Scale 4 consecutive output columns of one row by s_ga * s_gw[seg] and store
// them (4 columns never straddle a segment: boundaries are multiples of 16).
__device__ __forceinline__ void store4_scaled(const GemmParams& p, int row, int col, float s_ga, float4 v)
{
    const float alpha = __fmul_rn(s_ga, segment_scale(p.segs, col));
    const float o0 = __fmul_rn(v.x, alpha), o1 = __fmul_rn(v.y, alpha);
    const float o2 = __fmul_rn(v.z, alpha), o3 = __fmul_rn(v.w, alpha);
    if (p.out_fp32)
        *reinterpret_cast<float4*>(static_cast<float*>(p.c) + (int64_t)row * p.ldc + col) = make_float4(o0, o1, o2, o3);
    else {
        const uint2 w = make_uint2(pack_bf16x2(o0, o1), pack_bf16x2(o2, o3));
        *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.c) + (int64_t)row * p.ldc + col) = w;
        if (gdn_touches(p, col, 4))
            gdn_gate4(p, row, col, __bfloat162float(__float2bfloat16_rn(o0)), __bfloat162float(__float2bfloat16_rn(o1)),
                      __bfloat162float(__float2bfloat16_rn(o2)), __bfloat162float(__float2bfloat16_rn(o3)));
    }
}

// FQ: the activation quantisation is fused in.  Warps 2 and 3 then quantise
// the stage's BT x 256 slice of the raw activations straight into the A stage
// (the 128-byte-swizzled layout the TMA would have written) and the scale
// atoms into the scale stage, with the same block arithmetic as
// quantize_kernel, so the result is bit-identical to quantising first.
template <int BT, bool FQ>
__global__ void __launch_bounds__(decode::THREADS, 1)
    gemm_decode_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_w,
                       const __grid_constant__ GemmParams p)
{
    using namespace decode;
    using C = Cfg<BT>;
    constexpr int STAGES = C::STAGES;
    constexpr int A_STAGE = C::A_STAGE;
    constexpr int OFF_A = C::OFF_A, OFF_B = C::OFF_B, OFF_SFA = C::OFF_SFA, OFF_SFB = C::OFF_SFB;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* empty = full + STAGES;
    uint64_t* sf_ready = empty + STAGES;
    uint64_t* sf_free = sf_ready + SF_SLOTS;
    uint64_t* acc_full = sf_free + SF_SLOTS;
    uint64_t* acc_empty = acc_full + 1;
    uint64_t* drain = acc_empty + 1;
    uint64_t* sga_ready = drain + 1;   // FQ: the activation scale is in s_ga_smem
    uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* acc_ok = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);    // acc_full verdict
    volatile int* peers_bad = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8); // a peer wait ran out
    volatile float* s_ga_smem = reinterpret_cast<volatile float*>(smem + C::OFF_MISC + 12); // FQ: the scale used
    volatile float* amax_part = reinterpret_cast<volatile float*>(smem + C::OFF_MISC + 16); // FQ: [2]
    volatile int* sga_ok = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 24);         // FQ: sga_ready verdict
    float* acc_stage = reinterpret_cast<float*>(smem + C::OFF_ACC);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int cta = blockIdx.x;
    const int64_t u_begin = (int64_t)cta * p.units / p.ctas;
    const int64_t u_end = (int64_t)(cta + 1) * p.units / p.ctas;
    const int k_tiles = p.k_tiles;

    if (warp == 0 && lane == 0) {
        prefetch_tensor_map(&tmap_a);
        prefetch_tensor_map(&tmap_w);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], FQ ? 3 : 1);    // FQ: the producer and the two quantiser warps
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < SF_SLOTS; ++i) {
            mbar_init(&sf_ready[i], 4);
            mbar_init(&sf_free[i], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 4);
        mbar_init(drain, 1);
        mbar_init(sga_ready, 1);
        *peers_bad = 0;
        *acc_ok = 0;
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
            int nb = (int)(u_begin / k_tiles), kt = (int)(u_begin - (int64_t)nb * k_tiles);
            for (int64_t u = u_begin; u < u_end; ++u) {
                if (!mbar_wait(&empty[stage], phase ^ 1, kStatusTimeoutEmpty)) {
                    ok = false;
                    break;
                }
                const int nks = min(KSTEPS, p.katoms - kt * KSTEPS);
                const uint32_t sf_bytes = (uint32_t)nks * 512u;
                const bool rb1 = 2 * nb + 1 < p.w_rowblocks;
                if (FQ) {
                    mbar_arrive_expect_tx(&full[stage], B_STAGE + sf_bytes * (rb1 ? 2u : 1u));
                } else {
                    mbar_arrive_expect_tx(&full[stage], BT * BK_BYTES + B_STAGE + sf_bytes * (rb1 ? 3u : 2u));
                    tma_load_2d(smem + OFF_A + stage * A_STAGE, &tmap_a, &full[stage], kt * BK_BYTES, 0);
                    bulk_load(smem + OFF_SFA + stage * SFA_STAGE, p.a_sf + (int64_t)kt * KSTEPS * 512, sf_bytes,
                              &full[stage]);
                }
                tma_load_2d(smem + OFF_B + stage * B_STAGE, &tmap_w, &full[stage], kt * BK_BYTES, nb * BN);
                bulk_load(smem + OFF_SFB + stage * SFB_STAGE,
                          p.w_sf + ((int64_t)(2 * nb) * p.katoms + kt * KSTEPS) * 512, sf_bytes, &full[stage]);
                if (rb1)
                    bulk_load(smem + OFF_SFB + stage * SFB_STAGE + 2048,
                              p.w_sf + ((int64_t)(2 * nb + 1) * p.katoms + kt * KSTEPS) * 512, sf_bytes,
                              &full[stage]);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
                if (++kt == k_tiles) {
                    kt = 0;
                    ++nb;
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
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_nvf4(128, BN);
            int stage = 0, slot = 0;
            uint32_t slot_phase = 0, segs = 0;
            bool ok = true, first = true;
            int kt = (int)(u_begin % k_tiles);
            for (int64_t u = u_begin; u < u_end && ok; ++u) {
                if (u == u_begin || kt == 0) {
                    // a new segment: the accumulator has been drained
                    if (!mbar_wait(acc_empty, (segs & 1) ^ 1, kStatusTimeoutAccum)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    first = true;
                }
                if (!mbar_wait(&sf_ready[slot], slot_phase, kStatusTimeoutFull)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int nks = min(KSTEPS, p.katoms - kt * KSTEPS);
                const uint32_t sf_col = tmem_base + SF_COL + slot * SF_SLOT;
                const uint64_t adesc = desc_kmajor_sw128(smem + OFF_A + stage * A_STAGE);
                const uint64_t bdesc = desc_kmajor_sw128(smem + OFF_B + stage * B_STAGE);
                for (int ks = 0; ks < nks; ++ks)
                    mma_nvf4(tmem_base, adesc + 2 * ks, bdesc + 2 * ks, idesc, !(first && ks == 0), sf_col + 4 * ks,
                             sf_col + 16 + 8 * ks);
                first = false;
                mma_commit(&empty[stage]);
                mma_commit(&sf_free[slot]);
                if (++stage == STAGES) stage = 0;
                if (++slot == SF_SLOTS) {
                    slot = 0;
                    slot_phase ^= 1;
                }
                if (u == u_end - 1 || kt == k_tiles - 1) {
                    mma_commit(acc_full);
                    ++segs;
                }
                if (++kt == k_tiles) kt = 0;
            }
            if (!ok) {
                mma_commit(drain);
                mbar_wait(drain, 0, kStatusTimeoutDrain, kWaitCycles / 8);
            }
        }
        __syncwarp();
    } else if (FQ && (warp == 2 || warp == 3)) {
        // ------------------------------------------------------------ activation quantiser
        const int qt = threadIdx.x - 64;    // 0..63
        float s_ga;
        if (p.act_scale != nullptr) {
            s_ga = *p.act_scale;
        } else {
            // amax over the whole m x k activation (every CTA computes the same, exact value)
            const int vec = p.a_fp32 ? 4 : 8;
            const int64_t per_row = p.k / vec;
            const int64_t total = (int64_t)p.m * per_row;
            float mx = 0.0f;
            for (int64_t i = qt; i < total; i += 64) {
                const int64_t r = i / per_row;
                mx = fmaxf(mx, absmax_vec(p.a_in, r * p.lda + (i - r * per_row) * vec, p.a_fp32));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            if (lane == 0) amax_part[warp - 2] = mx;
            asm volatile("bar.sync 3, 64;" ::: "memory");
            s_ga = global_scale_from_amax(fmaxf(amax_part[0], amax_part[1]));
        }
        if (qt == 0) {
            *s_ga_smem = s_ga;
            mbar_arrive(sga_ready);
            if (cta == 0 && p.act_scale_out != nullptr) *p.act_scale_out = s_ga;
        }
        int stage = 0;
        uint32_t phase = 0;
        int kt = (int)(u_begin % k_tiles);
        const int64_t esz = p.a_fp32 ? 4 : 2;
        // Each thread owns BT / 8 chunks (row r, 32 columns) of a stage, taken two
        // at a time: all loads of a pair are issued before any arithmetic, and
        // the first pair's loads before the wait for the stage buffer (they do
        // not need it), so the L2 round trip overlaps the wait.
        constexpr int CPT = BT / 8;
        constexpr int CB = CPT < 2 ? CPT : 2;
        for (int64_t u = u_begin; u < u_end; ++u) {
            uint8_t* adst = smem + OFF_A + stage * A_STAGE;
            uint8_t* sdst = smem + OFF_SFA + stage * SFA_STAGE;
            bool waited = false, ok = true;
#pragma unroll
            for (int b0 = 0; b0 < CPT; b0 += CB) {
                uint4 raw[CB][8];
                bool l0[CB], l1[CB];
#pragma unroll
                for (int j = 0; j < CB; ++j) {
                    const int it = qt + 64 * (b0 + j);
                    const int r = it >> 3, c = it & 7;
                    const int64_t k0 = (int64_t)kt * 256 + c * 32;
                    l0[j] = r < p.m && k0 < p.k;
                    l1[j] = r < p.m && k0 + 16 < p.k;
                    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.a_in) +
                                                                      ((int64_t)r * p.lda + k0) * esz);
                    const int words = p.a_fp32 ? 8 : 4;   // 16-byte words per 32 elements
#pragma unroll
                    for (int w = 0; w < 8; ++w) {
                        const bool lv = (w < words / 2) ? l0[j] : l1[j];
                        raw[j][w] = (w < words && lv) ? __ldg(src + w) : make_uint4(0, 0, 0, 0);
                    }
                }
                if (!waited) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, kStatusTimeoutEmpty)) {
                        ok = false;
                        break;
                    }
                    waited = true;
                }
#pragma unroll
                for (int j = 0; j < CB; ++j) {
                    const int it = qt + 64 * (b0 + j);
                    const int r = it >> 3, c = it & 7;
                    float v0[16], v1[16];
                    if (p.a_fp32) {
#pragma unroll
                        for (int w = 0; w < 4; ++w) {
                            v0[4 * w] = __uint_as_float(raw[j][w].x);
                            v0[4 * w + 1] = __uint_as_float(raw[j][w].y);
                            v0[4 * w + 2] = __uint_as_float(raw[j][w].z);
                            v0[4 * w + 3] = __uint_as_float(raw[j][w].w);
                            v1[4 * w] = __uint_as_float(raw[j][4 + w].x);
                            v1[4 * w + 1] = __uint_as_float(raw[j][4 + w].y);
                            v1[4 * w + 2] = __uint_as_float(raw[j][4 + w].z);
                            v1[4 * w + 3] = __uint_as_float(raw[j][4 + w].w);
                        }
                    } else {
                        unpack_bf16x8(raw[j][0], v0);
                        unpack_bf16x8(raw[j][1], v0 + 8);
                        unpack_bf16x8(raw[j][2], v1);
                        unpack_bf16x8(raw[j][3], v1 + 8);
                    }
                    uint32_t sb0, sb1;
                    uint2 q0, q1;
                    quantize_block16(v0, s_ga, l0[j], sb0, q0);
                    quantize_block16(v1, s_ga, l1[j], sb1, q1);
                    // K-major 128-byte swizzle: 16-byte chunk c of row r sits at chunk c ^ (r % 8)
                    *reinterpret_cast<uint4*>(adst + (r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4)) =
                        make_uint4(q0.x, q0.y, q1.x, q1.y);
                    // scale atom of k-step c / 2: row r at (r % 32) * 16 + (r / 32 % 4) * 4, block (c % 2) * 2
                    *reinterpret_cast<uint16_t*>(sdst + (c >> 1) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 +
                                                 (c & 1) * 2) = (uint16_t)(sb0 | (sb1 << 8));
                }
            }
            if (!ok) break;
            fence_proxy_async_shared();     // the MMA reads the stage through the async proxy
            __syncwarp();
            if (lane == 0) mbar_arrive(&full[stage]);
            if (++stage == STAGES) {
                stage = 0;
                phase ^= 1;
            }
            if (++kt == k_tiles) kt = 0;
        }
    } else if (warp >= 8) {
        // ------------------------------------------------------------ scale staging
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        int stage = 0, slot = 0;
        uint32_t phase = 0, slot_phase = 0;
        for (int64_t u = u_begin; u < u_end; ++u) {
            if (!mbar_wait(&full[stage], phase, kStatusTimeoutFull) ||
                !mbar_wait(&sf_free[slot], slot_phase ^ 1, kStatusTimeoutFull))
                break;
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
            if (lane == 0) mbar_arrive(&sf_ready[slot]);
            if (++stage == STAGES) {
                stage = 0;
                phase ^= 1;
            }
            if (++slot == SF_SLOTS) {
                slot = 0;
                slot_phase ^= 1;
            }
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ epilogue
        // Per segment (one tile's k-range): the warps whose TMEM lanes hold
        // token rows move the FP32 accumulator into shared memory and release
        // TMEM at once, so the MMAs of the next segment start while this one is
        // stored.  Then all 128 epilogue threads work on the staged tile, 4
        // consecutive columns of one row each: a contributor (a range that
        // starts inside the tile) writes its partial to the workspace and
        // publishes it; the owner of a tile that lies wholly in this range
        // scales each column by s_ga * s_gw[seg] and stores the output.  An
        // owner whose range ends inside the tile waits for the peers' flags and
        // hands over to the all-warp finish below.  Every branch is uniform over
        // the four warps, so the named barrier (id 1, 128 threads) always matches.
        const int quad = warp & 3;
        const int et = threadIdx.x - 128;          // 0..127
        const int t = quad * 32 + lane;            // token row = accumulator lane
        const bool live = quad * 32 < BT;          // warp holds loaded token rows
        unsigned long long* flags = reinterpret_cast<unsigned long long*>(p.ws);
        float* parts = reinterpret_cast<float*>(p.ws + FLAGS_BYTES);
        float s_ga = FQ ? 0.0f : *p.act_scale;        // FQ: known once the first stage is in
        const int units4 = min(p.m, BT) * (BN / 4);  // float4 units of the live rows
        uint32_t segs = 0;
        int64_t u = u_begin;
        while (u < u_end) {
            const int nb = (int)(u / k_tiles), kb = (int)(u - (int64_t)nb * k_tiles);
            const int64_t seg_end = min(u_end, (int64_t)(nb + 1) * k_tiles);
            const bool owner = kb == 0;
            const bool complete = owner && seg_end == (int64_t)(nb + 1) * k_tiles;
            const int last = owner && !complete ? cta_of_unit((int64_t)(nb + 1) * k_tiles - 1, p.units, p.ctas) : cta;

            if (et == 0) *acc_ok = mbar_wait(acc_full, segs & 1, kStatusTimeoutAccum) ? 1 : 0;
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (!*acc_ok) break;
            if (FQ && segs == 0) {
                // bounded like every wait; the quantiser set it before its first stage
                if (et == 0) *sga_ok = mbar_wait(sga_ready, 0, kStatusTimeoutAccum) ? 1 : 0;
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (!*sga_ok) break;
                s_ga = *s_ga_smem;
            } else if (FQ) {
                s_ga = *s_ga_smem;
            }
            tc_fence_after();
            if (live) {
                const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16);
                float* row = acc_stage + t * ACC_PITCH;
#pragma unroll 1
                for (int j = 0; j < BN / 32; j += 2) {
                    uint32_t r0[32], r1[32];
                    __syncwarp();
                    tmem_ld_32x32b_x32(taddr + j * 32, r0);
                    tmem_ld_32x32b_x32(taddr + (j + 1) * 32, r1);
                    tmem_ld_wait();
                    if (t < BT) {
#pragma unroll
                        for (int e = 0; e < 32; e += 4) {
                            *reinterpret_cast<float4*>(row + j * 32 + e) =
                                make_float4(__uint_as_float(r0[e]), __uint_as_float(r0[e + 1]),
                                            __uint_as_float(r0[e + 2]), __uint_as_float(r0[e + 3]));
                            *reinterpret_cast<float4*>(row + (j + 1) * 32 + e) =
                                make_float4(__uint_as_float(r1[e]), __uint_as_float(r1[e + 1]),
                                            __uint_as_float(r1[e + 2]), __uint_as_float(r1[e + 3]));
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty);
            ++segs;

            if (owner && !complete) {
                // thread i waits for CTAs cta + 1 + i, cta + 1 + i + 128, ... to
                // publish their partials of tile nb
                for (int i = et; i < last - cta; i += 128) {
                    const long long t0 = clock64();
                    while (ld_acquire_u64(flags + cta + 1 + i) != p.epoch) {
                        if (clock64() - t0 > kWaitCycles) {
                            record_status(kStatusTimeoutCluster);
                            *peers_bad = 1;
                            break;
                        }
                    }
                }
            }
            // An owner whose range ends inside tile nb (always the CTA's last
            // segment) leaves the reduction to all twelve warps, below.
            if (owner && !complete) break;
            asm volatile("bar.sync 1, 128;" ::: "memory");   // staged tile complete
            if (*peers_bad) break;

            if (!owner) {
                float* mine = parts + (int64_t)cta * BT * BN;
                for (int x = et; x < units4; x += 128) {
                    const int r = x / (BN / 4), c4 = x % (BN / 4);
                    __stcg(reinterpret_cast<float4*>(mine + r * BN) + c4,
                           *reinterpret_cast<const float4*>(acc_stage + r * ACC_PITCH + 4 * c4));
                }
                __threadfence();
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (et == 0) st_release_u64(flags + cta, p.epoch);
            } else {
                // a complete tile: scale and store
                for (int x = et; x < units4; x += 128) {
                    const int r = x / (BN / 4);
                    const int col = nb * BN + 4 * (x % (BN / 4));
                    if (col < p.n)
                        store4_scaled(p, r, col, s_ga,
                                      *reinterpret_cast<const float4*>(acc_stage + r * ACC_PITCH + 4 * (x % (BN / 4))));
                }
            }
            u = seg_end;
        }
    }

    // ---------------------------------------------------------------- split-tile finish
    // The CTA whose range starts tile nb = (u_end - 1) / k_tiles but ends inside
    // it owns that tile's result: once the epilogue has staged this CTA's
    // accumulator and acquired the peers' flags, all 384 threads add the peers'
    // FP32 partials in CTA order (loads for FPG peers in flight together),
    // scale and store.  The condition is the same for every thread.
    {
        const int64_t fin_nb = u_end > u_begin ? (u_end - 1) / k_tiles : 0;
        const bool finish = u_end > u_begin && u_end % k_tiles != 0 && fin_nb * k_tiles >= u_begin;
        if (finish) {
            asm volatile("bar.sync 2, 384;" ::: "memory");
            if (*acc_ok && !*peers_bad) {
                constexpr int FDU = 3, FPG = 8;
                const int nb = (int)fin_nb;
                const int last = cta_of_unit((int64_t)(nb + 1) * k_tiles - 1, p.units, p.ctas);
                const int units4 = min(p.m, BT) * (BN / 4);
                const float* parts = reinterpret_cast<const float*>(p.ws + FLAGS_BYTES);
                const float s_ga = FQ ? *s_ga_smem : *p.act_scale;
                for (int x0 = threadIdx.x; x0 < units4; x0 += FDU * THREADS) {
                    float4 v[FDU];
#pragma unroll
                    for (int i = 0; i < FDU; ++i) {
                        const int x = x0 + i * THREADS;
                        if (x < units4)
                            v[i] = *reinterpret_cast<const float4*>(acc_stage + (x / (BN / 4)) * ACC_PITCH +
                                                                    4 * (x % (BN / 4)));
                    }
                    for (int c2 = cta + 1; c2 <= last; c2 += FPG) {
                        float4 q[FPG][FDU];
#pragma unroll
                        for (int g = 0; g < FPG; ++g) {
                            const float* src = parts + (int64_t)(c2 + g) * BT * BN;
#pragma unroll
                            for (int i = 0; i < FDU; ++i) {
                                const int x = x0 + i * THREADS;
                                if (x < units4 && c2 + g <= last)
                                    q[g][i] = __ldcg(reinterpret_cast<const float4*>(
                                        src + (x / (BN / 4)) * BN + 4 * (x % (BN / 4))));
                            }
                        }
#pragma unroll
                        for (int g = 0; g < FPG; ++g) {
                            if (c2 + g <= last) {
#pragma unroll
                                for (int i = 0; i < FDU; ++i) {
                                    v[i].x = __fadd_rn(v[i].x, q[g][i].x);
                                    v[i].y = __fadd_rn(v[i].y, q[g][i].y);
                                    v[i].z = __fadd_rn(v[i].z, q[g][i].z);
                                    v[i].w = __fadd_rn(v[i].w, q[g][i].w);
                                }
                            }
                        }
                    }
#pragma unroll
                    for (int i = 0; i < FDU; ++i) {
                        const int x = x0 + i * THREADS;
                        const int col = nb * BN + 4 * (x % (BN / 4));
                        if (x < units4 && col < p.n) store4_scaled(p, x / (BN / 4), col, s_ga, v[i]);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
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
