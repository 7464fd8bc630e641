// Decode (small-M) block-scaled FP4 GEMM kernel and the bounded-wait self-test
// kernel; see gemm_common.cuh for the product computed.
#pragma once

#include "gemm_common.cuh"
#include "quant.cuh"

namespace nvfp4 {

// ===========================================================================
// Decode kernel (M <= 64): stream-K over 128-column output tiles.
//
// Small M is pure weight streaming.  What a launch costs beyond the weight
// bytes is fixed: getting the CTAs onto the SMs, the first HBM round trip, and
// the hand-off of tiles whose K range is split between CTAs.  The kernel hides
// the first two under the previous kernel in the stream and keeps the third
// short:
//
//  * Programmatic dependent launch.  Every CTA lets the next kernel launch as
//    soon as its barriers exist.  Before it waits for the previous kernel to
//    complete it only touches weights (which no earlier kernel writes): it
//    fills its shared-memory ring with weight tiles.  Activations, the
//    activation scale, TMEM and every global write come after that wait.
//  * Few, large copies: a stage is two 256-deep k-tiles of one tile (32 KB of
//    weights), brought in by four copy instructions (weights, their scale
//    atoms, token rows, token scales; the two k-tiles of a 128-byte-wide
//    operand come as one 3-D box when K is a multiple of 256) -- the copy
//    engine's issue rate, not HBM, limits rings of many small copies.
//  * Stream-K: the (tile, k-tile) units are split evenly over one CTA per SM.
//    A tile whose k-tiles span several CTAs is finished by the CTA holding its
//    first k-tile (the "owner"), which reaches its part last (it ends its
//    range); the others reach their part first (it starts their range),
//    leave the FP32 partial in the workspace -- every value paired with a
//    32-bit tag fresh to this call in one 8-byte word, so no flag or fence is
//    needed -- and exit.  The owner loads the partials (waiting for their
//    tags) and adds them in CTA order, so the result does not depend on
//    timing.  Contributors leave early, which frees their SMs for the next
//    kernel's CTAs.
//
// The tokens are the MMA's M side: a 128-row operand of which only the first
// BT rows are loaded (the rest reads whatever follows in shared memory; those
// accumulator rows are never read back).  128 weight rows are its N side, so a
// split tile's partial is m x 128 and an owner adds few of them.  Two TMEM
// accumulators let the MMAs of the next segment run while the epilogue drains
// the last one.
//
// Warp roles: 0 TMA producer, 1 MMA issuer, 2 TMEM allocation (and, with the
// activation quantisation fused in, 2..3 quantise), 4..7 epilogue (TMEM lane
// quadrants 0..3 = token rows 0..127), 8..11 scale staging; an owner's twelve
// warps all take part in its finish.
// TMEM: accumulators [0, 128) and [128, 256), four 64-column scale slots
// [256, 512); allocated after the dependency wait.
// ===========================================================================
namespace decode {
constexpr int BN = 128;                      // output columns (weight rows) per tile = the MMA's N
constexpr int KT_BYTES = 128;                // one k-tile: 256 FP4 values = 128 bytes of a row
constexpr int KT_PER_STAGE = 2;
constexpr int KSTEPS = 4;                    // MMAs (K = 64) per k-tile
constexpr int THREADS = 384;
constexpr int W_KT = BN * KT_BYTES;          // 16 KB of weights per k-tile
constexpr int W_STAGE = KT_PER_STAGE * W_KT;
constexpr int SF_KT = KSTEPS * 512;          // scale atoms of one 128-row block per k-tile
constexpr int SF_STAGE = KT_PER_STAGE * SF_KT;
constexpr int SF_SLOTS = 4;
constexpr int SF_SLOT = 64;                  // per stage: A (8 k-steps x 4 columns), then B (8 x 4)
constexpr int ACC_PITCH = BN + 4;            // floats per staged accumulator row: float4 access is conflict-free
constexpr int TMEM_COLS = 512;
constexpr int SF_COL = 2 * BN;
constexpr int MAX_CTAS = 160;                // grid cap (one CTA per SM); sizes the workspace
static_assert(SF_COL + SF_SLOTS * SF_SLOT <= TMEM_COLS, "TMEM budget");

// Shared-memory plan for BT token rows.  The A stage holds only the BT loaded
// rows of each k-tile; the M = 128 MMA reads 16 KB from the start of a
// k-tile's rows, running on into the next buffers, and the accumulator rows
// that come from those bytes are never read.
template <int BT>
struct Cfg {
    static constexpr int STAGES = BT >= 64 ? 3 : 4;
    static constexpr int A_KT = BT * KT_BYTES;
    static constexpr int A_STAGE = KT_PER_STAGE * A_KT;
    static constexpr int OFF_A = 0;
    static constexpr int OFF_W = OFF_A + STAGES * A_STAGE;
    static constexpr int OFF_SFA = OFF_W + STAGES * W_STAGE;
    static constexpr int OFF_SFB = OFF_SFA + STAGES * SF_STAGE;
    static constexpr int OFF_ACC = OFF_SFB + STAGES * SF_STAGE;
    static constexpr int OFF_BAR = OFF_ACC + BT * ACC_PITCH * 4;
    // full[S], empty[S], sf_ready[SLOTS], sf_free[SLOTS], acc_full[2], acc_empty[2], drain, sga_ready
    static constexpr int NUM_BARS = 2 * STAGES + 2 * SF_SLOTS + 6;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;     // TMEM base, wait results, s_ga, amax partials
    static constexpr int SMEM_BYTES = OFF_MISC + 32 + 1024;
    static_assert(A_KT % 1024 == 0, "SW128 operand tiles are 1 KB aligned");
    static_assert(OFF_A + STAGES * A_STAGE - A_KT + 128 * KT_BYTES <= OFF_MISC, "MMA A reads stay in the buffer");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// Which CTA's range holds unit u when `units` are split over `ctas`:
// CTA c owns [floor(c U / G), floor((c+1) U / G)).
__device__ __forceinline__ int cta_of_unit(int64_t u, int units, int ctas)
{
    return (int)(((u + 1) * ctas + units - 1) / units) - 1;
}

// The stage starting at unit u of a CTA's range [u_begin, u_end): tile nb,
// k-tiles [kt, kt + nkt) (at most two, never crossing a tile), whether it
// opens and whether it closes a segment (the CTA's run of units in one tile).
struct Stage {
    int nb, kt, nkt;
    bool first, last;
};

__device__ __forceinline__ Stage stage_at(int64_t u, int64_t u_begin, int64_t u_end, int k_tiles)
{
    Stage s;
    s.nb = (int)(u / k_tiles);
    s.kt = (int)(u - (int64_t)s.nb * k_tiles);
    const int64_t seg_stop = min(u_end, (int64_t)(s.nb + 1) * k_tiles);
    s.nkt = (int)min((int64_t)KT_PER_STAGE, seg_stop - u);
    s.first = u == u_begin || s.kt == 0;
    s.last = u + s.nkt == seg_stop;
    return s;
}
}  // namespace decode

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

// Partial-tile words: (tag << 32) | FP32 bits, written and read as morally
// strong 8-byte accesses, so a word is either wholly this call's or not.
__device__ __forceinline__ void st_tagged4(unsigned long long* dst, float4 v, uint32_t tag)
{
    const unsigned long long t = (unsigned long long)tag << 32;
    asm volatile("st.relaxed.gpu.global.v2.b64 [%0], {%1, %2};" ::"l"(dst), "l"(t | __float_as_uint(v.x)),
                 "l"(t | __float_as_uint(v.y))
                 : "memory");
    asm volatile("st.relaxed.gpu.global.v2.b64 [%0], {%1, %2};" ::"l"(dst + 2), "l"(t | __float_as_uint(v.z)),
                 "l"(t | __float_as_uint(v.w))
                 : "memory");
}

// Four tagged words: load them, then (after any number of other loads are
// in flight) check that all carry this call's tag and unpack the values.
struct Tagged4 {
    unsigned long long w[4];
};

__device__ __forceinline__ void ld_tagged4(const unsigned long long* src, Tagged4& t)
{
    asm volatile("ld.relaxed.gpu.global.v2.b64 {%0, %1}, [%2];" : "=l"(t.w[0]), "=l"(t.w[1]) : "l"(src) : "memory");
    asm volatile("ld.relaxed.gpu.global.v2.b64 {%0, %1}, [%2];" : "=l"(t.w[2]), "=l"(t.w[3]) : "l"(src + 2) : "memory");
}

__device__ __forceinline__ bool tagged4_ok(const Tagged4& t, uint32_t tag)
{
    return (uint32_t)(t.w[0] >> 32) == tag && (uint32_t)(t.w[1] >> 32) == tag && (uint32_t)(t.w[2] >> 32) == tag &&
           (uint32_t)(t.w[3] >> 32) == tag;
}

__device__ __forceinline__ float4 tagged4_value(const Tagged4& t)
{
    return make_float4(__uint_as_float((uint32_t)t.w[0]), __uint_as_float((uint32_t)t.w[1]),
                       __uint_as_float((uint32_t)t.w[2]), __uint_as_float((uint32_t)t.w[3]));
}

// Copy k-tiles [kt, kt + nkt) of a 128-byte-wide operand (rows starting at
// `row`): one 3-D box for two k-tiles when the 3-D map exists (K a multiple of
// 256), else one 2-D box per k-tile.  Tiles of the stage sit `tile_bytes` apart.
__device__ __forceinline__ void load_ktiles(uint8_t* dst, const CUtensorMap* map2, const CUtensorMap* map3, bool use3,
                                            uint64_t* bar, int kt, int nkt, int row, int tile_bytes)
{
    if (use3 && nkt == 2) {
        asm volatile(
            "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
            " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
            "l"(map3), "r"(0), "r"(row), "r"(kt), "r"(smem_u32(bar))
            : "memory");
    } else {
        for (int j = 0; j < nkt; ++j)
            tma_load_2d(dst + j * tile_bytes, map2, bar, (kt + j) * decode::KT_BYTES, row);
    }
}

// The decode kernel's tensor maps: 2-D maps of the token rows (box 128 bytes x
// BT rows) and of the weight (128 bytes x 128 rows), and 3-D views
// {128 bytes, rows, K / 256} of the same buffers (boxes two k-tiles deep),
// used when K is a multiple of 256.
struct DecodeMaps {
    CUtensorMap a, w, a3, w3;
};

// FQ: the activation quantisation is fused in.  Warps 2 and 3 then quantise
// each stage's BT x 256 slices of the raw activations straight into the A
// stage (the 128-byte-swizzled layout the TMA would have written) and the
// scale atoms into the scale stage, with the same block arithmetic as
// quantize_kernel, so the result is bit-identical to quantising first.
template <int BT, bool FQ>
__global__ void __launch_bounds__(decode::THREADS, 1)
    gemm_decode_kernel(const __grid_constant__ DecodeMaps maps, const __grid_constant__ GemmParams p)
{
    using namespace decode;
    using C = Cfg<BT>;
    constexpr int STAGES = C::STAGES;
    constexpr int A_KT = C::A_KT, A_STAGE = C::A_STAGE;
    constexpr int OFF_A = C::OFF_A, OFF_W = C::OFF_W, OFF_SFA = C::OFF_SFA, OFF_SFB = C::OFF_SFB;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* empty = full + STAGES;
    uint64_t* sf_ready = empty + STAGES;
    uint64_t* sf_free = sf_ready + SF_SLOTS;
    uint64_t* acc_full = sf_free + SF_SLOTS;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* drain = acc_empty + 2;
    uint64_t* sga_ready = drain + 1;   // FQ: the activation scale is in s_ga_smem
    uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* bad = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);        // a wait ran out
    volatile int* wait_ok = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);    // the epilogue's shared wait result
    volatile float* s_ga_smem = reinterpret_cast<volatile float*>(smem + C::OFF_MISC + 12); // FQ: the scale used
    volatile float* amax_part = reinterpret_cast<volatile float*>(smem + C::OFF_MISC + 16); // FQ: [2]
    float* acc_stage = reinterpret_cast<float*>(smem + C::OFF_ACC);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int cta = blockIdx.x;
    const int64_t u_begin = (int64_t)cta * p.units / p.ctas;
    const int64_t u_end = (int64_t)(cta + 1) * p.units / p.ctas;
    const int k_tiles = p.k_tiles;
    const bool use3 = p.k % 256 == 0;
    // contributor c's partial tile: BT x BN tagged words at parts + c BT BN
    unsigned long long* parts = reinterpret_cast<unsigned long long*>(p.ws);
    const uint32_t tag = (uint32_t)p.epoch;

    if (warp == 0 && lane == 0) {
        prefetch_tensor_map(&maps.a);
        prefetch_tensor_map(&maps.w);
        prefetch_tensor_map(&maps.a3);
        prefetch_tensor_map(&maps.w3);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], FQ ? 3 : 1);    // FQ: the producer and the two quantiser warps
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < SF_SLOTS; ++i) {
            mbar_init(&sf_ready[i], 4);
            mbar_init(&sf_free[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], 4);
        }
        mbar_init(drain, 1);
        mbar_init(sga_ready, 1);
        *bad = 0;
        fence_mbarrier_init();
    }
    __syncthreads();
    // The next kernel in the stream may launch now; it waits for this one
    // before it reads or writes anything this one may write.
    if (threadIdx.x == 0) launch_dependents();

    uint32_t tmem_base = 0;
    if (warp != 0) {
        // Everything but the producer waits for the previous kernel here; then
        // TMEM, which that kernel may have held on this SM, is free.
        dependency_wait();
        if (warp == 2) {
            tmem_alloc(tmem_ptr, TMEM_COLS);
            tmem_relinquish();
        }
        if (warp != 3) {
            tc_fence_before();
            asm volatile("bar.sync 4, 320;" ::: "memory");   // warps 1, 2, 4..11
            tc_fence_after();
            tmem_base = *tmem_ptr;
        }
    }

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            bool ok = true;
            // Pass 1 (before the dependency wait): the weights and weight scales
            // of the first ring pass.  Without FQ each of these stages arrives
            // later, with its activation copies.
            int64_t u = u_begin;
            int pre = 0;
            for (; u < u_end && pre < STAGES; ++pre) {
                const Stage st = stage_at(u, u_begin, u_end, k_tiles);
                const int nsf = min(KSTEPS * st.nkt, p.katoms - st.kt * KSTEPS);
                const uint32_t wbytes = (uint32_t)(st.nkt * W_KT + nsf * 512);
                if (FQ)
                    mbar_arrive_expect_tx(&full[pre], wbytes);
                else
                    mbar_expect_tx(&full[pre], wbytes);
                load_ktiles(smem + OFF_W + pre * W_STAGE, &maps.w, &maps.w3, use3, &full[pre], st.kt, st.nkt,
                            st.nb * BN, W_KT);
                bulk_load(smem + OFF_SFB + pre * SF_STAGE, p.w_sf + ((int64_t)st.nb * p.katoms + st.kt * KSTEPS) * 512,
                          (uint32_t)nsf * 512u, &full[pre]);
                u += st.nkt;
            }
            dependency_wait();
            if (!FQ) {
                // Pass 2: the activation side of those stages.
                int64_t v = u_begin;
                for (int s = 0; s < pre; ++s) {
                    const Stage st = stage_at(v, u_begin, u_end, k_tiles);
                    const int nsf = min(KSTEPS * st.nkt, p.katoms - st.kt * KSTEPS);
                    mbar_arrive_expect_tx(&full[s], (uint32_t)(st.nkt * A_KT + nsf * 512));
                    load_ktiles(smem + OFF_A + s * A_STAGE, &maps.a, &maps.a3, use3, &full[s], st.kt, st.nkt, 0, A_KT);
                    bulk_load(smem + OFF_SFA + s * SF_STAGE, p.a_sf + (int64_t)st.kt * KSTEPS * 512,
                              (uint32_t)nsf * 512u, &full[s]);
                    v += st.nkt;
                }
            }
            // Steady state: whole stages as the ring frees them.
            int stage = 0;
            uint32_t phase = 1;
            while (u < u_end) {
                const Stage st = stage_at(u, u_begin, u_end, k_tiles);
                if (!mbar_wait(&empty[stage], phase ^ 1, kStatusTimeoutEmpty)) {
                    ok = false;
                    break;
                }
                const int nsf = min(KSTEPS * st.nkt, p.katoms - st.kt * KSTEPS);
                const uint32_t bytes =
                    (uint32_t)(st.nkt * W_KT + nsf * 512 + (FQ ? 0 : st.nkt * A_KT + nsf * 512));
                mbar_arrive_expect_tx(&full[stage], bytes);
                load_ktiles(smem + OFF_W + stage * W_STAGE, &maps.w, &maps.w3, use3, &full[stage], st.kt, st.nkt,
                            st.nb * BN, W_KT);
                bulk_load(smem + OFF_SFB + stage * SF_STAGE,
                          p.w_sf + ((int64_t)st.nb * p.katoms + st.kt * KSTEPS) * 512, (uint32_t)nsf * 512u,
                          &full[stage]);
                if (!FQ) {
                    load_ktiles(smem + OFF_A + stage * A_STAGE, &maps.a, &maps.a3, use3, &full[stage], st.kt, st.nkt, 0,
                                A_KT);
                    bulk_load(smem + OFF_SFA + stage * SF_STAGE, p.a_sf + (int64_t)st.kt * KSTEPS * 512,
                              (uint32_t)nsf * 512u, &full[stage]);
                }
                u += st.nkt;
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            if (!ok) {
                *bad = 1;
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
            int stage = 0, slot = 0, seg = 0;
            uint32_t slot_phase = 0;
            bool ok = true;
            for (int64_t u = u_begin; u < u_end;) {
                const Stage st = stage_at(u, u_begin, u_end, k_tiles);
                const int b = seg & 1;
                if (st.first) {
                    // a new segment: this accumulator's previous segment has been drained
                    if (!mbar_wait(&acc_empty[b], ((seg >> 1) & 1) ^ 1, kStatusTimeoutAccum)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                }
                if (!mbar_wait(&sf_ready[slot], slot_phase, kStatusTimeoutFull)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int nks = min(KSTEPS * st.nkt, p.katoms - st.kt * KSTEPS);
                const uint32_t sf_col = tmem_base + SF_COL + slot * SF_SLOT;
                const uint32_t acc = tmem_base + b * BN;
                const uint64_t adesc = desc_kmajor_sw128(smem + OFF_A + stage * A_STAGE);
                const uint64_t bdesc = desc_kmajor_sw128(smem + OFF_W + stage * W_STAGE);
                for (int ks = 0; ks < nks; ++ks) {
                    // k-tile j = ks / 4 of the stage, 64 FP4 values (32 bytes, +2 in the
                    // descriptor's 16-byte units) per k-step inside it
                    const int j = ks >> 2, q = ks & 3;
                    mma_nvf4(acc, adesc + (uint64_t)((j * A_KT) >> 4) + 2 * q, bdesc + (uint64_t)((j * W_KT) >> 4) + 2 * q,
                             idesc, !(st.first && ks == 0), sf_col + 4 * ks, sf_col + 32 + 4 * ks);
                }
                mma_commit(&empty[stage]);
                mma_commit(&sf_free[slot]);
                if (++stage == STAGES) stage = 0;
                if (++slot == SF_SLOTS) {
                    slot = 0;
                    slot_phase ^= 1;
                }
                if (st.last) {
                    mma_commit(&acc_full[b]);
                    ++seg;
                }
                u += st.nkt;
            }
            if (!ok) {
                *bad = 1;
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
        const int64_t esz = p.a_fp32 ? 4 : 2;
        // Each thread owns BT / 8 chunks (row r, 32 columns) of each k-tile of a
        // stage, taken two at a time: all loads of a pair are issued before any
        // arithmetic, and the first pair's loads before the wait for the stage
        // buffer (they do not need it), so the L2 round trip overlaps the wait.
        constexpr int CPT = BT / 8;
        constexpr int CB = CPT < 2 ? CPT : 2;
        for (int64_t u = u_begin; u < u_end;) {
            const Stage st = stage_at(u, u_begin, u_end, k_tiles);
            bool waited = false, ok = true;
            for (int h = 0; h < st.nkt && ok; ++h) {
                const int kt = st.kt + h;
                uint8_t* adst = smem + OFF_A + stage * A_STAGE + h * A_KT;
                uint8_t* sdst = smem + OFF_SFA + stage * SF_STAGE + h * SF_KT;
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
            }
            if (!ok) {
                *bad = 1;
                break;
            }
            fence_proxy_async_shared();     // the MMA reads the stage through the async proxy
            __syncwarp();
            if (lane == 0) mbar_arrive(&full[stage]);
            if (++stage == STAGES) {
                stage = 0;
                phase ^= 1;
            }
            u += st.nkt;
        }
    } else if (warp >= 8) {
        // ------------------------------------------------------------ scale staging
        // Lane l of quadrant q writes TMEM lane 32q + l: row l of every atom
        // (16 bytes = the scales of rows l, l+32, l+64, l+96), the layout the
        // block-scaled MMA reads for both operands; each k-tile of the stage
        // fills 16 columns of the slot's A half and 16 of its B half.
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        int stage = 0, slot = 0;
        uint32_t phase = 0, slot_phase = 0;
        for (int64_t u = u_begin; u < u_end;) {
            const Stage st = stage_at(u, u_begin, u_end, k_tiles);
            if (!mbar_wait(&full[stage], phase, kStatusTimeoutFull) ||
                !mbar_wait(&sf_free[slot], slot_phase ^ 1, kStatusTimeoutFull)) {
                *bad = 1;
                break;
            }
            tc_fence_after();
            const uint32_t col = tmem_base + lane_base + SF_COL + slot * SF_SLOT;
            for (int h = 0; h < st.nkt; ++h) {
                const uint8_t* sfa = smem + OFF_SFA + stage * SF_STAGE + h * SF_KT + lane * 16;
                const uint8_t* sfb = smem + OFF_SFB + stage * SF_STAGE + h * SF_KT + lane * 16;
                uint32_t ra[16], rb[16];
#pragma unroll
                for (int ks = 0; ks < KSTEPS; ++ks) {
                    const uint4 a = *reinterpret_cast<const uint4*>(sfa + ks * 512);
                    const uint4 b = *reinterpret_cast<const uint4*>(sfb + ks * 512);
                    ra[4 * ks] = a.x;
                    ra[4 * ks + 1] = a.y;
                    ra[4 * ks + 2] = a.z;
                    ra[4 * ks + 3] = a.w;
                    rb[4 * ks] = b.x;
                    rb[4 * ks + 1] = b.y;
                    rb[4 * ks + 2] = b.z;
                    rb[4 * ks + 3] = b.w;
                }
                tmem_st_32x32b_x16(col + 16 * h, ra);        // A: k-step ks at columns 4 ks .. 4 ks + 3
                tmem_st_32x32b_x16(col + 32 + 16 * h, rb);   // B: k-step ks at columns 32 + 4 ks ..
            }
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
            u += st.nkt;
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ epilogue
        // Per segment (one tile's k-range): the warps whose TMEM lanes hold
        // token rows move the FP32 accumulator into shared memory and release
        // it.  Then all 128 epilogue threads work on the staged tile, 4
        // consecutive columns of one row each: a contributor (a range that
        // starts inside the tile) writes its tagged partial to the workspace;
        // the owner of a tile that lies wholly in this range scales each
        // column by s_ga * s_gw[seg] and stores the output.  An owner whose
        // range ends inside the tile hands over to the all-warp finish below.
        // Every branch is uniform over the four warps, so the named barrier
        // (id 1, 128 threads) always matches.
        const int quad = warp & 3;
        const int et = threadIdx.x - 128;          // 0..127
        const int t = quad * 32 + lane;            // token row = accumulator lane
        const bool live = quad * 32 < BT;          // warp holds loaded token rows
        float s_ga = FQ ? 0.0f : *p.act_scale;        // FQ: known once the first stage is in
        const int units4 = min(p.m, BT) * (BN / 4);  // float4 units of the live rows
        int seg = 0;
        int64_t u = u_begin;
        while (u < u_end) {
            const int nb = (int)(u / k_tiles), kb = (int)(u - (int64_t)nb * k_tiles);
            const int64_t seg_end = min(u_end, (int64_t)(nb + 1) * k_tiles);
            const bool owner = kb == 0;
            const bool complete = owner && seg_end == (int64_t)(nb + 1) * k_tiles;
            const int b = seg & 1;

            if (et == 0) *wait_ok = mbar_wait(&acc_full[b], (seg >> 1) & 1, kStatusTimeoutAccum) ? 1 : 0;
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (!*wait_ok) {
                if (et == 0) *bad = 1;
                break;
            }
            if (FQ && seg == 0) {
                // bounded like every wait; the quantiser set it before its first stage
                if (et == 0) *wait_ok = mbar_wait(sga_ready, 0, kStatusTimeoutAccum) ? 1 : 0;
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (!*wait_ok) {
                    if (et == 0) *bad = 1;
                    break;
                }
                s_ga = *s_ga_smem;
            } else if (FQ) {
                s_ga = *s_ga_smem;
            }
            tc_fence_after();
            if (live) {
                const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + b * BN;
                float* row = acc_stage + t * ACC_PITCH;
                uint32_t r0[64], r1[64];
                __syncwarp();
                tmem_ld_32x32b_x64(taddr, r0);
                tmem_ld_32x32b_x64(taddr + 64, r1);
                tmem_ld_wait();
                if (t < BT) {
#pragma unroll
                    for (int e = 0; e < 64; e += 4) {
                        *reinterpret_cast<float4*>(row + e) =
                            make_float4(__uint_as_float(r0[e]), __uint_as_float(r0[e + 1]),
                                        __uint_as_float(r0[e + 2]), __uint_as_float(r0[e + 3]));
                        *reinterpret_cast<float4*>(row + 64 + e) =
                            make_float4(__uint_as_float(r1[e]), __uint_as_float(r1[e + 1]),
                                        __uint_as_float(r1[e + 2]), __uint_as_float(r1[e + 3]));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[b]);
            ++seg;
            // An owner whose range ends inside tile nb (always the CTA's last
            // segment) leaves the reduction to all twelve warps, below.
            if (owner && !complete) break;
            asm volatile("bar.sync 1, 128;" ::: "memory");   // staged tile complete

            if (!owner) {
                unsigned long long* mine = parts + (int64_t)cta * BT * BN;
                for (int x = et; x < units4; x += 128) {
                    const int r = x / (BN / 4), c4 = x % (BN / 4);
                    st_tagged4(mine + r * BN + 4 * c4, *reinterpret_cast<const float4*>(acc_stage + r * ACC_PITCH + 4 * c4),
                               tag);
                }
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
    // accumulator, all 384 threads add the contributors' partials (CTAs
    // cta + 1 .. last, in that order; FPG of them in flight per item and FDU
    // items per thread, each word waited for until it carries this call's
    // tag), scale and store.  The condition is the same for every thread.
    {
        const int64_t fin_nb = (u_end - 1) / k_tiles;
        const bool finish = u_end % k_tiles != 0 && fin_nb * k_tiles >= u_begin;
        if (finish) {
            asm volatile("bar.sync 2, 384;" ::: "memory");
            dependency_wait();
            if (!*bad) {
                constexpr int FDU = 2, FPG = 4;
                const int nb = (int)fin_nb;
                const int last = cta_of_unit((int64_t)(nb + 1) * k_tiles - 1, p.units, p.ctas);
                const int units4 = min(p.m, BT) * (BN / 4);
                const float s_ga = FQ ? *s_ga_smem : *p.act_scale;
                for (int x0 = threadIdx.x; x0 < units4; x0 += FDU * THREADS) {
                    float4 v[FDU];
                    int64_t off[FDU];
#pragma unroll
                    for (int i = 0; i < FDU; ++i) {
                        const int x = min(x0 + i * THREADS, units4 - 1);
                        off[i] = (int64_t)(x / (BN / 4)) * BN + 4 * (x % (BN / 4));
                        v[i] = *reinterpret_cast<const float4*>(acc_stage + (x / (BN / 4)) * ACC_PITCH +
                                                                4 * (x % (BN / 4)));
                    }
                    for (int c2 = cta + 1; c2 <= last; c2 += FPG) {
                        Tagged4 q[FDU][FPG];
#pragma unroll
                        for (int g = 0; g < FPG; ++g)
#pragma unroll
                            for (int i = 0; i < FDU; ++i)
                                if (c2 + g <= last) ld_tagged4(parts + (int64_t)(c2 + g) * BT * BN + off[i], q[i][g]);
                        uint32_t pending = 0;
#pragma unroll
                        for (int g = 0; g < FPG; ++g)
#pragma unroll
                            for (int i = 0; i < FDU; ++i)
                                if (c2 + g <= last && !tagged4_ok(q[i][g], tag)) pending |= 1u << (g * FDU + i);
                        if (pending) {
                            const long long t0 = clock64();
                            while (pending) {
#pragma unroll
                                for (int g = 0; g < FPG; ++g)
#pragma unroll
                                    for (int i = 0; i < FDU; ++i)
                                        if (pending & (1u << (g * FDU + i)))
                                            ld_tagged4(parts + (int64_t)(c2 + g) * BT * BN + off[i], q[i][g]);
#pragma unroll
                                for (int g = 0; g < FPG; ++g)
#pragma unroll
                                    for (int i = 0; i < FDU; ++i)
                                        if ((pending & (1u << (g * FDU + i))) && tagged4_ok(q[i][g], tag))
                                            pending &= ~(1u << (g * FDU + i));
                                if (pending && clock64() - t0 > kWaitCycles) {
                                    record_status(kStatusTimeoutCluster);
                                    *bad = 1;
                                    break;
                                }
                            }
                        }
#pragma unroll
                        for (int g = 0; g < FPG; ++g)
#pragma unroll
                            for (int i = 0; i < FDU; ++i)
                                if (c2 + g <= last) {
                                    const float4 w = tagged4_value(q[i][g]);
                                    v[i].x = __fadd_rn(v[i].x, w.x);
                                    v[i].y = __fadd_rn(v[i].y, w.y);
                                    v[i].z = __fadd_rn(v[i].z, w.z);
                                    v[i].w = __fadd_rn(v[i].w, w.w);
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
