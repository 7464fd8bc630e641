// NVFP4 quantisation kernels.
//
// Format ("Why Gated DeltaNet Survives 4-Bit Quantization", page summary,
// "Background", item 1): E2M1 values, one E4M3 scale per 16-element block set
// to blockmax/6, one FP32 scale per tensor.  Two-level reading: the tensor's
// decode scale is s_g = amax / 2688 (1 if that is 0); the block's E4M3 byte is
// sb = E4M3(bm / (6 s_g)); elements are encoded as E2M1(x * (1 / (e4m3(sb) s_g))).
// Every FP32 step rounds to nearest even (explicit _rn intrinsics, no FMA
// contraction, denormals kept), so the bytes are reproducible bit for bit.
//
// Layout written:
//   q  : rows x K/2 bytes, row-major, element 2j in the low nibble of byte j.
//   sf : tiled for the block-scaled MMA: 512-byte atoms of 128 rows x 4 scale
//        columns; inside an atom row r sits at (r%32)*16 + (r/32)*4, scale
//        column c at +c; atoms run along K first, then down 128-row blocks;
//        rows pad to 128 and K/16 to 4 with zero bytes.
#pragma once

#include <cuda_bf16.h>
#include <float.h>
#include <stdint.h>

#include "ptx.cuh"

namespace nvfp4 {

constexpr float kGlobalScaleDenominator = 2688.0f;  // 6 (largest E2M1) * 448 (largest E4M3)

enum ScaleMode : int {
    kScaleValue = 0,      // s_g passed by value
    kScaleDevice = 1,     // s_g read from a device float
    kScaleFromAmax = 2,   // s_g = amax / 2688 with amax read from a device float
};

struct QuantParams {
    const void* x;        // rows x k, row stride ldx elements
    int64_t rows;
    int64_t k;
    int64_t ldx;
    int in_fp32;          // 0: BF16, 1: FP32
    uint8_t* q;           // fused buffer base (row 0)
    uint8_t* sf;          // fused tiled scale buffer base
    int64_t row_offset;   // first row of this tensor inside the fused buffers
    int64_t sf_rows_end;  // rows (relative) whose scale entries this call writes (>= rows; covers padding)
    int scale_mode;
    const float* scale_ptr;
    float scale_value;
    float* scale_out;     // optional: receives s_g (written by one thread)
};

__device__ __forceinline__ float global_scale_from_amax(float amax)
{
    float s = __fdiv_rn(amax, kGlobalScaleDenominator);
    return s == 0.0f ? 1.0f : s;
}

// E4M3 byte (non-negative) -> float, exact.
__device__ __forceinline__ float e4m3_to_float(uint32_t b)
{
    const uint32_t e = (b >> 3) & 15u, m = b & 7u;
    if (e == 0) return (float)m * 0.001953125f;  // m * 2^-9, subnormal
    return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// Round-to-nearest-even, saturating FP32 -> E4M3 (hardware conversion).
__device__ __forceinline__ uint32_t float_to_e4m3(float v)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %1;" : "=h"(r) : "f"(v));
    return r & 0xFFu;
}

// Eight FP32 -> eight E2M1 codes packed into 32 bits, element 2j in the low
// nibble of byte j.  The paired conversion puts its FIRST source operand in
// the high nibble, so each pair is passed as (odd, even).
__device__ __forceinline__ uint32_t float8_to_e2m1x8(const float (&y)[8])
{
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(y[0]), "f"(y[1]), "f"(y[2]), "f"(y[3]), "f"(y[4]), "f"(y[5]), "f"(y[6]), "f"(y[7]));
    return r;
}

__device__ __forceinline__ int64_t sf_tiled_offset(int64_t row, int64_t kb, int64_t katoms)
{
    return (((row >> 7) * katoms + (kb >> 2)) << 9) + ((row & 31) << 4) + (((row >> 5) & 3) << 2) + (kb & 3);
}

__device__ __forceinline__ float load_scale(const QuantParams& p)
{
    if (p.scale_mode == kScaleValue) return p.scale_value;
    const float v = *p.scale_ptr;
    return p.scale_mode == kScaleFromAmax ? global_scale_from_amax(v) : v;
}

// ---------------------------------------------------------------------------
// amax = max |x| over a rows x cols matrix, combined into *out with an
// integer atomicMax on the (non-negative) float bits: order-independent and
// therefore deterministic.  *out must hold 0 (or a smaller amax) beforehand.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float absmax_vec(const void* base, int64_t elem_index, int in_fp32)
{
    if (in_fp32) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(base) + elem_index));
        return fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
    }
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(base) + elem_index));
    // |bf16| as the float with the sign bit cleared; both halves of each word.
    float m = 0.0f;
    m = fmaxf(m, __uint_as_float((v.x << 16) & 0x7FFF0000u));
    m = fmaxf(m, __uint_as_float(v.x & 0x7FFF0000u));
    m = fmaxf(m, __uint_as_float((v.y << 16) & 0x7FFF0000u));
    m = fmaxf(m, __uint_as_float(v.y & 0x7FFF0000u));
    m = fmaxf(m, __uint_as_float((v.z << 16) & 0x7FFF0000u));
    m = fmaxf(m, __uint_as_float(v.z & 0x7FFF0000u));
    m = fmaxf(m, __uint_as_float((v.w << 16) & 0x7FFF0000u));
    m = fmaxf(m, __uint_as_float(v.w & 0x7FFF0000u));
    return m;
}

__global__ void __launch_bounds__(256) amax_kernel(const void* __restrict__ x, int64_t rows, int64_t cols,
                                                   int64_t ldx, int in_fp32, unsigned int* __restrict__ out)
{
    const int64_t vec = in_fp32 ? 4 : 8;  // elements per 16-byte load; cols % 32 == 0
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    float m = 0.0f;
    if (ldx == cols) {
        // contiguous: one flat pass, four independent loads in flight per thread
        const int64_t nvec = rows * cols / vec;
        int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
        for (; i + 3 * stride < nvec; i += 4 * stride) {
            const float a0 = absmax_vec(x, i * vec, in_fp32);
            const float a1 = absmax_vec(x, (i + stride) * vec, in_fp32);
            const float a2 = absmax_vec(x, (i + 2 * stride) * vec, in_fp32);
            const float a3 = absmax_vec(x, (i + 3 * stride) * vec, in_fp32);
            m = fmaxf(m, fmaxf(fmaxf(a0, a1), fmaxf(a2, a3)));
        }
        for (; i < nvec; i += stride) m = fmaxf(m, absmax_vec(x, i * vec, in_fp32));
    } else {
        for (int64_t r = blockIdx.x; r < rows; r += gridDim.x)
            for (int64_t c = (int64_t)threadIdx.x * vec; c < cols; c += (int64_t)blockDim.x * vec)
                m = fmaxf(m, absmax_vec(x, r * ldx + c, in_fp32));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    __shared__ float red[8];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float b = 0.0f;
        for (int i = 0; i < (int)(blockDim.x >> 5); ++i) b = fmaxf(b, red[i]);
        if (b > 0.0f) atomicMax(out, __float_as_uint(b));
    }
}

// ---------------------------------------------------------------------------
// Block quantiser: one thread per two consecutive 16-element blocks.  Threads
// are numbered row-major over rows [row_begin, row_begin + launch rows) x the
// padded block pairs [0, 2 * katoms), so a warp reads 64 consecutive blocks
// (1024 values) of a row and writes 512 consecutive packed bytes.  Two
// neighbouring lanes hold one 32-bit word of a scale atom (four blocks), which
// the even lane stores.  Threads on padding (row >= rows or block >= K/16)
// write zero scales only.
// ---------------------------------------------------------------------------
constexpr int kQuantThreads = 256;

struct QuantLaunch {
    int64_t row_begin;    // first (relative) row of this launch
    uint32_t pairs;       // block pairs per row: 2 * katoms
    uint32_t total;       // threads that map to a (row, pair): rows_in_launch * pairs
    uint32_t div_mul;     // t / pairs == __umulhi(4 t, div_mul) >> div_shift for t < 2^30
    uint32_t div_shift;
};

__device__ __forceinline__ void quantize_block16(const float (&v)[16], float s_g, bool live, uint32_t& sb,
                                                 uint2& packed)
{
    float bm = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) bm = fmaxf(bm, fabsf(v[j]));
    sb = live ? float_to_e4m3(__fdiv_rn(bm, __fmul_rn(6.0f, s_g))) : 0u;
    const float se = __fmul_rn(e4m3_to_float(sb), s_g);
    packed = make_uint2(0u, 0u);
    if (se != 0.0f) {
        float inv = __frcp_rn(se);
        if (inv > FLT_MAX) inv = FLT_MAX;
        float y[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) y[j] = __fmul_rn(v[j], inv);
        packed.x = float8_to_e2m1x8(y);
#pragma unroll
        for (int j = 0; j < 8; ++j) y[j] = __fmul_rn(v[8 + j], inv);
        packed.y = float8_to_e2m1x8(y);
    }
}

__device__ __forceinline__ void unpack_bf16x8(const uint4& a, float* v)
{
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        v[2 * j] = __uint_as_float(w[j] << 16);
        v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
    }
}

// Quantise the two blocks a thread holds and store their codes and, from the
// even lane of each lane pair, the 32-bit scale word of four blocks.  Must be
// reached by every lane of the warp (the scale bytes are exchanged by shuffle).
__device__ __forceinline__ void quantize_pair_store(const QuantParams& p, const QuantLaunch& l, bool mapped,
                                                    uint32_t pr, int64_t r, int64_t kb0, bool live0, bool live1,
                                                    float s_g, const float (&v0)[16], const float (&v1)[16])
{
    uint32_t sb0, sb1;
    uint2 q0, q1;
    quantize_block16(v0, s_g, live0, sb0, q0);
    quantize_block16(v1, s_g, live1, sb1, q1);
    const int64_t grow = p.row_offset + r;
    uint8_t* qdst = p.q + grow * (p.k >> 1) + kb0 * 8;
    if (live1)
        *reinterpret_cast<uint4*>(qdst) = make_uint4(q0.x, q0.y, q1.x, q1.y);
    else if (live0)
        *reinterpret_cast<uint2*>(qdst) = q0;

    // Four consecutive blocks form one 32-bit word of an atom row.
    const uint32_t half = sb0 | (sb1 << 8);
    const uint32_t other = __shfl_down_sync(0xffffffffu, half, 1);
    if (mapped && (pr & 1u) == 0u) {
        const uint32_t word = half | (other << 16);
        *reinterpret_cast<uint32_t*>(p.sf + sf_tiled_offset(grow, kb0, l.pairs >> 1)) = word;
    }
}

// Each thread quantises ITEMS (row, block pair) items, 256 threads apart,
// and issues the loads of all of them before any arithmetic: two BF16 items
// keep 128 bytes of input in flight per thread within the register budget of
// four resident blocks (a streaming kernel is bound by the bytes in flight
// per SM).  FP32 input (64 bytes per item) takes one item per thread.
constexpr int kQuantMinBlocks = 4;

template <int ITEMS, bool FP32>
__global__ void __launch_bounds__(kQuantThreads, kQuantMinBlocks) quantize_kernel(const __grid_constant__ QuantParams p,
                                                                                const QuantLaunch l)
{
    constexpr int kQuantItems = ITEMS;
    // A GEMM launched after this kernel with programmatic dependent launch may
    // start now (it loads weights until this kernel has completed).
    if (threadIdx.x == 0) launch_dependents();
    const uint32_t t_first = blockIdx.x * (kQuantThreads * kQuantItems) + threadIdx.x;
    const int64_t nb = p.k >> 4;
    const float s_g = load_scale(p);
    if (p.scale_out != nullptr && t_first == 0 && l.row_begin == 0) *p.scale_out = s_g;

    bool mapped[kQuantItems], live0[kQuantItems], live1[kQuantItems];
    uint32_t pr[kQuantItems];
    int64_t r[kQuantItems], kb0[kQuantItems];
    uint4 u[kQuantItems][FP32 ? 8 : 4];
#pragma unroll
    for (int i = 0; i < kQuantItems; ++i) {
        const uint32_t t = t_first + i * kQuantThreads;
        mapped[i] = t < l.total;
        const uint32_t rl = mapped[i] ? __umulhi(t << 2, l.div_mul) >> l.div_shift : 0u;
        pr[i] = mapped[i] ? t - rl * l.pairs : 0u;
        r[i] = l.row_begin + rl;
        kb0[i] = (int64_t)pr[i] * 2;
        const bool row_live = mapped[i] && r[i] < p.rows;
        live0[i] = row_live && kb0[i] < nb;
        live1[i] = row_live && kb0[i] + 1 < nb;
        if (FP32) {
            const uint4* src = reinterpret_cast<const uint4*>(static_cast<const float*>(p.x) + r[i] * p.ldx + kb0[i] * 16);
#pragma unroll
            for (int j = 0; j < 8; ++j) u[i][j] = ((j < 4) ? live0[i] : live1[i]) ? __ldcs(src + j) : make_uint4(0, 0, 0, 0);
        } else {
            const uint4* src =
                reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.x) + r[i] * p.ldx + kb0[i] * 16);
#pragma unroll
            for (int j = 0; j < 4; ++j) u[i][j] = ((j < 2) ? live0[i] : live1[i]) ? __ldcs(src + j) : make_uint4(0, 0, 0, 0);
        }
    }
#pragma unroll
    for (int i = 0; i < kQuantItems; ++i) {
        float v0[16], v1[16];
        if (FP32) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                v0[4 * j] = __uint_as_float(u[i][j].x);
                v0[4 * j + 1] = __uint_as_float(u[i][j].y);
                v0[4 * j + 2] = __uint_as_float(u[i][j].z);
                v0[4 * j + 3] = __uint_as_float(u[i][j].w);
                v1[4 * j] = __uint_as_float(u[i][4 + j].x);
                v1[4 * j + 1] = __uint_as_float(u[i][4 + j].y);
                v1[4 * j + 2] = __uint_as_float(u[i][4 + j].z);
                v1[4 * j + 3] = __uint_as_float(u[i][4 + j].w);
            }
        } else {
            unpack_bf16x8(u[i][0], v0);
            unpack_bf16x8(u[i][1], v0 + 8);
            unpack_bf16x8(u[i][2], v1);
            unpack_bf16x8(u[i][3], v1 + 8);
        }
        quantize_pair_store(p, l, mapped[i], pr[i], r[i], kb0[i], live0[i], live1[i], s_g, v0, v1);
    }
}

// ---------------------------------------------------------------------------
// MLP glue: h = bf16(silu(g) * u) with silu(x) = x / (1 + e^-x), each step in
// FP32 with round-to-nearest (e^-x from CUDA's expf), from the BF16 gate and up
// halves of a fused gate/up GEMM output; h is then quantised like an
// activation with its own tensor scale.  Same thread mapping as
// quantize_kernel: one thread per two 16-element blocks of one row.
// ---------------------------------------------------------------------------
struct SiluParams {
    const __nv_bfloat16* g;   // rows x f, row stride ldgu
    const __nv_bfloat16* u;   // rows x f, row stride ldgu
    int64_t ldgu;
    __nv_bfloat16* h;         // optional rows x f output, row stride ldh (nullptr: not written)
    int64_t ldh;
};

// h as the float value of its BF16 rounding.
__device__ __forceinline__ float silu_mul_bf16(float g, float u)
{
    const float e = expf(-g);
    const float s = __fdiv_rn(g, __fadd_rn(1.0f, e));
    return __bfloat162float(__float2bfloat16_rn(__fmul_rn(s, u)));
}

__device__ __forceinline__ uint32_t pack_bf16_pair(float lo, float hi)
{
    return (__float_as_uint(lo) >> 16) | (__float_as_uint(hi) & 0xFFFF0000u);  // both already BF16 values
}

// Load the thread's 32 gate and 32 up values, form h for both blocks and, if
// requested, store h.
__device__ __forceinline__ void silu_mul_pair(const SiluParams& sp, int64_t r, int64_t kb0, bool live0, bool live1,
                                              float (&v0)[16], float (&v1)[16])
{
    const uint4* gs = reinterpret_cast<const uint4*>(sp.g + r * sp.ldgu + kb0 * 16);
    const uint4* us = reinterpret_cast<const uint4*>(sp.u + r * sp.ldgu + kb0 * 16);
    uint4 gw[4], uw[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const bool live = (j < 2) ? live0 : live1;
        gw[j] = live ? __ldcs(gs + j) : make_uint4(0, 0, 0, 0);
        uw[j] = live ? __ldcs(us + j) : make_uint4(0, 0, 0, 0);
    }
    float gf[32], uf[32];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        unpack_bf16x8(gw[j], gf + 8 * j);
        unpack_bf16x8(uw[j], uf + 8 * j);
    }
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        v0[e] = silu_mul_bf16(gf[e], uf[e]);
        v1[e] = silu_mul_bf16(gf[16 + e], uf[16 + e]);
    }
    if (sp.h != nullptr) {
        uint4* hd = reinterpret_cast<uint4*>(sp.h + r * sp.ldh + kb0 * 16);
        if (live0) {
            hd[0] = make_uint4(pack_bf16_pair(v0[0], v0[1]), pack_bf16_pair(v0[2], v0[3]),
                               pack_bf16_pair(v0[4], v0[5]), pack_bf16_pair(v0[6], v0[7]));
            hd[1] = make_uint4(pack_bf16_pair(v0[8], v0[9]), pack_bf16_pair(v0[10], v0[11]),
                               pack_bf16_pair(v0[12], v0[13]), pack_bf16_pair(v0[14], v0[15]));
        }
        if (live1) {
            hd[2] = make_uint4(pack_bf16_pair(v1[0], v1[1]), pack_bf16_pair(v1[2], v1[3]),
                               pack_bf16_pair(v1[4], v1[5]), pack_bf16_pair(v1[6], v1[7]));
            hd[3] = make_uint4(pack_bf16_pair(v1[8], v1[9]), pack_bf16_pair(v1[10], v1[11]),
                               pack_bf16_pair(v1[12], v1[13]), pack_bf16_pair(v1[14], v1[15]));
        }
    }
}

// Pass 1 of the dynamic-scale glue: amax of h (optionally storing h).
__global__ void __launch_bounds__(kQuantThreads) silu_mul_amax_kernel(const __grid_constant__ QuantParams p,
                                                                    const __grid_constant__ SiluParams sp,
                                                                    const QuantLaunch l, unsigned int* amax)
{
    const uint32_t t = blockIdx.x * kQuantThreads + threadIdx.x;
    const bool mapped = t < l.total;
    const uint32_t rl = mapped ? __umulhi(t << 2, l.div_mul) >> l.div_shift : 0u;
    const uint32_t pr = mapped ? t - rl * l.pairs : 0u;
    const int64_t r = l.row_begin + rl;
    const int64_t kb0 = (int64_t)pr * 2;
    const bool row_live = mapped && r < p.rows;
    const bool live0 = row_live && kb0 < (p.k >> 4);
    const bool live1 = row_live && kb0 + 1 < (p.k >> 4);
    float v0[16], v1[16];
    silu_mul_pair(sp, r, kb0, live0, live1, v0, v1);
    float m = 0.0f;
#pragma unroll
    for (int e = 0; e < 16; ++e) m = fmaxf(m, fmaxf(fabsf(v0[e]), fabsf(v1[e])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    __shared__ float red[kQuantThreads / 32];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float b = 0.0f;
        for (int i = 0; i < kQuantThreads / 32; ++i) b = fmaxf(b, red[i]);
        if (b > 0.0f) atomicMax(amax, __float_as_uint(b));
    }
}

// h = bf16(silu(g) * u) quantised to NVFP4 (optionally storing h).
__global__ void __launch_bounds__(kQuantThreads) silu_mul_quantize_kernel(const __grid_constant__ QuantParams p,
                                                                        const __grid_constant__ SiluParams sp,
                                                                        const QuantLaunch l)
{
    const uint32_t t = blockIdx.x * kQuantThreads + threadIdx.x;
    const bool mapped = t < l.total;
    const uint32_t rl = mapped ? __umulhi(t << 2, l.div_mul) >> l.div_shift : 0u;
    const uint32_t pr = mapped ? t - rl * l.pairs : 0u;
    const int64_t r = l.row_begin + rl;
    const int64_t kb0 = (int64_t)pr * 2;
    const bool row_live = mapped && r < p.rows;
    const bool live0 = row_live && kb0 < (p.k >> 4);
    const bool live1 = row_live && kb0 + 1 < (p.k >> 4);

    const float s_g = load_scale(p);
    if (p.scale_out != nullptr && t == 0 && l.row_begin == 0) *p.scale_out = s_g;
    float v0[16], v1[16];
    silu_mul_pair(sp, r, kb0, live0, live1, v0, v1);
    quantize_pair_store(p, l, mapped, pr, r, kb0, live0, live1, s_g, v0, v1);
}

}  // namespace nvfp4
