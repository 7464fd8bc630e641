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
__global__ void __launch_bounds__(256) amax_kernel(const void* __restrict__ x, int64_t rows, int64_t cols,
                                                   int64_t ldx, int in_fp32, unsigned int* __restrict__ out)
{
    const int64_t vec = in_fp32 ? 4 : 8;  // elements per 16-byte load
    const int64_t vpr = cols / vec;       // cols % 32 == 0
    const int64_t total = rows * vpr;
    float m = 0.0f;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / vpr, c = (i - r * vpr) * vec;
        if (in_fp32) {
            const float4 v = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(x) + r * ldx + c));
            m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
        } else {
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(x) + r * ldx + c));
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                m = fmaxf(m, fabsf(__uint_as_float(w[j] << 16)));
                m = fmaxf(m, fabsf(__uint_as_float(w[j] & 0xFFFF0000u)));
            }
        }
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
// Block quantiser.  A warp handles one 256-element segment of one row per
// unit (8 elements per lane, two lanes per 16-element block) and UNITS
// consecutive units per pass, issuing all loads first.
// ---------------------------------------------------------------------------
constexpr int kQuantUnits = 4;
constexpr int kQuantThreads = 256;

__device__ __forceinline__ void load8(const QuantParams& p, int64_t r, int64_t c0, bool live, float (&v)[8])
{
    if (!live) {
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = 0.0f;
        return;
    }
    if (p.in_fp32) {
        const float* src = static_cast<const float*>(p.x) + r * p.ldx + c0;
        const float4 a = __ldg(reinterpret_cast<const float4*>(src));
        const float4 b = __ldg(reinterpret_cast<const float4*>(src + 4));
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else {
        const uint4 a = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.x) + r * p.ldx + c0));
        const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            v[2 * j] = __uint_as_float(w[j] << 16);
            v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        }
    }
}

__global__ void __launch_bounds__(kQuantThreads) quantize_kernel(const __grid_constant__ QuantParams p)
{
    const int lane = threadIdx.x & 31;
    const int64_t segs = (p.k + 255) / 256;
    const int64_t nb = p.k / 16;
    const int64_t katoms = (nb + 3) / 4;
    const int64_t units = p.sf_rows_end * segs;
    const int64_t warp_global = ((int64_t)blockIdx.x * kQuantThreads + threadIdx.x) >> 5;
    const int64_t u0 = warp_global * kQuantUnits;
    if (u0 >= units) return;

    const float s_g = load_scale(p);
    if (p.scale_out != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *p.scale_out = s_g;
    const float t6 = __fmul_rn(6.0f, s_g);

    float v[kQuantUnits][8];
#pragma unroll
    for (int u = 0; u < kQuantUnits; ++u) {
        const int64_t unit = u0 + u;
        const int64_t r = unit / segs, seg = unit - r * segs;
        const int64_t c0 = seg * 256 + lane * 8;
        const bool live = unit < units && r < p.rows && c0 < p.k;
        load8(p, r, c0, live, v[u]);
    }

#pragma unroll
    for (int u = 0; u < kQuantUnits; ++u) {
        const int64_t unit = u0 + u;
        if (unit >= units) break;  // warp-uniform
        const int64_t r = unit / segs, seg = unit - r * segs;
        const int64_t c0 = seg * 256 + lane * 8;
        const bool row_live = r < p.rows;
        const bool live = row_live && c0 < p.k;

        float bm = 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j) bm = fmaxf(bm, fabsf(v[u][j]));
        bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 1));

        const uint32_t sb = live ? float_to_e4m3(__fdiv_rn(bm, t6)) : 0u;
        const float se = __fmul_rn(e4m3_to_float(sb), s_g);
        uint32_t packed = 0;
        if (se != 0.0f) {
            float inv = __frcp_rn(se);
            if (inv > FLT_MAX) inv = FLT_MAX;
            float y[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) y[j] = __fmul_rn(v[u][j], inv);
            packed = float8_to_e2m1x8(y);
        }
        const int64_t grow = p.row_offset + r;
        if (live) *reinterpret_cast<uint32_t*>(p.q + grow * (p.k / 2) + c0 / 2) = packed;

        // Scale bytes: even lanes own block kb = seg*16 + lane/2.  Gather each
        // group of four consecutive blocks (one 32-bit word of an atom row) in
        // lane 8i and store it whole; blocks past K/16 contribute zero padding.
        const uint32_t b1 = __shfl_down_sync(0xffffffffu, sb, 2);
        const uint32_t b2 = __shfl_down_sync(0xffffffffu, sb, 4);
        const uint32_t b3 = __shfl_down_sync(0xffffffffu, sb, 6);
        const int64_t kb0 = seg * 16 + (lane >> 1);
        if ((lane & 7) == 0 && kb0 < katoms * 4) {
            const uint32_t word = sb | (b1 << 8) | (b2 << 16) | (b3 << 24);
            *reinterpret_cast<uint32_t*>(p.sf + sf_tiled_offset(grow, kb0, katoms)) = word;
        }
    }
}

}  // namespace nvfp4
