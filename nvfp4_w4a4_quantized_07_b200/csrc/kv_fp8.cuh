// Calibrated FP8 (E4M3) KV cache: the serving recipe pairs the NVFP4 W4A4
// linear layers with an FP8 KV cache whose per-tensor scales are calibrated
// offline and shipped with the checkpoint ("Why Gated DeltaNet Survives 4-Bit
// Quantization": abstract; Glonce article, "How to use it"; aiany.app,
// "Mechanistic notes").
//
//   scale s (per tensor, K and V separately) = amax / 448, or 1 if that is 0
//   cache byte = E4M3_rne_satfinite(x * (1 / s)),   read back as byte * s
//
// kv_fp8_quantize_kernel quantises the new tokens' K and V rows and scatters
// them into the cache slots a slot table names, in one launch.  It moves 2 (or
// 4) bytes in and 1 byte out per element and does a handful of instructions
// per element, so it is bound by HBM: one thread handles 16 consecutive
// elements of a row (one or two 16-byte loads in flight per 16-byte store),
// consecutive threads take consecutive pieces of a row, and the grid is a few
// waves of resident blocks striding over the K units and then the V units.
#pragma once

#include <cuda_bf16.h>
#include <float.h>
#include <stdint.h>

namespace nvfp4 {

constexpr int kKvThreads = 256;
constexpr float kFp8Max = 448.0f;  // largest finite E4M3 value

struct KvParams {
    const void* x[2];        // K and V rows, tokens x width, row strides ld[] elements
    int64_t ld[2];
    int in_fp32;
    uint32_t tokens;
    uint32_t chunks;         // width / 16
    uint32_t units;          // tokens * chunks (per tensor)
    const int64_t* slots;    // cache slot of each token (NULL: slot = token)
    int64_t num_slots;
    const float* scale[2];   // calibrated per-tensor scales (device)
    uint8_t* cache[2];       // num_slots x width bytes, row stride cache_ld bytes
    int64_t cache_ld;
};

// 1 / s, correctly rounded, clamped to FLT_MAX if it overflows.
__device__ __forceinline__ float fp8_inverse_scale(float s)
{
    const float inv = __frcp_rn(s);
    return inv > FLT_MAX ? FLT_MAX : inv;
}

// Two products -> two E4M3 bytes, the first in the low byte.
__device__ __forceinline__ uint32_t fp8x2(float lo, float hi)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ uint32_t fp8x4(float a, float b, float c, float d)
{
    return fp8x2(a, b) | (fp8x2(c, d) << 16);
}

__device__ __forceinline__ void bf16x8_to_float(const uint4 v, float (&f)[8])
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

__global__ void __launch_bounds__(kKvThreads) kv_fp8_quantize_kernel(const __grid_constant__ KvParams p)
{
    const uint32_t total = 2 * p.units;
    const uint32_t stride = gridDim.x * blockDim.x;
    for (uint32_t u = blockIdx.x * blockDim.x + threadIdx.x; u < total; u += stride) {
        const int tensor = u >= p.units;              // 0: K, 1: V
        const uint32_t w = u - (tensor ? p.units : 0);
        const uint32_t t = w / p.chunks, c = w - t * p.chunks;
        const int64_t slot = p.slots != nullptr ? p.slots[t] : (int64_t)t;
        if (slot < 0 || slot >= p.num_slots) continue;  // padding token (or a slot past the cache)
        const float inv = fp8_inverse_scale(*p.scale[tensor]);
        float f[16];
        if (p.in_fp32) {
            const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(p.x[tensor]) +
                                                                (int64_t)t * p.ld[tensor] + 16 * c);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float4 v = __ldg(src + i);
                f[4 * i] = v.x;
                f[4 * i + 1] = v.y;
                f[4 * i + 2] = v.z;
                f[4 * i + 3] = v.w;
            }
        } else {
            const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.x[tensor]) +
                                                              (int64_t)t * p.ld[tensor] + 16 * c);
            const uint4 v0 = __ldg(src), v1 = __ldg(src + 1);
            float lo[8], hi[8];
            bf16x8_to_float(v0, lo);
            bf16x8_to_float(v1, hi);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                f[i] = lo[i];
                f[8 + i] = hi[i];
            }
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) f[i] = __fmul_rn(f[i], inv);
        const uint4 out = make_uint4(fp8x4(f[0], f[1], f[2], f[3]), fp8x4(f[4], f[5], f[6], f[7]),
                                     fp8x4(f[8], f[9], f[10], f[11]), fp8x4(f[12], f[13], f[14], f[15]));
        *reinterpret_cast<uint4*>(p.cache[tensor] + slot * p.cache_ld + 16 * (int64_t)c) = out;
    }
}

// scale = amax / 448 (1 if that is 0) from a running amax held as float bits.
__global__ void fp8_scale_kernel(const float* __restrict__ amax, float* __restrict__ scale)
{
    if (threadIdx.x == 0 && blockIdx.x == 0) {
        const float s = __fdiv_rn(*amax, kFp8Max);
        *scale = s == 0.0f ? 1.0f : s;
    }
}

}  // namespace nvfp4
