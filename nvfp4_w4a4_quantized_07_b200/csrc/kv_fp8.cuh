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
// per element, so it is bound by HBM: a piece is 16 consecutive elements of a
// row (two or four 16-byte loads, one 16-byte store), consecutive threads take
// consecutive pieces of a row, and a grid of resident blocks strides over the
// K pieces and then the V pieces, two pieces per thread at a time.
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

// Piece u (K pieces first, then V): its raw 16-byte words as loaded (two for
// BF16, four for FP32) and where it goes.
template <bool FP32>
struct KvPiece {
    uint4 raw[FP32 ? 4 : 2];
    int tensor;
    uint32_t t, c;
};

template <bool FP32>
__device__ __forceinline__ void kv_load(const KvParams& p, uint32_t u, KvPiece<FP32>& x)
{
    x.tensor = u >= p.units;
    const uint32_t w = u - (x.tensor ? p.units : 0);
    x.t = w / p.chunks;
    x.c = w - x.t * p.chunks;
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.x[x.tensor]) +
                                                      ((int64_t)x.t * p.ld[x.tensor] + 16 * (int64_t)x.c) *
                                                          (FP32 ? 4 : 2));
#pragma unroll
    for (int i = 0; i < (FP32 ? 4 : 2); ++i) x.raw[i] = __ldg(src + i);
}

template <bool FP32>
__device__ __forceinline__ void kv_store(const KvParams& p, const KvPiece<FP32>& x, int64_t slot, float inv)
{
    if (slot < 0 || slot >= p.num_slots) return;  // padding token (or a slot past the cache)
    float y[16];
    if (FP32) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            y[4 * i] = __uint_as_float(x.raw[i].x);
            y[4 * i + 1] = __uint_as_float(x.raw[i].y);
            y[4 * i + 2] = __uint_as_float(x.raw[i].z);
            y[4 * i + 3] = __uint_as_float(x.raw[i].w);
        }
    } else {
        float lo[8], hi[8];
        bf16x8_to_float(x.raw[0], lo);
        bf16x8_to_float(x.raw[FP32 ? 0 : 1], hi);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            y[i] = lo[i];
            y[8 + i] = hi[i];
        }
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) y[i] = __fmul_rn(y[i], inv);
    const uint4 out = make_uint4(fp8x4(y[0], y[1], y[2], y[3]), fp8x4(y[4], y[5], y[6], y[7]),
                                 fp8x4(y[8], y[9], y[10], y[11]), fp8x4(y[12], y[13], y[14], y[15]));
    *reinterpret_cast<uint4*>(p.cache[x.tensor] + slot * p.cache_ld + 16 * (int64_t)x.c) = out;
}

// Two pieces per iteration, their loads (and slot-table reads) issued before
// either is converted, so each thread keeps 64 (BF16) or 128 (FP32) bytes in
// flight; the scales are read once.
template <bool FP32>
__global__ void __launch_bounds__(kKvThreads) kv_fp8_quantize_kernel(const __grid_constant__ KvParams p)
{
    const uint64_t total = 2ull * p.units;  // < 2^32
    const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    const float inv_k = fp8_inverse_scale(*p.scale[0]), inv_v = fp8_inverse_scale(*p.scale[1]);
    for (uint64_t u = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; u < total; u += 2 * stride) {
        const bool two = u + stride < total;
        KvPiece<FP32> a, b;
        kv_load(p, (uint32_t)u, a);
        if (two) kv_load(p, (uint32_t)(u + stride), b);
        const int64_t sa = p.slots != nullptr ? p.slots[a.t] : (int64_t)a.t;
        const int64_t sb = two ? (p.slots != nullptr ? p.slots[b.t] : (int64_t)b.t) : -1;
        kv_store(p, a, sa, a.tensor ? inv_v : inv_k);
        if (two) kv_store(p, b, sb, b.tensor ? inv_v : inv_k);
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
