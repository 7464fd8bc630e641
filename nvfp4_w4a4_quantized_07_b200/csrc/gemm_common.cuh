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
// This file holds what the GEMM kernels share: the segment table, the launch
// parameters and the output helpers.  The kernels:
//  * gemm_large.cuh: gemm_large_kernel, persistent (one CTA per SM) and
//    warp-specialised, 128 x 256 tiles; gemm_pair_kernel, the same on CTA
//    pairs (cta_group::2) with 256 x 256 tiles.
//  * gemm_decode.cuh: gemm_decode_kernel, small M (<= 64 tokens), bound by
//    streaming the weight.  Stream-K: the (256-column tile, 256-deep k-tile)
//    units are split evenly over one CTA per SM; a tile whose k-range spans
//    several CTAs is finished by the CTA holding its first k-tile, which adds
//    the others' FP32 partials in CTA order, so the result is deterministic.
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
    int splits;                 // (unused by the current kernels)
    // decode kernel (stream-K): work units = w_tiles x k_tiles, split evenly
    // over `ctas` co-resident CTAs; partial tiles meet in `ws`
    int units, ctas;
    uint8_t* ws;                // [256] uint64 flags, then [256][BT][256] FP32 partial tiles
    unsigned long long epoch;   // this call's flag value
    // decode kernel with the activation quantisation fused in: the raw
    // activations (act_scale == nullptr: dynamic scale amax/2688, computed by
    // every CTA; CTA 0 writes it to act_scale_out when that is given)
    const void* a_in;
    int64_t lda;
    int a_fp32;
    float* act_scale_out;
    // large-M kernel with the SwiGLU epilogue: the weight is [gate (f rows);
    // up (f rows)] and the epilogue writes h = bf16(silu(g) * u) quantised
    // with the static decode scale h_scale (codes m x f/2, tiled scales)
    int swiglu_f;
    const float* h_scale;
    uint8_t* h_q;
    uint8_t* h_sf;
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

}  // namespace nvfp4
