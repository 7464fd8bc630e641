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
//    streaming the weight.  Stream-K: the (128-column tile, 256-deep k-tile)
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
    uint8_t* ws;                // [MAX_CTAS][BT][128] tagged partial-tile words
    unsigned long long epoch;   // this call's value; its low 32 bits tag the partial words
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
    // Gated DeltaNet gates from two head-wide column ranges of the BF16
    // output (gdn_heads == 0: none): g from columns [gdn_a_col, + heads),
    // beta from [gdn_b_col, + heads); FP32 outputs m x heads, row stride gdn_ld
    int gdn_heads, gdn_a_col, gdn_b_col;
    const float* gdn_A_log;
    const float* gdn_dt_bias;
    float* gdn_g;
    float* gdn_beta;
    int64_t gdn_ld;
    // large-M kernel: tile i of the persistent schedule is tile (i + tile_shift)
    // mod the tile count (0 keeps the column-major order)
    int tile_shift;
    // large-M kernel with the activation quantisation fused in: the raw BF16
    // activations (a_in, lda) are quantised with the static scale *act_scale
    // into qa_q / qa_sf (the buffers the A tensor map and a_sf point to);
    // m-block j may be loaded once qa_ready[j] == (call tag << 32 | CTAs).
    // The first qa_first m-blocks are quantised by every warp but the
    // producer and the MMA issuer before the mainloop, the rest by warps 2-3
    // while it runs.
    uint8_t* qa_q;
    uint8_t* qa_sf;
    unsigned long long* qa_ready;
    int qa_first;
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

// The Gated DeltaNet gates ("Why Gated DeltaNet Survives 4-Bit Quantization",
// page summary, "Gated DeltaNet Mechanics"; the sigmoid for beta from the
// abstract's mechanism (ii)) from one stored output element x = C[row, col],
// the BF16 value the next layer would read:
//   column a_col + h:  g[row, h]    = -exp(A_log[h]) * softplus(x + dt_bias[h])
//   column b_col + h:  beta[row, h] = 1 / (1 + exp(-x))
// Both are evaluated so that no intermediate overflows or goes subnormal on
// the common path (large |x| would otherwise send exp, log1p and the divide
// into their special-value paths): softplus(t) = max(t, 0) + log1p(exp(-|t|)),
// which equals t (t >= 17) or exp(t) (t <= -17) to within 2^-25 relative in
// FP32; the sigmoid as r or e * r with e = exp(-|x|) <= 1 and r the correctly
// rounded reciprocal of 1 + e, a value in [1, 2].
__device__ __forceinline__ float gdn_g(float x, float dt_bias, float rate)
{
    const float t = __fadd_rn(x, dt_bias);
    const float at = fabsf(t);
    const float e = expf(-at);                                   // = exp(t) when t < 0
    const float tail = t > 0.0f ? t : e;
    const float sp = at >= 17.0f ? tail : __fadd_rn(fmaxf(t, 0.0f), log1pf(e));
    return -__fmul_rn(rate, sp);
}

__device__ __forceinline__ float gdn_beta(float x)
{
    const float e = expf(-fabsf(x));
    const float r = __frcp_rn(__fadd_rn(1.0f, e));
    return x >= 0.0f ? r : __fmul_rn(e, r);
}

// Whether output columns [col0, col0 + ncols) hold any gate input.
__device__ __forceinline__ bool gdn_touches(const GemmParams& p, int col0, int ncols)
{
    return p.gdn_heads > 0 && ((col0 < p.gdn_a_col + p.gdn_heads && p.gdn_a_col < col0 + ncols) ||
                               (col0 < p.gdn_b_col + p.gdn_heads && p.gdn_b_col < col0 + ncols));
}

// Gates from 4 consecutive stored columns of one row (the decode kernel's
// output unit); called only where gdn_touches holds.
__device__ __forceinline__ void gdn_gate4(const GemmParams& p, int row, int col, float x0, float x1, float x2, float x3)
{
    const float x[4] = {x0, x1, x2, x3};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const unsigned ha = (unsigned)(col + e - p.gdn_a_col), hb = (unsigned)(col + e - p.gdn_b_col);
        if (ha < (unsigned)p.gdn_heads)
            p.gdn_g[(int64_t)row * p.gdn_ld + ha] = gdn_g(x[e], p.gdn_dt_bias[ha], expf(p.gdn_A_log[ha]));
        if (hb < (unsigned)p.gdn_heads) p.gdn_beta[(int64_t)row * p.gdn_ld + hb] = gdn_beta(x[e]);
    }
}

// Gates from one 16-row x 32-column BF16 output chunk staged in shared memory
// (64-byte rows; 16-byte unit u of row r at (u ^ ((r / 2) % 4)) * 16): lane =
// column; the head's parameters are read once and four rows at a time are
// unrolled so that their exp/log1p chains overlap (rows are otherwise a
// serial chain of dependent transcendental steps in a single warp).
__device__ __forceinline__ void gdn_chunk(const GemmParams& p, const uint8_t* cbuf, int row0, int col0, int lane)
{
    const int col = col0 + lane;
    const unsigned ha = (unsigned)(col - p.gdn_a_col), hb = (unsigned)(col - p.gdn_b_col);
    const bool is_a = ha < (unsigned)p.gdn_heads, is_b = hb < (unsigned)p.gdn_heads;
    if (!is_a && !is_b) return;
    const float dt_bias = is_a ? p.gdn_dt_bias[ha] : 0.0f;
    const float rate = is_a ? expf(p.gdn_A_log[ha]) : 0.0f;
    const int rows = min(16, p.m - row0);
    float* g = p.gdn_g + (int64_t)row0 * p.gdn_ld + ha;
    float* beta = p.gdn_beta + (int64_t)row0 * p.gdn_ld + hb;
#pragma unroll 4
    for (int r = 0; r < 16; ++r) {
        // every row of the buffer is read (rows past m hold stale values whose
        // results are dropped), so only the stores are conditional and the
        // unrolled rows' chains can interleave
        const uint8_t* src = cbuf + r * 64 + ((((lane >> 3) ^ ((r >> 1) & 3)) << 4) | ((lane & 7) << 1));
        const float x = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(src));
        if (is_a) {
            const float v = gdn_g(x, dt_bias, rate);
            if (r < rows) g[r * p.gdn_ld] = v;
        }
        if (is_b) {
            const float v = gdn_beta(x);
            if (r < rows) beta[r * p.gdn_ld] = v;
        }
    }
}

}  // namespace nvfp4
