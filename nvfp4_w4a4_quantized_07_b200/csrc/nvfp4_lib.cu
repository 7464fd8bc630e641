// libnvfp4: the C ABI declared in include/nvfp4.h.  Argument validation, TMA
// descriptor creation and kernel launches; all arithmetic runs in the kernels
// of quant.cuh, gemm_large.cuh and gemm_decode.cuh.  Single translation unit.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <atomic>
#include <chrono>
#include <mutex>
#include <random>

#include "../../include/nvfp4.h"
#include "gemm_decode.cuh"
#include "gemm_large.cuh"
#include "kv_fp8.cuh"
#include "quant.cuh"

using namespace nvfp4;

namespace {

constexpr int kVersion = 100;  // 0.1.0
constexpr int kMaxDevices = 64;

thread_local char g_err[512] = "";

nvfp4_status fail(nvfp4_status st, const char* fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return st;
}

nvfp4_status ok()
{
    g_err[0] = '\0';
    return NVFP4_OK;
}

#define NVFP4_CUDA_TRY(expr)                                                                         \
    do {                                                                                            \
        cudaError_t e_ = (expr);                                                                    \
        if (e_ != cudaSuccess) return fail(NVFP4_ERR_CUDA, "%s: %s", #expr, cudaGetErrorString(e_)); \
    } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t pad_to(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

// ---------------------------------------------------------------------------
// Per-device state: SM count and one-time kernel attribute setup.
// ---------------------------------------------------------------------------
struct DeviceState {
    bool ready = false;
    int sms = 0;
};
DeviceState g_dev[kMaxDevices];
std::mutex g_dev_mutex;

nvfp4_status device_state(DeviceState** out)
{
    int dev = 0;
    NVFP4_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return fail(NVFP4_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    DeviceState& d = g_dev[dev];
    if (!d.ready) {
        int major = 0, minor = 0;
        NVFP4_CUDA_TRY(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
        NVFP4_CUDA_TRY(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
        if (major != 10 || minor != 0)
            return fail(NVFP4_ERR_UNSUPPORTED, "device %d is sm_%d%d; libnvfp4 is built for sm_100a only", dev, major,
                        minor);
        NVFP4_CUDA_TRY(cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev));
        NVFP4_CUDA_TRY(cudaFuncSetAttribute(gemm_large_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            large::SMEM_BYTES));
        NVFP4_CUDA_TRY(cudaFuncSetAttribute(gemm_large_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            large::SMEM_BYTES));
        NVFP4_CUDA_TRY(cudaFuncSetAttribute(gemm_large_kernel<false, true>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, large::SMEM_BYTES));
        NVFP4_CUDA_TRY(cudaFuncSetAttribute(gemm_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            pairk::SMEM_BYTES));
        NVFP4_CUDA_TRY(cudaFuncSetAttribute(gemm_decode_kernel<16, false>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, decode::Cfg<16>::SMEM_BYTES));
        NVFP4_CUDA_TRY(cudaFuncSetAttribute(gemm_decode_kernel<16, true>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, decode::Cfg<16>::SMEM_BYTES));
        NVFP4_CUDA_TRY(cudaFuncSetAttribute(gemm_decode_kernel<32, false>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, decode::Cfg<32>::SMEM_BYTES));
        NVFP4_CUDA_TRY(cudaFuncSetAttribute(gemm_decode_kernel<32, true>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, decode::Cfg<32>::SMEM_BYTES));
        NVFP4_CUDA_TRY(cudaFuncSetAttribute(gemm_decode_kernel<64, false>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, decode::Cfg<64>::SMEM_BYTES));
        NVFP4_CUDA_TRY(cudaFuncSetAttribute(gemm_decode_kernel<64, true>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, decode::Cfg<64>::SMEM_BYTES));
        d.ready = true;
    }
    *out = &d;
    return NVFP4_OK;
}

// ---------------------------------------------------------------------------
// TMA descriptors through the CUDA driver API entry point (no link-time libcuda).
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

nvfp4_status encode_fp4_map(CUtensorMap* map, const uint8_t* base, int64_t rows, int64_t k, int box_rows)
{
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    if (g_encode == nullptr) return fail(NVFP4_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    // Packed FP4 viewed as bytes: dim 0 = K/2 bytes (contiguous), dim 1 = rows.
    const cuuint64_t dims[2] = {(cuuint64_t)(k / 2), (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)(k / 2)};
    const cuuint32_t box[2] = {128u, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1u, 1u};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(NVFP4_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return NVFP4_OK;
}

// 3-D view {128 bytes, rows, K / 256} of a packed FP4 buffer (row stride K/2
// bytes, k-tile stride 128 bytes) for boxes of two k-tiles of box_rows rows,
// which land as two consecutive 128-byte-swizzled tiles.  Needs K % 256 == 0,
// so every box lies inside the buffer.
nvfp4_status encode_fp4_map3(CUtensorMap* map, const uint8_t* base, int64_t rows, int64_t k, int box_rows)
{
    const cuuint64_t dims[3] = {128u, (cuuint64_t)rows, (cuuint64_t)(k / 256)};
    const cuuint64_t strides[2] = {(cuuint64_t)(k / 2), 128u};
    const cuuint32_t box[3] = {128u, (cuuint32_t)box_rows, 2u};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(NVFP4_ERR_CUDA, "cuTensorMapEncodeTiled (3-D) failed (%d)", (int)r);
    return NVFP4_OK;
}

// The decode kernel's maps: A with boxes of bt rows, W with boxes of 128 rows,
// and their two-k-tile 3-D views when K is a multiple of 256 (else copies of
// the 2-D maps, which the kernel then never reads as 3-D).  a_q == nullptr:
// the activations are quantised inside the kernel and A's maps are unused.
nvfp4_status encode_decode_maps(DecodeMaps* m, const uint8_t* a_q, const uint8_t* w_q, int64_t rows_a, int64_t n,
                                int64_t k, int bt)
{
    nvfp4_status st = encode_fp4_map(&m->w, w_q, n, k, decode::BN);
    if (st != NVFP4_OK) return st;
    if (a_q != nullptr) {
        if ((st = encode_fp4_map(&m->a, a_q, rows_a, k, bt)) != NVFP4_OK) return st;
    } else {
        m->a = m->w;
    }
    if (k % 256 == 0) {
        if ((st = encode_fp4_map3(&m->w3, w_q, n, k, decode::BN)) != NVFP4_OK) return st;
        if (a_q != nullptr) {
            if ((st = encode_fp4_map3(&m->a3, a_q, rows_a, k, bt)) != NVFP4_OK) return st;
        } else {
            m->a3 = m->w3;
        }
    } else {
        m->w3 = m->w;
        m->a3 = m->a;
    }
    return NVFP4_OK;
}

// Output C (m x n, row stride ldc elements) for TMA stores of 32-column
// chunks from swizzled shared memory: BF16 chunks are 16 rows of 64 bytes
// (64-byte swizzle); the FP32 map (32 x 32, 128-byte swizzle) is encoded for
// completeness, FP32 output is written with plain stores.  Stores past m or n
// are clipped by the copy engine.
// Output map: boxes of 32 columns x `bf16_rows` rows (BF16, 64-byte swizzle)
// or 32 x 32 (FP32, 128-byte swizzle).
nvfp4_status encode_c_map(CUtensorMap* map, void* c, int64_t m, int64_t n, int64_t ldc, bool fp32, int bf16_rows = 16)
{
    const cuuint64_t dims[2] = {(cuuint64_t)n, (cuuint64_t)m};
    const cuuint64_t strides[1] = {(cuuint64_t)(ldc * (fp32 ? 4 : 2))};
    const cuuint32_t box[2] = {32u, fp32 ? 32u : (cuuint32_t)bf16_rows};
    const cuuint32_t estr[2] = {1u, 1u};
    CUresult r = g_encode(map, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, c, dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          fp32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                          CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(NVFP4_ERR_CUDA, "cuTensorMapEncodeTiled (output) failed (%d)", (int)r);
    return NVFP4_OK;
}

// ---------------------------------------------------------------------------
// Quantisation launch shared by the activation and weight entry points.
// ---------------------------------------------------------------------------
nvfp4_status check_quant_input(const void* x, nvfp4_in_dtype dt, int64_t rows, int64_t k, int64_t ld,
                               const char* what)
{
    if (dt != NVFP4_IN_BF16 && dt != NVFP4_IN_FP32) return fail(NVFP4_ERR_INVALID_ARG, "%s: bad input dtype", what);
    if (rows < 0 || k <= 0 || k % 32 != 0)
        return fail(NVFP4_ERR_INVALID_ARG, "%s: need rows >= 0 and k a positive multiple of 32 (rows=%lld k=%lld)",
                    what, (long long)rows, (long long)k);
    if (rows >= (1ll << 31) || k >= (1ll << 31)) return fail(NVFP4_ERR_UNSUPPORTED, "%s: dimension >= 2^31", what);
    if (ld < k) return fail(NVFP4_ERR_INVALID_ARG, "%s: leading dimension %lld < k %lld", what, (long long)ld,
                            (long long)k);
    const int64_t esz = dt == NVFP4_IN_FP32 ? 4 : 2;
    if (rows > 0 && x == nullptr) return fail(NVFP4_ERR_INVALID_ARG, "%s: input pointer is NULL", what);
    if (!aligned16(x) || (ld * esz) % 16 != 0)
        return fail(NVFP4_ERR_ALIGNMENT, "%s: input rows must start on 16-byte boundaries", what);
    return NVFP4_OK;
}

// max(*out, amax(x)) into *out (float bits; *out holds a non-negative float).
nvfp4_status launch_amax_into(const void* x, nvfp4_in_dtype dt, int64_t rows, int64_t k, int64_t ld, unsigned int* out,
                              cudaStream_t s, int sms)
{
    if (rows == 0) return NVFP4_OK;
    const int64_t vec = dt == NVFP4_IN_FP32 ? 4 : 8;
    const int64_t total = rows * (k / vec);
    int64_t blocks = (total + 255) / 256;
    if (blocks > (int64_t)sms * 8) blocks = (int64_t)sms * 8;
    amax_kernel<<<(unsigned)blocks, 256, 0, s>>>(x, rows, k, ld, dt == NVFP4_IN_FP32, out);
    NVFP4_CUDA_TRY(cudaGetLastError());
    return NVFP4_OK;
}

nvfp4_status launch_amax(const void* x, nvfp4_in_dtype dt, int64_t rows, int64_t k, int64_t ld, void* ws,
                         cudaStream_t s, int sms)
{
    NVFP4_CUDA_TRY(cudaMemsetAsync(ws, 0, sizeof(unsigned int), s));
    return launch_amax_into(x, dt, rows, k, ld, static_cast<unsigned int*>(ws), s, sms);
}

// Multiply-shift constants for exact unsigned division by d (1 <= d < 2^31) of
// every dividend t < 2^30:  t / d == umulhi(4 t, mul) >> shift  with
// shift = ceil(log2 d) and mul = ceil(2^(30 + shift) / d) (< 2^32).  The
// rounding error t (mul - 2^(30+shift)/d) / 2^(30+shift) stays below
// 2^-shift <= 1/d, so the floor is exact.
void magic_divider(uint32_t d, uint32_t* mul, uint32_t* shift)
{
    uint32_t s = 0;
    while ((1ull << s) < d) ++s;
    *mul = (uint32_t)(((1ull << (30 + s)) + d - 1) / d);
    *shift = s;
}

enum QuantKind { kQuantPlain, kQuantSiluMul, kAmaxSiluMul };

// One thread per (row, pair of 16-element blocks) over rows [0, rows_end);
// launches of at most 2^30 threads keep the in-kernel index 32-bit.
nvfp4_status launch_quant(const QuantParams& p, cudaStream_t s, QuantKind kind = kQuantPlain,
                          const SiluParams* sp = nullptr, unsigned int* amax = nullptr)
{
    const int64_t pairs = pad_to(p.k / 16, 4) / 2;
    const int64_t rows_end = kind == kAmaxSiluMul ? p.rows : p.sf_rows_end;
    if (rows_end == 0) return NVFP4_OK;
    const int64_t rows_per_launch = ((int64_t)1 << 30) / pairs;
    if (rows_per_launch < 1) return fail(NVFP4_ERR_UNSUPPORTED, "quantise: k too large");
    QuantLaunch l;
    l.pairs = (uint32_t)pairs;
    magic_divider(l.pairs, &l.div_mul, &l.div_shift);
    for (int64_t r0 = 0; r0 < rows_end; r0 += rows_per_launch) {
        const int64_t rows = rows_end - r0 < rows_per_launch ? rows_end - r0 : rows_per_launch;
        l.row_begin = r0;
        l.total = (uint32_t)(rows * pairs);
        const unsigned blocks = (unsigned)((l.total + kQuantThreads - 1) / kQuantThreads);
        if (kind == kQuantPlain && !p.in_fp32)
            quantize_kernel<2, false><<<(unsigned)((l.total + kQuantThreads * 2 - 1) / (kQuantThreads * 2)),
                                        kQuantThreads, 0, s>>>(p, l);
        else if (kind == kQuantPlain)
            quantize_kernel<1, true><<<blocks, kQuantThreads, 0, s>>>(p, l);
        else if (kind == kQuantSiluMul)
            silu_mul_quantize_kernel<<<blocks, kQuantThreads, 0, s>>>(p, *sp, l);
        else
            silu_mul_amax_kernel<<<blocks, kQuantThreads, 0, s>>>(p, *sp, l, amax);
        NVFP4_CUDA_TRY(cudaGetLastError());
    }
    return NVFP4_OK;
}

nvfp4_status check_segments(const nvfp4_segment* segs, int nsegs, int64_t n, SegTable* out)
{
    if (segs == nullptr || nsegs < 1 || nsegs > NVFP4_MAX_SEGMENTS)
        return fail(NVFP4_ERR_INVALID_ARG, "gemm: need 1..%d segments (got %d)", NVFP4_MAX_SEGMENTS, nsegs);
    int64_t expect = 0;
    out->count = nsegs;
    for (int i = 0; i < nsegs; ++i) {
        const nvfp4_segment& g = segs[i];
        if (g.col_begin != expect)
            return fail(NVFP4_ERR_INVALID_ARG, "gemm: segment %d starts at %lld, expected %lld (sorted, contiguous)", i,
                        (long long)g.col_begin, (long long)expect);
        if (g.col_end <= g.col_begin)
            return fail(NVFP4_ERR_INVALID_ARG, "gemm: segment %d is empty or reversed", i);
        if (g.col_end % 16 != 0)
            return fail(NVFP4_ERR_INVALID_ARG, "gemm: segment %d ends at %lld, not a multiple of 16", i,
                        (long long)g.col_end);
        if (!(g.w_global_scale > 0.0f) || !std::isfinite(g.w_global_scale))
            return fail(NVFP4_ERR_INVALID_ARG, "gemm: segment %d scale must be positive and finite", i);
        out->end[i] = (int)g.col_end;
        out->scale[i] = g.w_global_scale;
        expect = g.col_end;
    }
    for (int i = nsegs; i < kMaxSegments; ++i) {
        out->end[i] = (int)n;
        out->scale[i] = out->scale[nsegs - 1];
    }
    if (expect != n)
        return fail(NVFP4_ERR_INVALID_ARG, "gemm: segments cover [0, %lld), expected [0, %lld)", (long long)expect,
                    (long long)n);
    return NVFP4_OK;
}

// Bytes of workspace the decode kernel needs for m tokens: one partial tile
// (16, 32 or 64 rows x 128 columns of tagged 8-byte words) per CTA slot.
size_t decode_ws_bytes(int64_t m)
{
    const int64_t bt = m <= 16 ? 16 : (m <= 32 ? 32 : 64);
    return (size_t)decode::MAX_CTAS * (size_t)bt * decode::BN * 8;
}

// Per-call tags for the decode kernel's partial-tile hand-off: a random
// starting point (so words left in a reused workspace by another process or an
// aborted call do not match) advanced once per call; the kernel uses the low
// 32 bits, which repeat only after 2^31 calls.
std::atomic<unsigned long long> g_epoch{0};
std::once_flag g_epoch_once;

unsigned long long next_epoch()
{
    std::call_once(g_epoch_once, [] {
        std::random_device rd;
        const unsigned long long seed = ((unsigned long long)rd() << 32) ^ rd() ^
                                        (unsigned long long)std::chrono::steady_clock::now().time_since_epoch().count();
        g_epoch.store(seed | 1ull);
    });
    return g_epoch.fetch_add(2ull) + 2ull;
}

// Per-call tags of the fused prefill kernel's ready words: 1, 2, 3, ... in
// this process (the kernel raises each word to the current tag with an atomic
// maximum, so tags must grow; 2^32 - 1 calls before they wrap).
std::atomic<unsigned int> g_prefill_tag{0};

unsigned long long next_prefill_tag()
{
    return (unsigned long long)g_prefill_tag.fetch_add(1u) + 1ull;
}

template <int BT, bool FQ>
nvfp4_status launch_decode(const DecodeMaps& maps, const GemmParams& p, cudaStream_t s)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.ctas, 1, 1);
    cfg.blockDim = dim3(decode::THREADS, 1, 1);
    cfg.dynamicSmemBytes = decode::Cfg<BT>::SMEM_BYTES;
    cfg.stream = s;
    // Programmatic dependent launch: the CTAs may start while the previous
    // kernel in the stream is still running; each touches only weights until
    // it has waited for that kernel (griddepcontrol.wait).  The grid is at
    // most one CTA per SM, so once the previous kernel is done every CTA is
    // resident; the participants of split tiles wait for each other's
    // partials with a bounded wait.
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    NVFP4_CUDA_TRY(cudaLaunchKernelEx(&cfg, gemm_decode_kernel<BT, FQ>, maps, p));
    return NVFP4_OK;
}

}  // namespace

// ---------------------------------------------------------------------------
// Built-in scratch of nvfp4_gemm_decode_noalloc: the decode kernel's partial
// tiles for up to NVFP4_NOALLOC_MAX_M tokens and every CTA slot, in device
// memory reserved when the module is loaded on a device (no allocation call).
// Its address on each device is looked up once, with that device current.
// ---------------------------------------------------------------------------
static_assert(NVFP4_NOALLOC_SCRATCH_BYTES == (size_t)decode::MAX_CTAS * NVFP4_NOALLOC_MAX_M * decode::BN * 8,
              "scratch = one 16-row partial tile per CTA slot");
static __device__ __align__(256) unsigned char g_noalloc_scratch[NVFP4_NOALLOC_SCRATCH_BYTES];

namespace {
void* g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mutex;

nvfp4_status noalloc_scratch(void** out)
{
    int dev = 0;
    NVFP4_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return fail(NVFP4_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (g_noalloc_ptr[dev] == nullptr) {
        void* ptr = nullptr;
        NVFP4_CUDA_TRY(cudaGetSymbolAddress(&ptr, g_noalloc_scratch));
        if (ptr == nullptr || (reinterpret_cast<uintptr_t>(ptr) & 255u) != 0)
            return fail(NVFP4_ERR_CUDA, "gemm_decode_noalloc: scratch address %p is not 256-byte aligned", ptr);
        g_noalloc_ptr[dev] = ptr;
    }
    *out = g_noalloc_ptr[dev];
    return NVFP4_OK;
}
}  // namespace

// ===========================================================================
// C ABI
// ===========================================================================
extern "C" {

size_t nvfp4_sf_bytes(int64_t rows, int64_t k)
{
    if (rows < 0 || k <= 0 || k % 16 != 0) return 0;
    return (size_t)(pad_to(rows, 128) * pad_to(k / 16, 4));
}

int64_t nvfp4_sf_offset(int64_t row, int64_t kblock, int64_t k)
{
    if (row < 0 || k <= 0 || k % 16 != 0 || kblock < 0 || kblock >= pad_to(k / 16, 4)) return -1;
    const int64_t katoms = pad_to(k / 16, 4) / 4;
    return ((row / 128) * katoms + kblock / 4) * 512 + (row % 32) * 16 + ((row % 128) / 32) * 4 + kblock % 4;
}

size_t nvfp4_quant_workspace_size(void) { return 256; }

size_t nvfp4_gemm_workspace_size(int64_t m, int64_t n, int64_t k, uint32_t flags)
{
    (void)n;
    (void)k;
    const bool decode_path = flags == NVFP4_GEMM_FORCE_DECODE || (flags == NVFP4_GEMM_AUTO && m <= 64);
    return decode_path && m >= 0 && m <= 64 ? decode_ws_bytes(m) : 0;
}

int nvfp4_gemm_kernel_for(int64_t m, int64_t n, int sms, uint32_t flags, int with_gates)
{
    if (m < 0 || n <= 0 || sms <= 0 || flags > NVFP4_GEMM_FORCE_LARGE_PAIR) return -1;
    if (flags != NVFP4_GEMM_AUTO) return (int)flags;
    if (m <= 64) return (int)NVFP4_GEMM_FORCE_DECODE;
    // Large M: the CTA-pair kernel (256 x 256 tiles on two SMs) when it needs
    // no more waves of tiles than the single-CTA kernel (128 x 256 tiles, one
    // per SM).  Per SM the two do the same work per wave and the pair kernel
    // runs each wave about 2 % faster.  Calls with gate outputs keep the
    // single-CTA kernel, which schedules the gate tiles first.
    if (with_gates || m < 256 || sms < 2) return (int)NVFP4_GEMM_FORCE_LARGE;
    const int64_t n_blocks = (n + 255) / 256;
    const int64_t single_waves = ((m + 127) / 128 * n_blocks + sms - 1) / sms;
    const int64_t pair_waves = ((m + 255) / 256 * n_blocks + sms / 2 - 1) / (sms / 2);
    return (int)(pair_waves <= single_waves ? NVFP4_GEMM_FORCE_LARGE_PAIR : NVFP4_GEMM_FORCE_LARGE);
}

const char* nvfp4_get_last_error_string(void) { return g_err; }

int nvfp4_version(void) { return kVersion; }

nvfp4_status nvfp4_quantize_act(const void* a, nvfp4_in_dtype dt, int64_t m, int64_t k, int64_t lda,
                                const float* act_scale_dev, float* act_scale_out_dev, uint8_t* a_q, uint8_t* a_sf,
                                void* workspace, size_t ws_bytes, void* stream)
{
    nvfp4_status st = check_quant_input(a, dt, m, k, lda, "quantize_act");
    if (st != NVFP4_OK) return st;
    if (m > 0 && (a_q == nullptr || a_sf == nullptr))
        return fail(NVFP4_ERR_INVALID_ARG, "quantize_act: a_q / a_sf is NULL");
    if (!aligned16(a_q) || !aligned16(a_sf)) return fail(NVFP4_ERR_ALIGNMENT, "quantize_act: outputs not 16-byte aligned");
    const bool dynamic = act_scale_dev == nullptr;
    if (dynamic) {
        if (act_scale_out_dev == nullptr)
            return fail(NVFP4_ERR_INVALID_ARG, "quantize_act: dynamic mode needs act_scale_out_dev");
        if (workspace == nullptr || ws_bytes < nvfp4_quant_workspace_size())
            return fail(NVFP4_ERR_WORKSPACE, "quantize_act: dynamic mode needs %zu bytes of workspace",
                        nvfp4_quant_workspace_size());
        if (!aligned16(workspace)) return fail(NVFP4_ERR_ALIGNMENT, "quantize_act: workspace not 16-byte aligned");
    }
    if (m == 0) return ok();
    DeviceState* dev = nullptr;
    if ((st = device_state(&dev)) != NVFP4_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dynamic && (st = launch_amax(a, dt, m, k, lda, workspace, s, dev->sms)) != NVFP4_OK) return st;
    QuantParams p = {};
    p.x = a;
    p.rows = m;
    p.k = k;
    p.ldx = lda;
    p.in_fp32 = dt == NVFP4_IN_FP32;
    p.q = a_q;
    p.sf = a_sf;
    p.row_offset = 0;
    p.sf_rows_end = pad_to(m, 128);
    p.scale_mode = dynamic ? kScaleFromAmax : kScaleDevice;
    p.scale_ptr = dynamic ? static_cast<const float*>(workspace) : act_scale_dev;
    p.scale_out = act_scale_out_dev;
    if ((st = launch_quant(p, s)) != NVFP4_OK) return st;
    return ok();
}

nvfp4_status nvfp4_silu_mul_quantize(const void* g, const void* u, int64_t m, int64_t f, int64_t ldgu,
                                     const float* h_scale_dev, float* h_scale_out_dev, uint8_t* h_q, uint8_t* h_sf,
                                     void* h_out, int64_t ldh, void* workspace, size_t ws_bytes, void* stream)
{
    if (m < 0 || f <= 0 || f % 32 != 0)
        return fail(NVFP4_ERR_INVALID_ARG, "silu_mul_quantize: need m >= 0 and f a positive multiple of 32 "
                                           "(m=%lld f=%lld)", (long long)m, (long long)f);
    if (m >= (1ll << 31) || f >= (1ll << 31)) return fail(NVFP4_ERR_UNSUPPORTED, "silu_mul_quantize: dimension >= 2^31");
    if (ldgu < f) return fail(NVFP4_ERR_INVALID_ARG, "silu_mul_quantize: ldgu %lld < f %lld", (long long)ldgu,
                              (long long)f);
    if (h_out != nullptr && ldh < f)
        return fail(NVFP4_ERR_INVALID_ARG, "silu_mul_quantize: ldh %lld < f %lld", (long long)ldh, (long long)f);
    if (m > 0 && (g == nullptr || u == nullptr || h_q == nullptr || h_sf == nullptr))
        return fail(NVFP4_ERR_INVALID_ARG, "silu_mul_quantize: NULL input or output pointer");
    if (!aligned16(g) || !aligned16(u) || (ldgu * 2) % 16 != 0 || !aligned16(h_q) || !aligned16(h_sf) ||
        !aligned16(h_out) || (h_out != nullptr && (ldh * 2) % 16 != 0))
        return fail(NVFP4_ERR_ALIGNMENT, "silu_mul_quantize: rows and outputs must be 16-byte aligned");
    const bool dynamic = h_scale_dev == nullptr;
    if (dynamic) {
        if (h_scale_out_dev == nullptr)
            return fail(NVFP4_ERR_INVALID_ARG, "silu_mul_quantize: dynamic mode needs h_scale_out_dev");
        if (workspace == nullptr || ws_bytes < nvfp4_quant_workspace_size())
            return fail(NVFP4_ERR_WORKSPACE, "silu_mul_quantize: dynamic mode needs %zu bytes of workspace",
                        nvfp4_quant_workspace_size());
        if (!aligned16(workspace)) return fail(NVFP4_ERR_ALIGNMENT, "silu_mul_quantize: workspace not 16-byte aligned");
    }
    if (m == 0) return ok();
    DeviceState* dev = nullptr;
    nvfp4_status st = device_state(&dev);
    if (st != NVFP4_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    QuantParams p = {};
    p.x = g;
    p.rows = m;
    p.k = f;
    p.ldx = ldgu;
    p.q = h_q;
    p.sf = h_sf;
    p.sf_rows_end = pad_to(m, 128);
    p.scale_mode = dynamic ? kScaleFromAmax : kScaleDevice;
    p.scale_ptr = dynamic ? static_cast<const float*>(workspace) : h_scale_dev;
    p.scale_out = h_scale_out_dev;
    SiluParams sp;
    sp.g = static_cast<const __nv_bfloat16*>(g);
    sp.u = static_cast<const __nv_bfloat16*>(u);
    sp.ldgu = ldgu;
    sp.h = static_cast<__nv_bfloat16*>(h_out);
    sp.ldh = ldh;
    if (dynamic) {
        // pass 1: amax of h (h itself is stored here when asked for)
        NVFP4_CUDA_TRY(cudaMemsetAsync(workspace, 0, sizeof(unsigned int), s));
        if ((st = launch_quant(p, s, kAmaxSiluMul, &sp, static_cast<unsigned int*>(workspace))) != NVFP4_OK)
            return st;
        if (h_out != nullptr) {
            // pass 2 quantises the stored h: silu is evaluated once per element
            p.x = h_out;
            p.ldx = ldh;
            p.in_fp32 = 0;
            if ((st = launch_quant(p, s)) != NVFP4_OK) return st;
            return ok();
        }
    }
    if ((st = launch_quant(p, s, kQuantSiluMul, &sp)) != NVFP4_OK) return st;
    return ok();
}

nvfp4_status nvfp4_quantize_weight(const void* w, nvfp4_in_dtype dt, int64_t n, int64_t k, int64_t ldw,
                                   int64_t row_offset, int64_t n_total, const float* global_scale_in,
                                   uint8_t* w_q, uint8_t* w_sf, float* global_scale_out, void* workspace,
                                   size_t ws_bytes, void* stream)
{
    nvfp4_status st = check_quant_input(w, dt, n, k, ldw, "quantize_weight");
    if (st != NVFP4_OK) return st;
    if (row_offset < 0 || n_total < row_offset + n || n_total >= (1ll << 31))
        return fail(NVFP4_ERR_INVALID_ARG, "quantize_weight: rows [%lld, %lld) do not fit in n_total %lld",
                    (long long)row_offset, (long long)(row_offset + n), (long long)n_total);
    if (n > 0 && (w_q == nullptr || w_sf == nullptr))
        return fail(NVFP4_ERR_INVALID_ARG, "quantize_weight: w_q / w_sf is NULL");
    if (!aligned16(w_q) || !aligned16(w_sf))
        return fail(NVFP4_ERR_ALIGNMENT, "quantize_weight: outputs not 16-byte aligned");
    const bool computed = global_scale_in == nullptr;
    if (computed) {
        if (global_scale_out == nullptr)
            return fail(NVFP4_ERR_INVALID_ARG, "quantize_weight: computed scale needs global_scale_out");
        if (workspace == nullptr || ws_bytes < nvfp4_quant_workspace_size())
            return fail(NVFP4_ERR_WORKSPACE, "quantize_weight: computing the scale needs %zu bytes of workspace",
                        nvfp4_quant_workspace_size());
        if (!aligned16(workspace)) return fail(NVFP4_ERR_ALIGNMENT, "quantize_weight: workspace not 16-byte aligned");
    } else if (!(*global_scale_in > 0.0f) || !std::isfinite(*global_scale_in)) {
        return fail(NVFP4_ERR_INVALID_ARG, "quantize_weight: global scale must be positive and finite");
    }
    const bool owns_tail = row_offset + n == n_total;
    const int64_t sf_rows_end = owns_tail ? pad_to(n_total, 128) - row_offset : n;
    if (sf_rows_end == 0) {
        if (computed) *global_scale_out = 1.0f;
        return ok();
    }
    DeviceState* dev = nullptr;
    if ((st = device_state(&dev)) != NVFP4_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    float* ws_f = static_cast<float*>(workspace);
    if (computed && (st = launch_amax(w, dt, n, k, ldw, workspace, s, dev->sms)) != NVFP4_OK) return st;
    QuantParams p = {};
    p.x = w;
    p.rows = n;
    p.k = k;
    p.ldx = ldw;
    p.in_fp32 = dt == NVFP4_IN_FP32;
    p.q = w_q;
    p.sf = w_sf;
    p.row_offset = row_offset;
    p.sf_rows_end = sf_rows_end;
    if (computed) {
        p.scale_mode = kScaleFromAmax;
        p.scale_ptr = ws_f;
        p.scale_out = ws_f + 1;
    } else {
        p.scale_mode = kScaleValue;
        p.scale_value = *global_scale_in;
    }
    if ((st = launch_quant(p, s)) != NVFP4_OK) return st;
    if (computed) {
        NVFP4_CUDA_TRY(cudaMemcpyAsync(global_scale_out, ws_f + 1, sizeof(float), cudaMemcpyDeviceToHost, s));
        NVFP4_CUDA_TRY(cudaStreamSynchronize(s));
    } else if (global_scale_out != nullptr) {
        *global_scale_out = *global_scale_in;
    }
    return ok();
}

// nvfp4_gemm and nvfp4_gemm_gdn: `gates` (checked by the caller) or NULL.
static nvfp4_status gemm_impl(const uint8_t* a_q, const uint8_t* a_sf, const float* act_scale_dev, const uint8_t* w_q,
                              const uint8_t* w_sf, int64_t m, int64_t n, int64_t k, const nvfp4_segment* segs,
                              int nsegs, void* c, nvfp4_out_dtype odt, int64_t ldc, const nvfp4_gdn_gates* gates,
                              void* workspace, size_t ws_bytes, uint32_t flags, void* stream)
{
    if (m < 0 || n <= 0 || k <= 0 || n % 16 != 0 || k % 32 != 0)
        return fail(NVFP4_ERR_INVALID_ARG, "gemm: need m >= 0, n a positive multiple of 16, k a positive multiple of 32 "
                                           "(m=%lld n=%lld k=%lld)", (long long)m, (long long)n, (long long)k);
    if (m >= (1ll << 31) || n >= (1ll << 31) || k >= (1ll << 31))
        return fail(NVFP4_ERR_UNSUPPORTED, "gemm: dimension >= 2^31");
    if (odt != NVFP4_OUT_BF16 && odt != NVFP4_OUT_FP32) return fail(NVFP4_ERR_INVALID_ARG, "gemm: bad output dtype");
    if (flags > NVFP4_GEMM_FORCE_LARGE_PAIR) return fail(NVFP4_ERR_INVALID_ARG, "gemm: unknown flags 0x%x", flags);
    if (ldc < n) return fail(NVFP4_ERR_INVALID_ARG, "gemm: ldc %lld < n %lld", (long long)ldc, (long long)n);
    SegTable table;
    nvfp4_status st = check_segments(segs, nsegs, n, &table);
    if (st != NVFP4_OK) return st;
    if (m > 0 && (a_q == nullptr || a_sf == nullptr || act_scale_dev == nullptr || w_q == nullptr ||
                  w_sf == nullptr || c == nullptr))
        return fail(NVFP4_ERR_INVALID_ARG, "gemm: NULL operand pointer");
    const int64_t osz = odt == NVFP4_OUT_FP32 ? 4 : 2;
    if (!aligned16(a_q) || !aligned16(a_sf) || !aligned16(w_q) || !aligned16(w_sf) || !aligned16(c) ||
        (ldc * osz) % 16 != 0)
        return fail(NVFP4_ERR_ALIGNMENT, "gemm: operands and output rows must be 16-byte aligned");
    const bool use_decode = flags == NVFP4_GEMM_FORCE_DECODE || (flags == NVFP4_GEMM_AUTO && m <= 64);
    if (use_decode && m > 64) return fail(NVFP4_ERR_UNSUPPORTED, "gemm: the decode kernel handles m <= 64");
    if (m == 0) return ok();
    if (use_decode) {
        if (workspace == nullptr || ws_bytes < decode_ws_bytes(m))
            return fail(NVFP4_ERR_WORKSPACE, "gemm: the decode kernel needs %zu bytes of workspace (got %zu)",
                        decode_ws_bytes(m), ws_bytes);
        if (!aligned16(workspace)) return fail(NVFP4_ERR_ALIGNMENT, "gemm: workspace not 16-byte aligned");
    }

    DeviceState* dev = nullptr;
    if ((st = device_state(&dev)) != NVFP4_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    GemmParams p = {};
    p.m = (int)m;
    p.n = (int)n;
    p.k = (int)k;
    p.a_sf = a_sf;
    p.w_sf = w_sf;
    p.act_scale = act_scale_dev;
    p.c = c;
    p.ldc = ldc;
    p.out_fp32 = odt == NVFP4_OUT_FP32;
    p.segs = table;
    p.katoms = (int)(pad_to(k / 16, 4) / 4);
    p.k_tiles = (int)((k + 255) / 256);
    p.a_rowblocks = (int)((m + 127) / 128);
    p.w_rowblocks = (int)((n + 127) / 128);
    p.splits = 1;
    if (gates != nullptr) {
        p.gdn_heads = gates->heads;
        p.gdn_a_col = gates->a_col;
        p.gdn_b_col = gates->b_col;
        p.gdn_A_log = gates->A_log;
        p.gdn_dt_bias = gates->dt_bias;
        p.gdn_g = gates->g;
        p.gdn_beta = gates->beta;
        p.gdn_ld = gates->ldg;
    }

    const bool use_pair =
        !use_decode && nvfp4_gemm_kernel_for(m, n, dev->sms, flags, gates != nullptr) == (int)NVFP4_GEMM_FORCE_LARGE_PAIR;
    CUtensorMap ta, tw;
    if (!use_decode && !use_pair) {
        p.m_tiles = (int)((m + large::BM - 1) / large::BM);
        p.n_tiles = (int)((n + large::BN - 1) / large::BN);
        if ((st = encode_fp4_map(&ta, a_q, m, k, large::BM)) != NVFP4_OK) return st;
        if ((st = encode_fp4_map(&tw, w_q, n, k, large::BN)) != NVFP4_OK) return st;
        CUtensorMap tc;
        if ((st = encode_c_map(&tc, c, m, n, ldc, p.out_fp32 != 0)) != NVFP4_OK) return st;
        const int64_t tiles = (int64_t)p.m_tiles * p.n_tiles;
        const int grid = (int)(tiles < dev->sms ? tiles : dev->sms);
        if (gates != nullptr) {
            // The gate columns' tiles carry the longest epilogue: schedule them
            // first, on CTAs [extra, ...) which run one tile fewer than CTAs
            // [0, extra), so that the slower epilogue overlaps later MMAs
            // instead of ending the kernel (in column-major order they are
            // the last tiles when the gate ranges close the fused weight).
            const int64_t extra = tiles % grid;
            const int64_t first = (int64_t)((gates->a_col < gates->b_col ? gates->a_col : gates->b_col) / large::BN) *
                                  p.m_tiles;
            p.tile_shift = (int)(((first - extra) % tiles + tiles) % tiles);
        }
        gemm_large_kernel<false><<<grid, large::THREADS, large::SMEM_BYTES, s>>>(ta, tw, tc, p);
        NVFP4_CUDA_TRY(cudaGetLastError());
        return ok();
    }
    if (!use_decode) {
        // NVFP4_GEMM_FORCE_LARGE_PAIR: CTA pairs, 256 x 256 tiles, one pair per two SMs.
        p.m_tiles = (int)((m + 255) / 256);
        p.n_tiles = (int)((n + pairk::BN - 1) / pairk::BN);
        if ((st = encode_fp4_map(&ta, a_q, m, k, pairk::CTA_ROWS)) != NVFP4_OK) return st;
        if ((st = encode_fp4_map(&tw, w_q, n, k, pairk::BN / 2)) != NVFP4_OK) return st;
        CUtensorMap tc;
        if ((st = encode_c_map(&tc, c, m, n, ldc, p.out_fp32 != 0, 32)) != NVFP4_OK) return st;
        const int64_t tiles = (int64_t)p.m_tiles * p.n_tiles;
        const int pairs = (int)(tiles < dev->sms / 2 ? tiles : dev->sms / 2);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
        cfg.blockDim = dim3(pairk::THREADS, 1, 1);
        cfg.dynamicSmemBytes = pairk::SMEM_BYTES;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        NVFP4_CUDA_TRY(cudaLaunchKernelEx(&cfg, gemm_pair_kernel, ta, tw, tc, p));
        return ok();
    }

    const int bt = m <= 16 ? 16 : (m <= 32 ? 32 : 64);
    const int w_tiles = (int)((n + decode::BN - 1) / decode::BN);
    const int64_t units = (int64_t)w_tiles * p.k_tiles;
    if (units >= (1ll << 31)) return fail(NVFP4_ERR_UNSUPPORTED, "gemm: decode problem too large");
    int64_t ctas = dev->sms < decode::MAX_CTAS ? dev->sms : decode::MAX_CTAS;
    if (ctas > units) ctas = units;
    p.units = (int)units;
    p.ctas = (int)ctas;
    p.ws = static_cast<uint8_t*>(workspace);
    p.epoch = next_epoch();
    p.m_tiles = 1;
    p.n_tiles = w_tiles;
    DecodeMaps maps;
    if ((st = encode_decode_maps(&maps, a_q, w_q, m, n, k, bt)) != NVFP4_OK) return st;
    if (bt == 16) st = launch_decode<16, false>(maps, p, s);
    else if (bt == 32) st = launch_decode<32, false>(maps, p, s);
    else st = launch_decode<64, false>(maps, p, s);
    if (st != NVFP4_OK) return st;
    return ok();
}

nvfp4_status nvfp4_gemm(const uint8_t* a_q, const uint8_t* a_sf, const float* act_scale_dev, const uint8_t* w_q,
                        const uint8_t* w_sf, int64_t m, int64_t n, int64_t k, const nvfp4_segment* segs, int nsegs,
                        void* c, nvfp4_out_dtype odt, int64_t ldc, void* workspace, size_t ws_bytes, uint32_t flags,
                        void* stream)
{
    return gemm_impl(a_q, a_sf, act_scale_dev, w_q, w_sf, m, n, k, segs, nsegs, c, odt, ldc, nullptr, workspace,
                     ws_bytes, flags, stream);
}

nvfp4_status nvfp4_gemm_gdn(const uint8_t* a_q, const uint8_t* a_sf, const float* act_scale_dev, const uint8_t* w_q,
                            const uint8_t* w_sf, int64_t m, int64_t n, int64_t k, const nvfp4_segment* segs,
                            int nsegs, void* c, int64_t ldc, const nvfp4_gdn_gates* gates, void* workspace,
                            size_t ws_bytes, uint32_t flags, void* stream)
{
    if (gates == nullptr) return fail(NVFP4_ERR_INVALID_ARG, "gemm_gdn: NULL gates");
    const int64_t heads = gates->heads;
    if (heads < 1 || gates->a_col < 0 || gates->b_col < 0 || gates->a_col + heads > n || gates->b_col + heads > n)
        return fail(NVFP4_ERR_INVALID_ARG, "gemm_gdn: gate columns [%d, +%d) and [%d, +%d) must lie in [0, n=%lld)",
                    gates->a_col, gates->heads, gates->b_col, gates->heads, (long long)n);
    if (gates->ldg < heads)
        return fail(NVFP4_ERR_INVALID_ARG, "gemm_gdn: ldg %lld < heads %d", (long long)gates->ldg, gates->heads);
    if (m > 0 && (gates->A_log == nullptr || gates->dt_bias == nullptr || gates->g == nullptr ||
                  gates->beta == nullptr))
        return fail(NVFP4_ERR_INVALID_ARG, "gemm_gdn: NULL gate pointer");
    if (reinterpret_cast<uintptr_t>(gates->A_log) % 4 || reinterpret_cast<uintptr_t>(gates->dt_bias) % 4 ||
        reinterpret_cast<uintptr_t>(gates->g) % 4 || reinterpret_cast<uintptr_t>(gates->beta) % 4)
        return fail(NVFP4_ERR_ALIGNMENT, "gemm_gdn: gate vectors must be 4-byte aligned");
    if (m > 0 && m * gates->ldg >= (1ll << 40))
        return fail(NVFP4_ERR_UNSUPPORTED, "gemm_gdn: gate outputs too large");
    return gemm_impl(a_q, a_sf, act_scale_dev, w_q, w_sf, m, n, k, segs, nsegs, c, NVFP4_OUT_BF16, ldc, gates,
                     workspace, ws_bytes, flags, stream);
}

nvfp4_status nvfp4_gemm_swiglu_quantize(const uint8_t* a_q, const uint8_t* a_sf, const float* act_scale_dev,
                                        const uint8_t* w_q, const uint8_t* w_sf, int64_t m, int64_t f, int64_t k,
                                        const nvfp4_segment* segs, int nsegs, const float* h_scale_dev,
                                        uint8_t* h_q, uint8_t* h_sf, void* stream)
{
    if (m < 0 || f <= 0 || f % 128 != 0 || k <= 0 || k % 32 != 0)
        return fail(NVFP4_ERR_INVALID_ARG, "gemm_swiglu_quantize: need m >= 0, f a positive multiple of 128 and k a "
                                           "positive multiple of 32 (m=%lld f=%lld k=%lld)",
                    (long long)m, (long long)f, (long long)k);
    if (m >= (1ll << 31) || 2 * f >= (1ll << 31) || k >= (1ll << 31))
        return fail(NVFP4_ERR_UNSUPPORTED, "gemm_swiglu_quantize: dimension >= 2^31");
    SegTable table;
    nvfp4_status st = check_segments(segs, nsegs, 2 * f, &table);
    if (st != NVFP4_OK) return st;
    if (m > 0 && (a_q == nullptr || a_sf == nullptr || act_scale_dev == nullptr || w_q == nullptr ||
                  w_sf == nullptr || h_scale_dev == nullptr || h_q == nullptr || h_sf == nullptr))
        return fail(NVFP4_ERR_INVALID_ARG, "gemm_swiglu_quantize: NULL pointer");
    if (!aligned16(a_q) || !aligned16(a_sf) || !aligned16(w_q) || !aligned16(w_sf) || !aligned16(h_q) ||
        !aligned16(h_sf))
        return fail(NVFP4_ERR_ALIGNMENT, "gemm_swiglu_quantize: operands and outputs must be 16-byte aligned");
    if (m == 0) return ok();
    DeviceState* dev = nullptr;
    if ((st = device_state(&dev)) != NVFP4_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    GemmParams p = {};
    p.m = (int)m;
    p.n = (int)(2 * f);
    p.k = (int)k;
    p.a_sf = a_sf;
    p.w_sf = w_sf;
    p.act_scale = act_scale_dev;
    p.segs = table;
    p.katoms = (int)(pad_to(k / 16, 4) / 4);
    p.k_tiles = (int)((k + 255) / 256);
    p.a_rowblocks = (int)((m + 127) / 128);
    p.w_rowblocks = (int)((2 * f + 127) / 128);
    p.splits = 1;
    p.swiglu_f = (int)f;
    p.h_scale = h_scale_dev;
    p.h_q = h_q;
    p.h_sf = h_sf;
    p.m_tiles = (int)((m + large::BM - 1) / large::BM);
    p.n_tiles = (int)(f / 128);
    CUtensorMap ta, tw;
    if ((st = encode_fp4_map(&ta, a_q, m, k, large::BM)) != NVFP4_OK) return st;
    if ((st = encode_fp4_map(&tw, w_q, 2 * f, k, 128)) != NVFP4_OK) return st;
    const int64_t tiles = (int64_t)p.m_tiles * p.n_tiles;
    const int grid = (int)(tiles < dev->sms ? tiles : dev->sms);
    // no C is written: the C map argument is not read
    gemm_large_kernel<true><<<grid, large::THREADS, large::SMEM_BYTES, s>>>(ta, tw, tw, p);
    NVFP4_CUDA_TRY(cudaGetLastError());
    return ok();
}

nvfp4_status nvfp4_linear_decode(const void* a, nvfp4_in_dtype dt, int64_t m, int64_t k, int64_t lda,
                                 const float* act_scale_dev, float* act_scale_out_dev, const uint8_t* w_q,
                                 const uint8_t* w_sf, int64_t n, const nvfp4_segment* segs, int nsegs, void* c,
                                 nvfp4_out_dtype odt, int64_t ldc, void* workspace, size_t ws_bytes, void* stream)
{
    nvfp4_status st = check_quant_input(a, dt, m, k, lda, "linear_decode");
    if (st != NVFP4_OK) return st;
    if (m > 64) return fail(NVFP4_ERR_UNSUPPORTED, "linear_decode: m = %lld > 64 (use nvfp4_quantize_act + nvfp4_gemm)",
                            (long long)m);
    if (n <= 0 || n % 16 != 0)
        return fail(NVFP4_ERR_INVALID_ARG, "linear_decode: n must be a positive multiple of 16 (n=%lld)", (long long)n);
    if (n >= (1ll << 31)) return fail(NVFP4_ERR_UNSUPPORTED, "linear_decode: dimension >= 2^31");
    if (odt != NVFP4_OUT_BF16 && odt != NVFP4_OUT_FP32)
        return fail(NVFP4_ERR_INVALID_ARG, "linear_decode: bad output dtype");
    if (ldc < n) return fail(NVFP4_ERR_INVALID_ARG, "linear_decode: ldc %lld < n %lld", (long long)ldc, (long long)n);
    SegTable table;
    if ((st = check_segments(segs, nsegs, n, &table)) != NVFP4_OK) return st;
    if (m > 0 && (w_q == nullptr || w_sf == nullptr || c == nullptr))
        return fail(NVFP4_ERR_INVALID_ARG, "linear_decode: NULL weight or output pointer");
    const int64_t osz = odt == NVFP4_OUT_FP32 ? 4 : 2;
    if (!aligned16(w_q) || !aligned16(w_sf) || !aligned16(c) || (ldc * osz) % 16 != 0)
        return fail(NVFP4_ERR_ALIGNMENT, "linear_decode: weights and output rows must be 16-byte aligned");
    if (workspace == nullptr || ws_bytes < decode_ws_bytes(m < 1 ? 1 : m))
        return fail(NVFP4_ERR_WORKSPACE, "linear_decode: needs %zu bytes of workspace (got %zu)",
                    decode_ws_bytes(m < 1 ? 1 : m), ws_bytes);
    if (!aligned16(workspace)) return fail(NVFP4_ERR_ALIGNMENT, "linear_decode: workspace not 16-byte aligned");
    if (m == 0) return ok();

    DeviceState* dev = nullptr;
    if ((st = device_state(&dev)) != NVFP4_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    GemmParams p = {};
    p.m = (int)m;
    p.n = (int)n;
    p.k = (int)k;
    p.w_sf = w_sf;
    p.act_scale = act_scale_dev;
    p.c = c;
    p.ldc = ldc;
    p.out_fp32 = odt == NVFP4_OUT_FP32;
    p.segs = table;
    p.katoms = (int)(pad_to(k / 16, 4) / 4);
    p.k_tiles = (int)((k + 255) / 256);
    p.a_rowblocks = 1;
    p.w_rowblocks = (int)((n + 127) / 128);
    p.splits = 1;
    p.a_in = a;
    p.lda = lda;
    p.a_fp32 = dt == NVFP4_IN_FP32;
    p.act_scale_out = act_scale_out_dev;
    const int bt = m <= 16 ? 16 : (m <= 32 ? 32 : 64);
    const int w_tiles = (int)((n + decode::BN - 1) / decode::BN);
    const int64_t units = (int64_t)w_tiles * p.k_tiles;
    if (units >= (1ll << 31)) return fail(NVFP4_ERR_UNSUPPORTED, "linear_decode: problem too large");
    int64_t ctas = dev->sms < decode::MAX_CTAS ? dev->sms : decode::MAX_CTAS;
    if (ctas > units) ctas = units;
    p.units = (int)units;
    p.ctas = (int)ctas;
    p.ws = static_cast<uint8_t*>(workspace);
    p.epoch = next_epoch();
    p.m_tiles = 1;
    p.n_tiles = w_tiles;
    DecodeMaps maps;   // the A maps are not read when the quantisation is fused in
    if ((st = encode_decode_maps(&maps, nullptr, w_q, m, n, k, bt)) != NVFP4_OK) return st;
    if (bt == 16) st = launch_decode<16, true>(maps, p, s);
    else if (bt == 32) st = launch_decode<32, true>(maps, p, s);
    else st = launch_decode<64, true>(maps, p, s);
    if (st != NVFP4_OK) return st;
    return ok();
}

size_t nvfp4_linear_prefill_workspace_size(int64_t m)
{
    if (m < 0) return 0;
    return (size_t)pad_to((m + 127) / 128 * 8, 16);
}

nvfp4_status nvfp4_linear_prefill(const void* a, nvfp4_in_dtype dt, int64_t m, int64_t k, int64_t lda,
                                  const float* act_scale_dev, uint8_t* a_q, uint8_t* a_sf, const uint8_t* w_q,
                                  const uint8_t* w_sf, int64_t n, const nvfp4_segment* segs, int nsegs, void* c,
                                  nvfp4_out_dtype odt, int64_t ldc, void* workspace, size_t ws_bytes, void* stream)
{
    nvfp4_status st = check_quant_input(a, dt, m, k, lda, "linear_prefill");
    if (st != NVFP4_OK) return st;
    if (dt != NVFP4_IN_BF16)
        return fail(NVFP4_ERR_UNSUPPORTED, "linear_prefill: BF16 activations only (use nvfp4_quantize_act + nvfp4_gemm)");
    if (m > 0 && m <= 64)
        return fail(NVFP4_ERR_UNSUPPORTED, "linear_prefill: m = %lld <= 64 (use nvfp4_linear_decode)", (long long)m);
    if (act_scale_dev == nullptr)
        return fail(NVFP4_ERR_INVALID_ARG, "linear_prefill: needs the static activation scale act_scale_dev");
    if (n <= 0 || n % 16 != 0)
        return fail(NVFP4_ERR_INVALID_ARG, "linear_prefill: n must be a positive multiple of 16 (n=%lld)", (long long)n);
    if (n >= (1ll << 31)) return fail(NVFP4_ERR_UNSUPPORTED, "linear_prefill: dimension >= 2^31");
    if (odt != NVFP4_OUT_BF16 && odt != NVFP4_OUT_FP32)
        return fail(NVFP4_ERR_INVALID_ARG, "linear_prefill: bad output dtype");
    if (ldc < n) return fail(NVFP4_ERR_INVALID_ARG, "linear_prefill: ldc %lld < n %lld", (long long)ldc, (long long)n);
    SegTable table;
    if ((st = check_segments(segs, nsegs, n, &table)) != NVFP4_OK) return st;
    if (m > 0 && (a_q == nullptr || a_sf == nullptr || w_q == nullptr || w_sf == nullptr || c == nullptr))
        return fail(NVFP4_ERR_INVALID_ARG, "linear_prefill: NULL pointer");
    const int64_t osz = odt == NVFP4_OUT_FP32 ? 4 : 2;
    if (!aligned16(a_q) || !aligned16(a_sf) || !aligned16(w_q) || !aligned16(w_sf) || !aligned16(c) ||
        (ldc * osz) % 16 != 0)
        return fail(NVFP4_ERR_ALIGNMENT, "linear_prefill: buffers and output rows must be 16-byte aligned");
    if (workspace == nullptr || ws_bytes < nvfp4_linear_prefill_workspace_size(m))
        return fail(NVFP4_ERR_WORKSPACE, "linear_prefill: needs %zu bytes of workspace (got %zu)",
                    nvfp4_linear_prefill_workspace_size(m), ws_bytes);
    if (!aligned16(workspace)) return fail(NVFP4_ERR_ALIGNMENT, "linear_prefill: workspace not 16-byte aligned");
    if (m == 0) return ok();

    DeviceState* dev = nullptr;
    if ((st = device_state(&dev)) != NVFP4_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    GemmParams p = {};
    p.m = (int)m;
    p.n = (int)n;
    p.k = (int)k;
    p.a_sf = a_sf;
    p.w_sf = w_sf;
    p.act_scale = act_scale_dev;
    p.c = c;
    p.ldc = ldc;
    p.out_fp32 = odt == NVFP4_OUT_FP32;
    p.segs = table;
    p.katoms = (int)(pad_to(k / 16, 4) / 4);
    p.k_tiles = (int)((k + 255) / 256);
    p.a_rowblocks = (int)((m + 127) / 128);
    p.w_rowblocks = (int)((n + 127) / 128);
    p.splits = 1;
    p.a_in = a;
    p.lda = lda;
    p.qa_q = a_q;
    p.qa_sf = a_sf;
    p.qa_ready = static_cast<unsigned long long*>(workspace);
    p.epoch = next_prefill_tag();
    p.m_tiles = (int)((m + large::BM - 1) / large::BM);
    p.n_tiles = (int)((n + large::BN - 1) / large::BN);
    const int64_t tiles = (int64_t)p.m_tiles * p.n_tiles;
    const int grid = (int)(tiles < dev->sms ? tiles : dev->sms);
    // m-blocks quantised before the mainloop: those the first two waves of
    // tiles read (band b of the tile order holds m-blocks [BAND b, BAND b +
    // BAND), column-major inside the band)
    {
        const int64_t last = std::min<int64_t>(tiles, 2 * (int64_t)grid) - 1;
        const int64_t band_tiles = (int64_t)qa::BAND * p.n_tiles;
        const int64_t band = last / band_tiles;
        const int64_t r = last - band * band_tiles;
        const int64_t bsz = std::min<int64_t>(qa::BAND, p.m_tiles - band * qa::BAND);
        p.qa_first = (int)(band * qa::BAND + std::min<int64_t>(r + 1, bsz));
    }
    CUtensorMap ta, tw, tc;
    if ((st = encode_fp4_map(&ta, a_q, m, k, large::BM)) != NVFP4_OK) return st;
    if ((st = encode_fp4_map(&tw, w_q, n, k, large::BN)) != NVFP4_OK) return st;
    if ((st = encode_c_map(&tc, c, m, n, ldc, p.out_fp32 != 0)) != NVFP4_OK) return st;
    gemm_large_kernel<false, true><<<grid, large::THREADS, large::SMEM_BYTES, s>>>(ta, tw, tc, p);
    NVFP4_CUDA_TRY(cudaGetLastError());
    return ok();
}

nvfp4_status nvfp4_gemm_decode_noalloc(const uint8_t* a_q, const uint8_t* a_sf, const float* act_scale_dev,
                                       const uint8_t* w_q, const uint8_t* w_sf, int64_t m, int64_t n, int64_t k,
                                       const nvfp4_segment* segs, int nsegs, void* c, nvfp4_out_dtype odt,
                                       int64_t ldc, void* stream)
{
    if (m < 0) return fail(NVFP4_ERR_INVALID_ARG, "gemm_decode_noalloc: m = %lld < 0", (long long)m);
    if (m > NVFP4_NOALLOC_MAX_M)
        return fail(NVFP4_ERR_UNSUPPORTED,
                    "gemm_decode_noalloc: m = %lld needs %zu bytes of decode scratch, but the built-in array holds "
                    "%zu (m <= %d); call nvfp4_gemm with a workspace instead",
                    (long long)m, decode_ws_bytes(m), (size_t)NVFP4_NOALLOC_SCRATCH_BYTES, NVFP4_NOALLOC_MAX_M);
    void* scratch = nullptr;
    if (m > 0) {
        DeviceState* dev = nullptr;
        nvfp4_status st = device_state(&dev);
        if (st != NVFP4_OK) return st;
        if ((st = noalloc_scratch(&scratch)) != NVFP4_OK) return st;
    }
    return nvfp4_gemm(a_q, a_sf, act_scale_dev, w_q, w_sf, m, n, k, segs, nsegs, c, odt, ldc, scratch,
                      NVFP4_NOALLOC_SCRATCH_BYTES, NVFP4_GEMM_FORCE_DECODE, stream);
}

nvfp4_status nvfp4_check_device_status(void* stream)
{
    NVFP4_CUDA_TRY(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
    unsigned int v = 0;
    NVFP4_CUDA_TRY(cudaMemcpyFromSymbol(&v, g_device_status, sizeof v));
    if (v != 0) {
        const unsigned int zero = 0;
        NVFP4_CUDA_TRY(cudaMemcpyToSymbol(g_device_status, &zero, sizeof zero));
        return fail(NVFP4_ERR_TIMEOUT, "a bounded wait inside a kernel ran out (status 0x%x)", v);
    }
    return ok();
}

nvfp4_status nvfp4_selftest_wait_timeout(long long limit_cycles, void* stream)
{
    if (limit_cycles <= 0 || limit_cycles > kWaitCycles)
        return fail(NVFP4_ERR_INVALID_ARG, "selftest: limit must be in (0, %lld] cycles", kWaitCycles);
    selftest_wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_cycles);
    NVFP4_CUDA_TRY(cudaGetLastError());
    return ok();
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Calibrated FP8 KV cache
// ---------------------------------------------------------------------------
nvfp4_status nvfp4_fp8_calibrate(const void* x, nvfp4_in_dtype dt, int64_t rows, int64_t width, int64_t ld,
                                 float* amax_inout_dev, float* scale_out_dev, void* stream)
{
    if (dt != NVFP4_IN_BF16 && dt != NVFP4_IN_FP32) return fail(NVFP4_ERR_INVALID_ARG, "fp8_calibrate: bad input dtype");
    if (rows < 0 || width <= 0 || width % 16 != 0)
        return fail(NVFP4_ERR_INVALID_ARG, "fp8_calibrate: need rows >= 0 and width a positive multiple of 16 "
                                           "(rows=%lld width=%lld)", (long long)rows, (long long)width);
    if (rows >= (1ll << 31) || width >= (1ll << 31)) return fail(NVFP4_ERR_UNSUPPORTED, "fp8_calibrate: dimension >= 2^31");
    if (ld < width) return fail(NVFP4_ERR_INVALID_ARG, "fp8_calibrate: ld %lld < width %lld", (long long)ld,
                                (long long)width);
    if (amax_inout_dev == nullptr || scale_out_dev == nullptr || (rows > 0 && x == nullptr))
        return fail(NVFP4_ERR_INVALID_ARG, "fp8_calibrate: NULL pointer");
    const int64_t esz = dt == NVFP4_IN_FP32 ? 4 : 2;
    if (!aligned16(x) || (ld * esz) % 16 != 0 || reinterpret_cast<uintptr_t>(amax_inout_dev) % 4 ||
        reinterpret_cast<uintptr_t>(scale_out_dev) % 4)
        return fail(NVFP4_ERR_ALIGNMENT, "fp8_calibrate: rows must start on 16-byte boundaries");
    DeviceState* dev = nullptr;
    nvfp4_status st = device_state(&dev);
    if (st != NVFP4_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((st = launch_amax_into(x, dt, rows, width, ld, reinterpret_cast<unsigned int*>(amax_inout_dev), s, dev->sms)) !=
        NVFP4_OK)
        return st;
    fp8_scale_kernel<<<1, 32, 0, s>>>(amax_inout_dev, scale_out_dev);
    NVFP4_CUDA_TRY(cudaGetLastError());
    return ok();
}

nvfp4_status nvfp4_kv_cache_quantize_fp8(const void* k, const void* v, nvfp4_in_dtype dt, int64_t tokens,
                                         int64_t width, int64_t ld_k, int64_t ld_v, const int64_t* slot_mapping,
                                         int64_t num_slots, const float* k_scale_dev, const float* v_scale_dev,
                                         uint8_t* k_cache, uint8_t* v_cache, int64_t cache_ld, void* stream)
{
    if (dt != NVFP4_IN_BF16 && dt != NVFP4_IN_FP32)
        return fail(NVFP4_ERR_INVALID_ARG, "kv_cache_quantize_fp8: bad input dtype");
    if (tokens < 0 || width <= 0 || width % 16 != 0 || num_slots < 0)
        return fail(NVFP4_ERR_INVALID_ARG, "kv_cache_quantize_fp8: need tokens >= 0, width a positive multiple of 16 "
                                           "and num_slots >= 0 (tokens=%lld width=%lld num_slots=%lld)",
                    (long long)tokens, (long long)width, (long long)num_slots);
    if (tokens * (width / 16) >= (1ll << 31))
        return fail(NVFP4_ERR_UNSUPPORTED, "kv_cache_quantize_fp8: tokens x width / 16 >= 2^31");
    if (ld_k < width || ld_v < width || cache_ld < width)
        return fail(NVFP4_ERR_INVALID_ARG, "kv_cache_quantize_fp8: ld_k, ld_v and cache_ld must be >= width");
    if (slot_mapping == nullptr && tokens > num_slots)
        return fail(NVFP4_ERR_INVALID_ARG, "kv_cache_quantize_fp8: without a slot table token t goes to slot t, so "
                                           "tokens (%lld) must not exceed num_slots (%lld)",
                    (long long)tokens, (long long)num_slots);
    if (tokens == 0) return ok();
    if (k == nullptr || v == nullptr || k_scale_dev == nullptr || v_scale_dev == nullptr || k_cache == nullptr ||
        v_cache == nullptr)
        return fail(NVFP4_ERR_INVALID_ARG, "kv_cache_quantize_fp8: NULL pointer");
    const int64_t esz = dt == NVFP4_IN_FP32 ? 4 : 2;
    if (!aligned16(k) || !aligned16(v) || (ld_k * esz) % 16 != 0 || (ld_v * esz) % 16 != 0 || !aligned16(k_cache) ||
        !aligned16(v_cache) || cache_ld % 16 != 0 || reinterpret_cast<uintptr_t>(slot_mapping) % 8 ||
        reinterpret_cast<uintptr_t>(k_scale_dev) % 4 || reinterpret_cast<uintptr_t>(v_scale_dev) % 4)
        return fail(NVFP4_ERR_ALIGNMENT, "kv_cache_quantize_fp8: rows must start on 16-byte boundaries");
    DeviceState* dev = nullptr;
    nvfp4_status st = device_state(&dev);
    if (st != NVFP4_OK) return st;
    KvParams p = {};
    p.x[0] = k;
    p.x[1] = v;
    p.ld[0] = ld_k;
    p.ld[1] = ld_v;
    p.in_fp32 = dt == NVFP4_IN_FP32;
    p.tokens = (uint32_t)tokens;
    p.chunks = (uint32_t)(width / 16);
    p.units = (uint32_t)(tokens * (width / 16));
    p.slots = slot_mapping;
    p.num_slots = num_slots;
    p.scale[0] = k_scale_dev;
    p.scale[1] = v_scale_dev;
    p.cache[0] = k_cache;
    p.cache[1] = v_cache;
    p.cache_ld = cache_ld;
    const int64_t total = 2 * (int64_t)p.units;
    int64_t blocks = (total + kKvThreads - 1) / kKvThreads;
    if (blocks > (int64_t)dev->sms * 16) blocks = (int64_t)dev->sms * 16;
    if (p.in_fp32)
        kv_fp8_quantize_kernel<true><<<(unsigned)blocks, kKvThreads, 0, static_cast<cudaStream_t>(stream)>>>(p);
    else
        kv_fp8_quantize_kernel<false><<<(unsigned)blocks, kKvThreads, 0, static_cast<cudaStream_t>(stream)>>>(p);
    NVFP4_CUDA_TRY(cudaGetLastError());
    return ok();
}
