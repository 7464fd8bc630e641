// libnvfp4_probes: two measurement kernels that give the roofline
// denominators of the linear-layer kernels on the machine at hand.  They are
// not part of the linear-layer path and libnvfp4 does not contain them.
//
//  * mma_peak_kernel: the dense block-scaled FP4 tensor-core rate with both
//    operands resident in shared memory and the scales in TMEM, i.e. the
//    mainloop of gemm_large_kernel without TMA, epilogue or scale staging:
//    one elected thread per CTA issues back-to-back
//    tcgen05.mma.cta_group::1.kind::mxf4nvf4 (M = 128, N = 256, K = 64).
//  * hbm_read_kernel: read-only streaming of a buffer much larger than L2
//    (16-byte loads, four in flight per thread), the bound of a read-mostly
//    kernel such as the decode GEMM.
#include <cuda.h>
#include <cuda_runtime.h>

#include "ptx.cuh"

#define NVFP4_PROBE_API extern "C" __attribute__((visibility("default")))

namespace nvfp4 {
namespace probe {

constexpr int MMA_THREADS = 128;
constexpr int A_BYTES = 128 * 128;       // 128 rows x 256 FP4 values
constexpr int B_BYTES = 256 * 128;       // 256 rows x 256 FP4 values
constexpr int SMEM_BYTES = A_BYTES + B_BYTES + 64 + 1024;
constexpr int TMEM_COLS = 512;
constexpr int SF_COL = 256;              // 16 columns of A scales + 32 of B scales

__global__ void __launch_bounds__(MMA_THREADS, 1) mma_peak_kernel(int iters, unsigned long long* cycles)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* a = smem;
    uint8_t* b = smem + A_BYTES;
    uint64_t* done = reinterpret_cast<uint64_t*>(smem + A_BYTES + B_BYTES);
    uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(done + 1);
    const int warp = threadIdx.x >> 5;

    // Operands: a fixed mix of codes (the values do not matter for the rate).
    for (int i = threadIdx.x; i < (A_BYTES + B_BYTES) / 4; i += MMA_THREADS)
        reinterpret_cast<uint32_t*>(a)[i] = 0x3A5C1E97u ^ ((uint32_t)i * 2654435761u);
    if (threadIdx.x == 0) {
        mbar_init(done, 1);
        fence_mbarrier_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_ptr, TMEM_COLS);
        tmem_relinquish();
    }
    fence_proxy_async_shared();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_ptr;

    // Scales 1.0 (UE4M3 0x38) in every scale column of every lane.
    uint32_t ones[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) ones[j] = 0x38383838u;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    tmem_st_32x32b_x16(tbase + lane_base + SF_COL, ones);
    tmem_st_32x32b_x16(tbase + lane_base + SF_COL + 16, ones);
    tmem_st_32x32b_x16(tbase + lane_base + SF_COL + 32, ones);
    tmem_st_wait();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (threadIdx.x == 0) {
        const uint32_t idesc = idesc_nvf4(128, 256);
        const uint64_t ad = desc_kmajor_sw128(a), bd = desc_kmajor_sw128(b);
        const long long t0 = clock64();
        for (int i = 0; i < iters; ++i) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_nvf4(tbase, ad + 2 * ks, bd + 2 * ks, idesc, (i | ks) != 0, tbase + SF_COL + 4 * ks,
                         tbase + SF_COL + 16 + 8 * ks);
        }
        mma_commit(done);
        mbar_wait(done, 0, kStatusTimeoutAccum);
        const long long t1 = clock64();
        if (blockIdx.x == 0 && cycles != nullptr) *cycles = (unsigned long long)(t1 - t0);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tbase, TMEM_COLS);
    }
}

// The same on CTA pairs: clusters of two CTAs, the even one issuing
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 64), each CTA holding its
// half of A and B in shared memory and its scales in TMEM.
__global__ void __launch_bounds__(MMA_THREADS, 1) mma_peak_pair_kernel(int iters, unsigned long long* cycles)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* a = smem;                       // 128 rows
    uint8_t* b = smem + A_BYTES;             // 128 of the 256 B rows
    uint64_t* done = reinterpret_cast<uint64_t*>(smem + A_BYTES + B_BYTES);
    uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(done + 1);
    const int warp = threadIdx.x >> 5;
    const uint32_t rank = cluster_ctarank();

    for (int i = threadIdx.x; i < (A_BYTES + A_BYTES) / 4; i += MMA_THREADS)
        reinterpret_cast<uint32_t*>(a)[i] = 0x3A5C1E97u ^ ((uint32_t)i * 2654435761u) ^ rank;
    if (threadIdx.x == 0) {
        mbar_init(done, 1);
        fence_mbarrier_init();
    }
    if (warp == 0) {
        tmem_alloc_pair(tmem_ptr, TMEM_COLS);
        tmem_relinquish_pair();
    }
    fence_proxy_async_shared();
    tc_fence_before();
    cluster_arrive_release();
    cluster_wait_acquire();
    tc_fence_after();
    const uint32_t tbase = *tmem_ptr;
    uint32_t ones[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) ones[j] = 0x38383838u;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    tmem_st_32x32b_x16(tbase + lane_base + SF_COL, ones);
    tmem_st_32x32b_x16(tbase + lane_base + SF_COL + 16, ones);
    tmem_st_32x32b_x16(tbase + lane_base + SF_COL + 32, ones);
    tmem_st_wait();
    tc_fence_before();
    cluster_arrive_release();
    cluster_wait_acquire();
    tc_fence_after();

    if (threadIdx.x == 0 && rank == 0) {
        const uint32_t idesc = idesc_nvf4(256, 256);
        const uint64_t ad = desc_kmajor_sw128(a), bd = desc_kmajor_sw128(b);
        const long long t0 = clock64();
        for (int i = 0; i < iters; ++i) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_nvf4_pair(tbase, ad + 2 * ks, bd + 2 * ks, idesc, (i | ks) != 0, tbase + SF_COL + 4 * ks,
                              tbase + SF_COL + 16 + 8 * ks);
        }
        mma_commit_pair(done, 0x1);
        mbar_wait(done, 0, kStatusTimeoutAccum);
        const long long t1 = clock64();
        if (blockIdx.x == 0 && cycles != nullptr) *cycles = (unsigned long long)(t1 - t0);
    }
    tc_fence_before();
    cluster_arrive_release();
    cluster_wait_acquire();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc_pair(tbase, TMEM_COLS);
    }
}

__global__ void __launch_bounds__(256) hbm_read_kernel(const uint4* __restrict__ src, int64_t n16,
                                                       unsigned int* __restrict__ sink)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    uint32_t acc = 0;
    for (; i + 3 * stride < n16; i += 4 * stride) {
        const uint4 v0 = ldg_nc_v4(src + i);
        const uint4 v1 = ldg_nc_v4(src + i + stride);
        const uint4 v2 = ldg_nc_v4(src + i + 2 * stride);
        const uint4 v3 = ldg_nc_v4(src + i + 3 * stride);
        acc ^= v0.x ^ v0.y ^ v0.z ^ v0.w ^ v1.x ^ v1.y ^ v1.z ^ v1.w;
        acc ^= v2.x ^ v2.y ^ v2.z ^ v2.w ^ v3.x ^ v3.y ^ v3.z ^ v3.w;
    }
    for (; i < n16; i += stride) {
        const uint4 v = ldg_nc_v4(src + i);
        acc ^= v.x ^ v.y ^ v.z ^ v.w;
    }
    if (acc == 0x9E3779B9u) *sink = acc;   // keeps the loads; practically never taken
}

}  // namespace probe
}  // namespace nvfp4

using namespace nvfp4;

// Launch `ctas` CTAs (one per SM at most), each issuing iters x 4 MMAs of
// 2 * 128 * 256 * 64 FLOP.  `cycles` (device, may be NULL) receives CTA 0's
// SM-clock cycles from the first issue to the completion of the last MMA.
// Returns a cudaError_t value (0 on success).
NVFP4_PROBE_API int nvfp4_probe_mma_peak(int iters, int ctas, unsigned long long* cycles, void* stream)
{
    if (iters <= 0 || ctas <= 0 || iters > (1 << 22)) return (int)cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(probe::mma_peak_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         probe::SMEM_BYTES);
    if (e != cudaSuccess) return (int)e;
    probe::mma_peak_kernel<<<ctas, probe::MMA_THREADS, probe::SMEM_BYTES, static_cast<cudaStream_t>(stream)>>>(
        iters, cycles);
    return (int)cudaGetLastError();
}

// The pair form: `ctas` (even) CTAs in clusters of two, each pair issuing
// iters x 4 MMAs of 2 * 256 * 256 * 64 FLOP.
NVFP4_PROBE_API int nvfp4_probe_mma_peak_pair(int iters, int ctas, unsigned long long* cycles, void* stream)
{
    if (iters <= 0 || ctas <= 0 || ctas % 2 != 0 || iters > (1 << 22)) return (int)cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(probe::mma_peak_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         probe::SMEM_BYTES);
    if (e != cudaSuccess) return (int)e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)ctas, 1, 1);
    cfg.blockDim = dim3(probe::MMA_THREADS, 1, 1);
    cfg.dynamicSmemBytes = probe::SMEM_BYTES;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, probe::mma_peak_pair_kernel, iters, cycles);
    if (e != cudaSuccess) return (int)e;
    return (int)cudaGetLastError();
}

// Stream `bytes` (a multiple of 16, 16-byte aligned) from `src` once.
NVFP4_PROBE_API int nvfp4_probe_hbm_read(const void* src, long long bytes, unsigned int* sink, int blocks,
                                         void* stream)
{
    if (src == nullptr || sink == nullptr || bytes <= 0 || bytes % 16 != 0 || blocks <= 0 ||
        (reinterpret_cast<uintptr_t>(src) & 15u) != 0)
        return (int)cudaErrorInvalidValue;
    probe::hbm_read_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<const uint4*>(src),
                                                                                  bytes / 16, sink);
    return (int)cudaGetLastError();
}

// Reads and clears the bounded-wait status word of this library (non-zero:
// the probe's completion wait ran out and its timing is void).
NVFP4_PROBE_API int nvfp4_probe_status(unsigned int* out)
{
    cudaError_t e = cudaMemcpyFromSymbol(out, g_device_status, sizeof(unsigned int));
    if (e != cudaSuccess) return (int)e;
    const unsigned int zero = 0;
    return (int)cudaMemcpyToSymbol(g_device_status, &zero, sizeof zero);
}
