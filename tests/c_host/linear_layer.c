/* A C program on the library's C boundary (include/nvfp4.h): one W4A4 linear
 * layer, C = A W^T, with the three calls a user makes - nvfp4_quantize_weight
 * (offline, computed global scale), nvfp4_quantize_act (dynamic scale) and
 * nvfp4_gemm (FP32 and BF16 output, one segment) - plus the boundary's error
 * behaviour on a few invalid calls.  Device memory and the stream come from
 * the CUDA driver API, so nothing here shares state with the library except
 * the device's primary context.
 *
 * usage: linear_layer DIR M N K
 *   reads   DIR/a.bf16 (M x K BF16, row-major), DIR/w.bf16 (N x K BF16)
 *   writes  DIR/a_q.bin, a_sf.bin, w_q.bin, w_sf.bin (the library's buffers),
 *           DIR/scales.bin (s_ga, s_gw as two FP32), DIR/c32.bin (M x N FP32),
 *           DIR/c16.bin (M x N BF16)
 * Exit status 0 on success; otherwise the failing call is printed. */
#include <cuda.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "nvfp4.h"

#define CHECK_CU(expr)                                                             \
    do {                                                                           \
        CUresult r_ = (expr);                                                      \
        if (r_ != CUDA_SUCCESS) {                                                  \
            fprintf(stderr, "%s failed: CUresult %d\n", #expr, (int)r_);           \
            return 2;                                                              \
        }                                                                          \
    } while (0)

#define CHECK_NV(expr)                                                             \
    do {                                                                           \
        nvfp4_status s_ = (expr);                                                  \
        if (s_ != NVFP4_OK) {                                                      \
            fprintf(stderr, "%s failed: status %d (%s)\n", #expr, (int)s_,         \
                    nvfp4_get_last_error_string());                                \
            return 3;                                                              \
        }                                                                          \
    } while (0)

/* An invalid call must return `want` and leave a non-empty message. */
#define EXPECT_STATUS(expr, want)                                                  \
    do {                                                                           \
        nvfp4_status s_ = (expr);                                                  \
        const char* msg_ = nvfp4_get_last_error_string();                          \
        if (s_ != (want) || msg_ == NULL || msg_[0] == '\0') {                     \
            fprintf(stderr, "%s returned %d, expected %d (message '%s')\n", #expr, \
                    (int)s_, (int)(want), msg_ ? msg_ : "(null)");                 \
            return 4;                                                              \
        }                                                                          \
    } while (0)

static void* read_file(const char* dir, const char* name, size_t bytes)
{
    char path[4096];
    snprintf(path, sizeof path, "%s/%s", dir, name);
    FILE* f = fopen(path, "rb");
    if (f == NULL) return NULL;
    void* buf = malloc(bytes ? bytes : 1);
    size_t got = buf ? fread(buf, 1, bytes, f) : 0;
    fclose(f);
    if (got != bytes) {
        free(buf);
        return NULL;
    }
    return buf;
}

static int write_file(const char* dir, const char* name, const void* p, size_t bytes)
{
    char path[4096];
    snprintf(path, sizeof path, "%s/%s", dir, name);
    FILE* f = fopen(path, "wb");
    if (f == NULL) return -1;
    size_t put = fwrite(p, 1, bytes, f);
    fclose(f);
    return put == bytes ? 0 : -1;
}

/* Copy a device buffer to DIR/name. */
static int dump(const char* dir, const char* name, CUdeviceptr src, size_t bytes)
{
    void* h = malloc(bytes);
    if (h == NULL) return -1;
    int rc = cuMemcpyDtoH(h, src, bytes) == CUDA_SUCCESS ? write_file(dir, name, h, bytes) : -1;
    free(h);
    return rc;
}

int main(int argc, char** argv)
{
    if (argc != 5) {
        fprintf(stderr, "usage: %s DIR M N K\n", argv[0]);
        return 1;
    }
    const char* dir = argv[1];
    const int64_t m = atoll(argv[2]), n = atoll(argv[3]), k = atoll(argv[4]);
    if (m < 1 || n < 16 || k < 32) {
        fprintf(stderr, "bad shape\n");
        return 1;
    }
    const size_t a_bytes = (size_t)(m * k * 2), w_bytes = (size_t)(n * k * 2);
    void* a_host = read_file(dir, "a.bf16", a_bytes);
    void* w_host = read_file(dir, "w.bf16", w_bytes);
    if (a_host == NULL || w_host == NULL) {
        fprintf(stderr, "cannot read the inputs\n");
        return 1;
    }

    CUdevice dev;
    CUcontext ctx;
    CUstream stream;
    CHECK_CU(cuInit(0));
    CHECK_CU(cuDeviceGet(&dev, 0));
    CHECK_CU(cuDevicePrimaryCtxRetain(&ctx, dev));
    CHECK_CU(cuCtxSetCurrent(ctx));
    CHECK_CU(cuStreamCreate(&stream, CU_STREAM_NON_BLOCKING));

    const size_t aq_bytes = (size_t)(m * k / 2), wq_bytes = (size_t)(n * k / 2);
    const size_t asf_bytes = nvfp4_sf_bytes(m, k), wsf_bytes = nvfp4_sf_bytes(n, k);
    const size_t qws_bytes = nvfp4_quant_workspace_size();
    const size_t gws_bytes = nvfp4_gemm_workspace_size(m, n, k, NVFP4_GEMM_AUTO);
    if (asf_bytes == 0 || wsf_bytes == 0 || qws_bytes == 0) {
        fprintf(stderr, "layout helpers returned 0\n");
        return 1;
    }
    CUdeviceptr d_a, d_w, d_aq, d_asf, d_wq, d_wsf, d_scale, d_qws, d_c32, d_c16, d_gws = 0;
    CHECK_CU(cuMemAlloc(&d_a, a_bytes));
    CHECK_CU(cuMemAlloc(&d_w, w_bytes));
    CHECK_CU(cuMemAlloc(&d_aq, aq_bytes));
    CHECK_CU(cuMemAlloc(&d_asf, asf_bytes));
    CHECK_CU(cuMemAlloc(&d_wq, wq_bytes));
    CHECK_CU(cuMemAlloc(&d_wsf, wsf_bytes));
    CHECK_CU(cuMemAlloc(&d_scale, sizeof(float)));
    CHECK_CU(cuMemAlloc(&d_qws, qws_bytes));
    CHECK_CU(cuMemAlloc(&d_c32, (size_t)(m * n) * 4));
    CHECK_CU(cuMemAlloc(&d_c16, (size_t)(m * n) * 2));
    if (gws_bytes > 0) CHECK_CU(cuMemAlloc(&d_gws, gws_bytes));
    CHECK_CU(cuMemcpyHtoD(d_a, a_host, a_bytes));
    CHECK_CU(cuMemcpyHtoD(d_w, w_host, w_bytes));

    /* offline: the weight with its own computed global scale (synchronising) */
    float s_gw = 0.0f;
    CHECK_NV(nvfp4_quantize_weight((const void*)d_w, NVFP4_IN_BF16, n, k, k, 0, n, NULL, (uint8_t*)d_wq,
                                   (uint8_t*)d_wsf, &s_gw, (void*)d_qws, qws_bytes, stream));
    /* online: dynamic-scale activation quantisation, then the GEMM twice */
    CHECK_NV(nvfp4_quantize_act((const void*)d_a, NVFP4_IN_BF16, m, k, k, NULL, (float*)d_scale, (uint8_t*)d_aq,
                                (uint8_t*)d_asf, (void*)d_qws, qws_bytes, stream));
    const nvfp4_segment seg = {0, n, s_gw};
    CHECK_NV(nvfp4_gemm((const uint8_t*)d_aq, (const uint8_t*)d_asf, (const float*)d_scale, (const uint8_t*)d_wq,
                        (const uint8_t*)d_wsf, m, n, k, &seg, 1, (void*)d_c32, NVFP4_OUT_FP32, n, (void*)d_gws,
                        gws_bytes, NVFP4_GEMM_AUTO, stream));
    CHECK_NV(nvfp4_gemm((const uint8_t*)d_aq, (const uint8_t*)d_asf, (const float*)d_scale, (const uint8_t*)d_wq,
                        (const uint8_t*)d_wsf, m, n, k, &seg, 1, (void*)d_c16, NVFP4_OUT_BF16, n, (void*)d_gws,
                        gws_bytes, NVFP4_GEMM_AUTO, stream));
    CHECK_CU(cuStreamSynchronize(stream));
    CHECK_NV(nvfp4_check_device_status(stream));

    /* invalid calls: rejected on the host, nothing launched */
    EXPECT_STATUS(nvfp4_gemm((const uint8_t*)d_aq, (const uint8_t*)d_asf, (const float*)d_scale,
                             (const uint8_t*)d_wq, (const uint8_t*)d_wsf, m, n - 8, k, &seg, 1, (void*)d_c32,
                             NVFP4_OUT_FP32, n, NULL, 0, NVFP4_GEMM_FORCE_LARGE, stream),
                  NVFP4_ERR_INVALID_ARG);
    EXPECT_STATUS(nvfp4_gemm((const uint8_t*)d_aq, (const uint8_t*)d_asf, (const float*)d_scale,
                             (const uint8_t*)d_wq, (const uint8_t*)d_wsf, m, n, k, &seg, 1, (void*)(d_c32 + 4),
                             NVFP4_OUT_FP32, n, NULL, 0, NVFP4_GEMM_FORCE_LARGE, stream),
                  NVFP4_ERR_ALIGNMENT);
    EXPECT_STATUS(nvfp4_gemm((const uint8_t*)d_aq, (const uint8_t*)d_asf, (const float*)d_scale,
                             (const uint8_t*)d_wq, (const uint8_t*)d_wsf, 16, n, k, &seg, 1, (void*)d_c32,
                             NVFP4_OUT_FP32, n, NULL, 0, NVFP4_GEMM_FORCE_DECODE, stream),
                  NVFP4_ERR_WORKSPACE);
    const nvfp4_segment bad_seg = {0, n, -1.0f};
    EXPECT_STATUS(nvfp4_gemm((const uint8_t*)d_aq, (const uint8_t*)d_asf, (const float*)d_scale,
                             (const uint8_t*)d_wq, (const uint8_t*)d_wsf, m, n, k, &bad_seg, 1, (void*)d_c32,
                             NVFP4_OUT_FP32, n, NULL, 0, NVFP4_GEMM_FORCE_LARGE, stream),
                  NVFP4_ERR_INVALID_ARG);
    EXPECT_STATUS(nvfp4_quantize_act((const void*)d_a, NVFP4_IN_BF16, m, k, k, NULL, NULL, (uint8_t*)d_aq,
                                     (uint8_t*)d_asf, (void*)d_qws, qws_bytes, stream),
                  NVFP4_ERR_INVALID_ARG);
    if (nvfp4_sf_offset(-1, 0, k) != -1 || nvfp4_sf_bytes(1, 15) != 0) {
        fprintf(stderr, "layout helpers accept out-of-range arguments\n");
        return 4;
    }

    float s_ga = 0.0f;
    CHECK_CU(cuMemcpyDtoH(&s_ga, d_scale, sizeof s_ga));
    const float scales[2] = {s_ga, s_gw};
    if (write_file(dir, "scales.bin", scales, sizeof scales) || dump(dir, "a_q.bin", d_aq, aq_bytes) ||
        dump(dir, "a_sf.bin", d_asf, asf_bytes) || dump(dir, "w_q.bin", d_wq, wq_bytes) ||
        dump(dir, "w_sf.bin", d_wsf, wsf_bytes) || dump(dir, "c32.bin", d_c32, (size_t)(m * n) * 4) ||
        dump(dir, "c16.bin", d_c16, (size_t)(m * n) * 2)) {
        fprintf(stderr, "cannot write the outputs\n");
        return 5;
    }

    CUdeviceptr all[] = {d_a, d_w, d_aq, d_asf, d_wq, d_wsf, d_scale, d_qws, d_c32, d_c16, d_gws};
    for (size_t i = 0; i < sizeof all / sizeof all[0]; ++i)
        if (all[i]) cuMemFree(all[i]);
    cuStreamDestroy(stream);
    cuDevicePrimaryCtxRelease(dev);
    free(a_host);
    free(w_host);
    printf("ok: libnvfp4 version %d, s_ga %.9g, s_gw %.9g\n", nvfp4_version(), (double)s_ga, (double)s_gw);
    return 0;
}
