/* Plain-C use of the library through include/zr.h: device buffers from
 * cudaMalloc, no Python, no torch.  Builds a plan for one rank of a small
 * flat partition, binds a workspace, runs four steps with constant
 * gradients (the last in checked mode, whose status must stay clean) and
 * checks the closed form of AdamW with a constant gradient:
 * each step moves p to p * (1 - lr * wd) - lr * g / (|g| + eps) (the bias
 * corrections cancel), within fp32 rounding.  Exit status 0 on success. */
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "zr.h"

#define CHECK_ZR(call)                                                          \
    do {                                                                        \
        zr_status s_ = (call);                                                  \
        if (s_ != ZR_OK) {                                                      \
            fprintf(stderr, "%s: %s\n", #call, zr_status_string(s_));          \
            return 1;                                                           \
        }                                                                       \
    } while (0)
#define CHECK_CUDA(call)                                                        \
    do {                                                                        \
        cudaError_t e_ = (call);                                                \
        if (e_ != cudaSuccess) {                                                \
            fprintf(stderr, "%s: %s\n", #call, cudaGetErrorString(e_));        \
            return 1;                                                           \
        }                                                                       \
    } while (0)

static uint16_t bf16_of(float x) { /* exact for the values used here */
    uint32_t b;
    memcpy(&b, &x, 4);
    return (uint16_t)(b >> 16);
}

int main(void) {
    const int64_t d0[2] = {1000, 33}, d1[1] = {7777}, d2[3] = {4, 5, 6};
    const int64_t* shapes[3] = {d0, d1, d2};
    const int32_t ndims[3] = {2, 1, 3};
    const int32_t W = 4, rank = 1;
    const zr_adamw hp = {3e-4f, 0.9f, 0.999f, 1e-8f, 0.1f, 0.0f};
    zr_plan* plan = NULL;
    CHECK_ZR(zr_plan_create(3, ndims, shapes, W, rank, ZR_PARTITION_FLAT, 4096, &hp, &plan));
    int64_t total, padded, owned;
    int32_t nb;
    int64_t nseg;
    CHECK_ZR(zr_plan_query(plan, &total, &padded, &owned, &nb, &nseg));
    if (total != 33000 + 7777 + 120 || padded % W != 0 || owned != padded / W) {
        fprintf(stderr, "unexpected sizes\n");
        return 1;
    }
    uint64_t ws_bytes;
    CHECK_ZR(zr_plan_workspace_bytes(plan, &ws_bytes));
    void* ws;
    CHECK_CUDA(cudaMalloc(&ws, ws_bytes));
    cudaStream_t stream;
    CHECK_CUDA(cudaStreamCreate(&stream));
    CHECK_ZR(zr_plan_set_workspace(plan, ws, ws_bytes, (zr_stream_t)stream));

    /* replica w's gradient is the constant (w + 1) / 4: the average is 5/8 */
    void* grads[4];
    uint16_t* host_g = (uint16_t*)malloc(sizeof(uint16_t) * owned);
    for (int w = 0; w < W; ++w) {
        for (int64_t i = 0; i < owned; ++i) host_g[i] = bf16_of((float)(w + 1) / 4.0f);
        CHECK_CUDA(cudaMalloc(&grads[w], sizeof(uint16_t) * owned));
        CHECK_CUDA(cudaMemcpy(grads[w], host_g, sizeof(uint16_t) * owned, cudaMemcpyHostToDevice));
    }
    float *master, *m, *v;
    void* param_out;
    CHECK_CUDA(cudaMalloc((void**)&master, sizeof(float) * owned));
    CHECK_CUDA(cudaMalloc((void**)&m, sizeof(float) * owned));
    CHECK_CUDA(cudaMalloc((void**)&v, sizeof(float) * owned));
    CHECK_CUDA(cudaMalloc(&param_out, sizeof(uint16_t) * padded));
    float* host_p = (float*)malloc(sizeof(float) * owned);
    for (int64_t i = 0; i < owned; ++i) host_p[i] = 0.01f * (float)((i % 17) - 8);
    CHECK_CUDA(cudaMemcpy(master, host_p, sizeof(float) * owned, cudaMemcpyHostToDevice));
    CHECK_CUDA(cudaMemset(m, 0, sizeof(float) * owned));
    CHECK_CUDA(cudaMemset(v, 0, sizeof(float) * owned));

    for (int64_t t = 1; t <= 3; ++t)
        CHECK_ZR(zr_step(plan, (const void* const*)grads, master, m, v, param_out, t, (zr_stream_t)stream));
    /* a fourth step in checked mode: the device tables are verified first
     * and the status stays clean */
    CHECK_ZR(zr_plan_set_checked(plan, 1));
    CHECK_ZR(zr_step(plan, (const void* const*)grads, master, m, v, param_out, 4, (zr_stream_t)stream));
    zr_check_result cr;
    CHECK_ZR(zr_plan_check_result(plan, &cr, (zr_stream_t)stream));
    if (cr.bad_tiles != 0 || cr.first_bad != -1 || cr.hash_mismatch != 0 || cr.tables_emptied != 0) {
        fprintf(stderr, "checked mode flagged a clean plan\n");
        return 1;
    }
    CHECK_CUDA(cudaStreamSynchronize(stream));

    float* got = (float*)malloc(sizeof(float) * owned);
    CHECK_CUDA(cudaMemcpy(got, master, sizeof(float) * owned, cudaMemcpyDeviceToHost));
    const double g = 0.625, lr = 3e-4, wd = 0.1, eps = 1e-8;
    int64_t bad = 0;
    const int64_t first_global = rank * owned;
    for (int64_t i = 0; i < owned; ++i) {
        double want = host_p[i];
        const int is_pad = first_global + i >= total;
        for (int t = 1; t <= 4; ++t) want = want * (1.0 - lr * wd) - (is_pad ? 0.0 : lr * g / (fabs(g) + eps));
        if (fabs(got[i] - want) > 1e-6 * fmax(fabs(want), lr)) ++bad;
    }
    zr_plan_destroy(plan);
    printf("owned %lld, mismatches %lld\n", (long long)owned, (long long)bad);
    return bad == 0 ? 0 : 1;
}
