/* Plain-C use of the library through include/zr.h: device buffers from
 * cudaMalloc, no Python, no torch.  Builds a plan for one rank of a small
 * flat partition, binds a workspace, runs four steps with constant
 * gradients (the last in checked mode, whose status must stay clean) and
 * checks the closed form of AdamW with a constant gradient: each step moves
 * p to p * (1 - lr * wd) - lr * g / (|g| + eps) (the bias corrections
 * cancel), within fp32 rounding.  Then the ZeRO-3 calls and a grouped
 * plan stepped bucket by bucket with clipping (see below).  Exit status 0
 * on success. */
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

    /* ZeRO-3 calls from C: a one-rank plan of the same tensors steps once
     * in the global layout and once (on its own copy of the state) in the
     * owned-order layout; zr_gather_params then reassembles the tensors
     * from the shard, which must equal the global-layout result. */
    int64_t mism3 = 0;
    {
        const zr_adamw hp1 = {3e-4f, 0.9f, 0.999f, 1e-8f, 0.1f, 0.0f};
        zr_plan *g1 = NULL, *s1 = NULL;
        CHECK_ZR(zr_plan_create(3, ndims, shapes, 1, 0, ZR_PARTITION_FLAT, 4096, &hp1, &g1));
        CHECK_ZR(zr_plan_create(3, ndims, shapes, 1, 0, ZR_PARTITION_FLAT, 4096, &hp1, &s1));
        uint64_t b1 = 0, b2 = 0;
        CHECK_ZR(zr_plan_workspace_bytes(g1, &b1));
        CHECK_ZR(zr_plan_workspace_bytes(s1, &b2));
        void *w1, *w2;
        CHECK_CUDA(cudaMalloc(&w1, b1));
        CHECK_CUDA(cudaMalloc(&w2, b2));
        CHECK_ZR(zr_plan_set_workspace(g1, w1, b1, (zr_stream_t)stream));
        CHECK_ZR(zr_plan_set_workspace(s1, w2, b2, (zr_stream_t)stream));
        CHECK_ZR(zr_plan_set_param_layout(s1, ZR_PARAMS_OWNED, (zr_stream_t)stream));
        const int64_t N = total;
        uint16_t* hg = (uint16_t*)malloc(sizeof(uint16_t) * N);
        float* hp0 = (float*)malloc(sizeof(float) * N);
        for (int64_t i = 0; i < N; ++i) {
            hg[i] = bf16_of((float)((i % 7) - 3) / 8.0f);
            hp0[i] = 0.01f * (float)((i % 13) - 6);
        }
        void *grad1, *out_g, *shard, *gathered;
        float *ms[2], *mm[2], *vv[2];
        CHECK_CUDA(cudaMalloc(&grad1, sizeof(uint16_t) * N));
        CHECK_CUDA(cudaMemcpy(grad1, hg, sizeof(uint16_t) * N, cudaMemcpyHostToDevice));
        for (int k = 0; k < 2; ++k) {
            CHECK_CUDA(cudaMalloc((void**)&ms[k], sizeof(float) * N));
            CHECK_CUDA(cudaMalloc((void**)&mm[k], sizeof(float) * N));
            CHECK_CUDA(cudaMalloc((void**)&vv[k], sizeof(float) * N));
            CHECK_CUDA(cudaMemcpy(ms[k], hp0, sizeof(float) * N, cudaMemcpyHostToDevice));
            CHECK_CUDA(cudaMemset(mm[k], 0, sizeof(float) * N));
            CHECK_CUDA(cudaMemset(vv[k], 0, sizeof(float) * N));
        }
        CHECK_CUDA(cudaMalloc(&out_g, sizeof(uint16_t) * N));
        CHECK_CUDA(cudaMalloc(&shard, sizeof(uint16_t) * N));
        CHECK_CUDA(cudaMalloc(&gathered, sizeof(uint16_t) * N));
        const void* one_grad[1] = {grad1};
        CHECK_ZR(zr_step(g1, one_grad, ms[0], mm[0], vv[0], out_g, 1, (zr_stream_t)stream));
        CHECK_ZR(zr_step(s1, one_grad, ms[1], mm[1], vv[1], shard, 1, (zr_stream_t)stream));
        const void* shards[1] = {shard};
        CHECK_ZR(zr_gather_params(s1, 0, 3, shards, gathered, 0, (zr_stream_t)stream));
        CHECK_CUDA(cudaStreamSynchronize(stream));
        uint16_t* a = (uint16_t*)malloc(sizeof(uint16_t) * N);
        uint16_t* b = (uint16_t*)malloc(sizeof(uint16_t) * N);
        CHECK_CUDA(cudaMemcpy(a, out_g, sizeof(uint16_t) * N, cudaMemcpyDeviceToHost));
        CHECK_CUDA(cudaMemcpy(b, gathered, sizeof(uint16_t) * N, cudaMemcpyDeviceToHost));
        for (int64_t i = 0; i < N; ++i) mism3 += a[i] != b[i];
        zr_plan_destroy(g1);
        zr_plan_destroy(s1);
    }
    /* Buckets by tensor group with clipping, from C: one rank, groups
     * {0, 1, 1} (two buckets).  zr_step on one copy of the state; on the
     * other, zr_step_bucket for both buckets (each bucket's gradient is
     * overwritten right after its call: a grouped plan keeps the fp32
     * averaged gradient), zr_bucket_sumsq, zr_step_finish.  Master weights
     * and the sum of squares must agree bit for bit. */
    int64_t mismg = 0;
    {
        const zr_adamw hpc = {3e-4f, 0.9f, 0.999f, 1e-8f, 0.1f, 0.5f};
        const int32_t groups[3] = {0, 1, 1};
        zr_plan *pa = NULL, *pb = NULL;
        CHECK_ZR(zr_plan_create_grouped(3, ndims, shapes, groups, 1, 0, ZR_PARTITION_FLAT, &hpc, &pa));
        CHECK_ZR(zr_plan_create_grouped(3, ndims, shapes, groups, 1, 0, ZR_PARTITION_FLAT, &hpc, &pb));
        int32_t n_buckets = 0;
        CHECK_ZR(zr_plan_query(pb, NULL, NULL, NULL, &n_buckets, NULL));
        if (n_buckets != 2) {
            fprintf(stderr, "grouped plan: %d buckets\n", (int)n_buckets);
            return 1;
        }
        uint64_t ba = 0, bb = 0;
        CHECK_ZR(zr_plan_workspace_bytes(pa, &ba));
        CHECK_ZR(zr_plan_workspace_bytes(pb, &bb));
        void *wa, *wb;
        double* part;                       /* [0]: plan a's partials, [1]: plan b's, [2]: zr_bucket_sumsq */
        CHECK_CUDA(cudaMalloc(&wa, ba));
        CHECK_CUDA(cudaMalloc(&wb, bb));
        CHECK_CUDA(cudaMalloc((void**)&part, 3 * sizeof(double)));
        CHECK_ZR(zr_plan_set_workspace(pa, wa, ba, (zr_stream_t)stream));
        CHECK_ZR(zr_plan_set_workspace(pb, wb, bb, (zr_stream_t)stream));
        CHECK_ZR(zr_plan_set_sumsq_partials(pa, part));
        CHECK_ZR(zr_plan_set_sumsq_partials(pb, part + 1));
        const int64_t N = total;
        uint16_t* hg = (uint16_t*)malloc(sizeof(uint16_t) * N);
        float* hp0 = (float*)malloc(sizeof(float) * N);
        for (int64_t i = 0; i < N; ++i) {
            hg[i] = bf16_of((float)((i % 11) - 5) / 16.0f);
            hp0[i] = 0.01f * (float)((i % 9) - 4);
        }
        void *ga, *gb, *oa, *ob;
        float *ms[2], *mm[2], *vv[2];
        CHECK_CUDA(cudaMalloc(&ga, sizeof(uint16_t) * N));
        CHECK_CUDA(cudaMalloc(&gb, sizeof(uint16_t) * N));
        CHECK_CUDA(cudaMemcpy(ga, hg, sizeof(uint16_t) * N, cudaMemcpyHostToDevice));
        CHECK_CUDA(cudaMemcpy(gb, hg, sizeof(uint16_t) * N, cudaMemcpyHostToDevice));
        for (int k = 0; k < 2; ++k) {
            CHECK_CUDA(cudaMalloc((void**)&ms[k], sizeof(float) * N));
            CHECK_CUDA(cudaMalloc((void**)&mm[k], sizeof(float) * N));
            CHECK_CUDA(cudaMalloc((void**)&vv[k], sizeof(float) * N));
            CHECK_CUDA(cudaMemcpy(ms[k], hp0, sizeof(float) * N, cudaMemcpyHostToDevice));
            CHECK_CUDA(cudaMemset(mm[k], 0, sizeof(float) * N));
            CHECK_CUDA(cudaMemset(vv[k], 0, sizeof(float) * N));
        }
        CHECK_CUDA(cudaMalloc(&oa, sizeof(uint16_t) * N));
        CHECK_CUDA(cudaMalloc(&ob, sizeof(uint16_t) * N));
        const void* grad_a[1] = {ga};
        const void* grad_b[1] = {gb};
        CHECK_ZR(zr_step(pa, grad_a, ms[0], mm[0], vv[0], oa, 1, (zr_stream_t)stream));
        zr_segment segs[16];
        int64_t n_seg = 0;
        CHECK_ZR(zr_plan_segments(pb, segs, 16, &n_seg));
        for (int32_t bkt = 0; bkt < n_buckets; ++bkt) {
            CHECK_ZR(zr_step_bucket(pb, bkt, grad_b, ms[1], mm[1], vv[1], ob, 1, (zr_stream_t)stream));
            for (int64_t k = 0; k < n_seg; ++k)     /* release: the bucket's gradient is gone */
                if (segs[k].bucket == bkt)
                    CHECK_CUDA(cudaMemsetAsync((uint16_t*)gb + segs[k].owned_offset, 0xFF,
                                               sizeof(uint16_t) * segs[k].length, stream));
        }
        CHECK_ZR(zr_bucket_sumsq(pb, part + 2, (zr_stream_t)stream));
        CHECK_ZR(zr_step_finish(pb, NULL, ms[1], mm[1], vv[1], ob, 1, (zr_stream_t)stream));
        CHECK_CUDA(cudaStreamSynchronize(stream));
        uint32_t* a = (uint32_t*)malloc(sizeof(float) * N);
        uint32_t* b = (uint32_t*)malloc(sizeof(float) * N);
        CHECK_CUDA(cudaMemcpy(a, ms[0], sizeof(float) * N, cudaMemcpyDeviceToHost));
        CHECK_CUDA(cudaMemcpy(b, ms[1], sizeof(float) * N, cudaMemcpyDeviceToHost));
        for (int64_t i = 0; i < N; ++i) mismg += a[i] != b[i];
        double hpart[3];
        CHECK_CUDA(cudaMemcpy(hpart, part, sizeof(hpart), cudaMemcpyDeviceToHost));
        if (hpart[0] != hpart[1] || hpart[1] != hpart[2] || !(hpart[0] > 0.0)) {
            fprintf(stderr, "sums of squares differ: %.17g %.17g %.17g\n", hpart[0], hpart[1], hpart[2]);
            ++mismg;
        }
        zr_plan_destroy(pa);
        zr_plan_destroy(pb);
    }
    printf("owned %lld, mismatches %lld, zero-3 mismatches %lld, grouped mismatches %lld\n", (long long)owned,
           (long long)bad, (long long)mism3, (long long)mismg);
    return (bad == 0 && mism3 == 0 && mismg == 0) ? 0 : 1;
}
