/* Oracle for the ZeRO-1/2 sharded optimizer step -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, single-threaded CPU statement of what one sharded step
 * computes.  Only the tests, the smoke check and the benchmark's CPU-baseline
 * leg may load it; the product path never does.  It shares no code with the
 * CUDA library (its own partitioner, its own bf16 rounding, its own AdamW).
 *
 * Sources (the web pages on distributed data parallelism and ZeRO):
 *  - "CS336 lecture 8, parallelism basics" (runguoli.com course notes), section
 *    "ZeRO levels" and the ZeRO-1 code sketch: full local gradient ->
 *    reduce-scatter (SUM) -> each rank updates only its slice's fp32 state ->
 *    all-gather of the updated bf16 parameters; 16 bytes per parameter.
 *  - "Scaling training to thousands of GPUs" (Tazi talk summary), section
 *    11:24 ZeRO: AllReduce = reduce-scatter + all-gather; flattened (FSDP1)
 *    versus whole-tensor (FSDP2 / Muon) sharding; 03:41 DP: bucketed
 *    gradients sized by bucket_cap_mb, gradients averaged over replicas.
 *  - "DDP -> ZeRO -> TP/PP/CP" blog, section 2.1 (25 MB default bucket, the
 *    backward pass fills buckets), section 3.1 (the memory ledger), 1.1
 *    (AdamW keeps fp32 master, m and v).
 * The pages do not write the AdamW formula; it is the published one
 * (Kingma & Ba 2015, bias-corrected Adam; Loshchilov & Hutter 2019, decoupled
 * weight decay).  Gradient clipping is not on the pages; the convention is the
 * common global-norm one.  Readings where the pages are silent:
 *  - reduce: left fold in rank order 0..W-1 in fp32 starting from g_0, then
 *    one IEEE division by W;
 *  - AdamW scalars (bias corrections, step size, decay factor) in fp64,
 *    rounded once to fp32; per-element arithmetic in fp32 in the order
 *    written in oracle_adamw_element(), no fused multiply-add (built with
 *    -ffp-contract=off);
 *  - clip coefficient c = min(1, max_norm / (sqrt(S) + 1e-6)) in fp64,
 *    rounded to fp32, S the sum of the exact fp64 squares of the averaged
 *    gradient over all N parameters, accumulated with compensated summation
 *    so that the sum is accurate to a few ulps at any length; g <- g * c in
 *    fp32 before m and v;
 *  - bf16 conversion: round to nearest, ties to even; NaN stays a quiet NaN.
 *
 * Parity of every function here is pinned by tests/test_oracle_*.py against
 * closed forms, library routines on special cases, brute force and the
 * numbers printed on the pages.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_FLAT 0
#define OR_WHOLE 1

/* ------------------------------------------------------------------------ */
/* bf16 <-> fp32                                                             */
/* ------------------------------------------------------------------------ */

float oracle_bf16_to_f32(uint16_t h) {
    /* bf16 is the top half of an fp32 bit pattern. */
    uint32_t bits = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return f;
}

uint16_t oracle_f32_to_bf16(float f) {
    uint32_t bits;
    memcpy(&bits, &f, sizeof bits);
    uint32_t exponent = (bits >> 23) & 0xFFu;
    uint32_t fraction = bits & 0x7FFFFFu;
    if (exponent == 0xFFu && fraction != 0u) {
        /* NaN: keep the sign and the top payload bits, force it quiet. */
        return (uint16_t)((bits >> 16) | 0x0040u);
    }
    /* Keep the top 16 bits; the lower 16 are the part to round away. */
    uint32_t kept = bits >> 16;
    uint32_t rest = bits & 0xFFFFu;
    const uint32_t half = 0x8000u;
    int round_up = 0;
    if (rest > half) round_up = 1;                      /* more than half an ulp */
    else if (rest == half && (kept & 1u)) round_up = 1; /* a tie: go to even */
    /* Sign-magnitude: incrementing the magnitude rounds away from zero; a
     * carry out of the fraction bumps the exponent, up to infinity. */
    return (uint16_t)(kept + (uint32_t)round_up);
}

void oracle_f32_to_bf16_array(const float* x, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_f32_to_bf16(x[i]);
}

/* ------------------------------------------------------------------------ */
/* Partition, buckets and segments                                          */
/* ------------------------------------------------------------------------ */

typedef struct {
    int32_t bucket;
    int32_t tensor;   /* -1: the flat partition's zero pad */
    int32_t owner;
    int32_t reserved;
    int64_t offset_in_tensor;
    int64_t length;
    int64_t global_offset;
    int64_t owned_offset;
} oracle_segment;

typedef struct {
    int64_t total_numel;   /* N */
    int64_t padded_numel;  /* W * C (flat) or N (whole-tensor) */
    int64_t chunk;         /* C = ceil(N / W) (flat), 0 (whole-tensor) */
    int32_t n_buckets;
    int32_t reserved;
    int64_t n_segments;
} oracle_plan_info;

/* Returns 0 on success, -1 on bad arguments, -2 if seg_cap is too small
 * (n_segments is still filled in).  groups == NULL: buckets by the cap
 * rule; else one group id per tensor, non-decreasing in declaration order,
 * and one bucket per group (cap_bytes unused). */
int oracle_plan_groups(int32_t n_tensors, const int32_t* ndims, const int64_t* dims_flat,
                       int32_t world_size, int32_t mode, uint64_t cap_bytes, const int32_t* groups,
                       int32_t* tensor_owner,     /* [n_tensors]; -1 in flat mode       */
                       int32_t* tensor_bucket,    /* [n_tensors]                        */
                       int64_t* owned_numel,      /* [world_size]                       */
                       oracle_segment* segs, int64_t seg_cap, oracle_plan_info* info) {
    if (n_tensors < 0 || world_size < 1 || (mode != OR_FLAT && mode != OR_WHOLE)) return -1;
    if (groups)
        for (int32_t t = 1; t < n_tensors; ++t)
            if (groups[t] < groups[t - 1]) return -1;

    int64_t* numel = (int64_t*)calloc((size_t)n_tensors + 1, sizeof(int64_t));
    int64_t* goff = (int64_t*)calloc((size_t)n_tensors + 1, sizeof(int64_t));
    int64_t* owned_off = (int64_t*)calloc((size_t)n_tensors + 1, sizeof(int64_t));
    int32_t* order = (int32_t*)calloc((size_t)n_tensors + 1, sizeof(int32_t));
    if (!numel || !goff || !owned_off || !order) return -1;

    /* Element counts from the shapes; global flat layout = declaration order. */
    int64_t pos = 0, N = 0;
    for (int32_t t = 0; t < n_tensors; ++t) {
        int64_t n = 1;
        for (int32_t d = 0; d < ndims[t]; ++d) {
            if (dims_flat[pos + d] < 0) { free(numel); free(goff); free(owned_off); free(order); return -1; }
            n *= dims_flat[pos + d];
        }
        pos += ndims[t];
        numel[t] = n;
        goff[t] = N;
        N += n;
    }

    for (int32_t r = 0; r < world_size; ++r) owned_numel[r] = 0;
    int64_t C = 0, padded = N;
    if (mode == OR_FLAT) {
        /* Concatenate and pad with zeros to W equal chunks of C = ceil(N/W). */
        C = (N + world_size - 1) / world_size;
        padded = C * world_size;
        for (int32_t r = 0; r < world_size; ++r) owned_numel[r] = C;
        for (int32_t t = 0; t < n_tensors; ++t) tensor_owner[t] = -1;
    } else {
        /* Whole tensors, greedy longest-processing-time: largest tensor first
         * (ties: lower declaration index first), each to the least-loaded rank
         * (ties: lowest rank).  Insertion sort keeps it obvious. */
        for (int32_t t = 0; t < n_tensors; ++t) order[t] = t;
        for (int32_t i = 1; i < n_tensors; ++i) {
            int32_t cur = order[i];
            int32_t j = i - 1;
            while (j >= 0 && (numel[order[j]] < numel[cur] ||
                              (numel[order[j]] == numel[cur] && order[j] > cur))) {
                order[j + 1] = order[j];
                --j;
            }
            order[j + 1] = cur;
        }
        for (int32_t i = 0; i < n_tensors; ++i) {
            int32_t t = order[i];
            int32_t best = 0;
            for (int32_t r = 1; r < world_size; ++r)
                if (owned_numel[r] < owned_numel[best]) best = r;
            tensor_owner[t] = best;
            owned_numel[best] += numel[t];
        }
        /* Owned order: a rank's tensors in declaration order. */
        int64_t* fill = (int64_t*)calloc((size_t)world_size, sizeof(int64_t));
        for (int32_t t = 0; t < n_tensors; ++t) {
            owned_off[t] = fill[tensor_owner[t]];
            fill[tensor_owner[t]] += numel[t];
        }
        free(fill);
    }

    /* Buckets: walk the tensors in reverse declaration order (the order the
     * backward pass produces gradients); open a new bucket when the next
     * tensor's bf16 gradient bytes would push a non-empty bucket past the cap
     * -- or, with groups, whenever the next tensor belongs to another group
     * (a layer's gradients are reduced together once its backward is done). */
    int32_t bucket = 0;
    uint64_t fill_bytes = 0;
    int holds_any = 0;
    for (int32_t t = n_tensors - 1; t >= 0; --t) {
        uint64_t bytes = 2u * (uint64_t)numel[t];
        int new_bucket = groups ? (holds_any && groups[t] != groups[t + 1])
                                : (holds_any && fill_bytes + bytes > cap_bytes);
        if (new_bucket) {
            bucket += 1;
            fill_bytes = 0;
            holds_any = 0;
        }
        tensor_bucket[t] = bucket;
        fill_bytes += bytes;
        holds_any = 1;
    }
    int32_t n_buckets = n_tensors > 0 ? bucket + 1 : 0;

    /* Segments: bucket by bucket, tensors in packing order, each tensor cut
     * where the owner changes; the flat pad closes bucket 0. */
    int64_t ns = 0;
#define EMIT(B, T, OFF, LEN, OWN, GOFF, OOFF)                                    \
    do {                                                                         \
        if (ns < seg_cap) {                                                      \
            segs[ns].bucket = (B); segs[ns].tensor = (T); segs[ns].owner = (OWN); \
            segs[ns].reserved = 0; segs[ns].offset_in_tensor = (OFF);            \
            segs[ns].length = (LEN); segs[ns].global_offset = (GOFF);            \
            segs[ns].owned_offset = (OOFF);                                      \
        }                                                                        \
        ++ns;                                                                    \
    } while (0)

    for (int32_t b = 0; b < n_buckets; ++b) {
        for (int32_t t = n_tensors - 1; t >= 0; --t) {
            if (tensor_bucket[t] != b || numel[t] == 0) continue;
            if (mode == OR_FLAT) {
                int64_t x = goff[t], end = goff[t] + numel[t];
                while (x < end) {
                    int64_t r = x / C;
                    int64_t stop = (r + 1) * C < end ? (r + 1) * C : end;
                    EMIT(b, t, x - goff[t], stop - x, (int32_t)r, x, x - r * C);
                    x = stop;
                }
            } else {
                EMIT(b, t, 0, numel[t], tensor_owner[t], goff[t], owned_off[t]);
            }
        }
        if (b == 0 && mode == OR_FLAT && padded > N) {
            int64_t x = N;
            while (x < padded) {
                int64_t r = x / C;
                int64_t stop = (r + 1) * C < padded ? (r + 1) * C : padded;
                EMIT(b, -1, x - N, stop - x, (int32_t)r, x, x - r * C);
                x = stop;
            }
        }
    }
#undef EMIT

    info->total_numel = N;
    info->padded_numel = padded;
    info->chunk = C;
    info->n_buckets = n_buckets;
    info->reserved = 0;
    info->n_segments = ns;
    free(numel); free(goff); free(owned_off); free(order);
    return ns > seg_cap ? -2 : 0;
}

/* The cap rule alone (no groups). */
int oracle_plan(int32_t n_tensors, const int32_t* ndims, const int64_t* dims_flat,
                int32_t world_size, int32_t mode, uint64_t cap_bytes,
                int32_t* tensor_owner, int32_t* tensor_bucket, int64_t* owned_numel,
                oracle_segment* segs, int64_t seg_cap, oracle_plan_info* info) {
    return oracle_plan_groups(n_tensors, ndims, dims_flat, world_size, mode, cap_bytes, NULL,
                              tensor_owner, tensor_bucket, owned_numel, segs, seg_cap, info);
}

/* ------------------------------------------------------------------------ */
/* Reduce (the local stand-in for the gradient reduce-scatter)               */
/* ------------------------------------------------------------------------ */

/* g[i] = (g_0[i] + g_1[i] + ... + g_{W-1}[i]) / W, fp32, left to right. */
void oracle_reduce(int32_t world_size, const uint16_t* const* grads, int64_t n, float* g_out) {
    for (int64_t i = 0; i < n; ++i) {
        float s = oracle_bf16_to_f32(grads[0][i]);
        for (int32_t w = 1; w < world_size; ++w) s = s + oracle_bf16_to_f32(grads[w][i]);
        g_out[i] = s / (float)world_size;
    }
}

/* ------------------------------------------------------------------------ */
/* AdamW                                                                    */
/* ------------------------------------------------------------------------ */

typedef struct {
    float lr, beta1, beta2, eps, weight_decay, max_grad_norm;
} oracle_hp;

typedef struct {
    float beta1, beta2, one_minus_beta1, one_minus_beta2;
    float step_size;   /* lr / (1 - beta1^t)          */
    float bc2_sqrt;    /* sqrt(1 - beta2^t)           */
    float decay;       /* 1 - lr * weight_decay       */
    float eps;
} oracle_scalars;

/* Step t >= 1.  Everything in fp64 from the fp32 hyperparameters, rounded once. */
void oracle_adamw_scalars(const oracle_hp* hp, int64_t t, oracle_scalars* out) {
    double b1 = (double)hp->beta1, b2 = (double)hp->beta2, lr = (double)hp->lr;
    double bias1 = 1.0 - pow(b1, (double)t);
    double bias2 = 1.0 - pow(b2, (double)t);
    out->beta1 = hp->beta1;
    out->beta2 = hp->beta2;
    out->one_minus_beta1 = (float)(1.0 - b1);
    out->one_minus_beta2 = (float)(1.0 - b2);
    out->step_size = (float)(lr / bias1);
    out->bc2_sqrt = (float)sqrt(bias2);
    out->decay = (float)(1.0 - lr * (double)hp->weight_decay);
    out->eps = hp->eps;
}

/* One element: decoupled decay on the pre-update weight, then the
 * bias-corrected Adam step.  fp32, one rounding per operation. */
static void oracle_adamw_element(const oracle_scalars* s, float g, float* p, float* m, float* v) {
    float m_new = s->beta1 * *m + s->one_minus_beta1 * g;
    float g_sq = g * g;
    float v_new = s->beta2 * *v + s->one_minus_beta2 * g_sq;
    float p_new = *p * s->decay;
    float denom = sqrtf(v_new) / s->bc2_sqrt + s->eps;
    float update = (s->step_size * m_new) / denom;
    p_new = p_new - update;
    *m = m_new;
    *v = v_new;
    *p = p_new;
}

void oracle_adamw(const oracle_scalars* s, const float* g, int64_t n, float* p, float* m, float* v) {
    for (int64_t i = 0; i < n; ++i) oracle_adamw_element(s, g[i], &p[i], &m[i], &v[i]);
}

/* ------------------------------------------------------------------------ */
/* Global-norm clip                                                         */
/* ------------------------------------------------------------------------ */

/* Sum of squares in fp64.  Each square of an fp32 value is exact in fp64
 * (24-bit significand squared fits in 53 bits).  The additions use
 * Neumaier's compensated summation: alongside the running sum, a running
 * correction collects the low-order bits every addition rounds away, so the
 * result is within about two units in the last place of the exact sum
 * however many terms there are (a plain running sum of 1e8 terms can drift
 * by ~1e-11 relative). */
double oracle_sumsq(const float* g, int64_t n) {
    double sum = 0.0, correction = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        double x = (double)g[i] * (double)g[i];
        double t = sum + x;
        if (fabs(sum) >= fabs(x)) correction += (sum - t) + x;
        else correction += (x - t) + sum;
        sum = t;
    }
    return sum + correction;
}

float oracle_clip_coef(double sumsq, float max_norm) {
    double c = (double)max_norm / (sqrt(sumsq) + 1e-6);
    return (float)(c < 1.0 ? c : 1.0);
}

void oracle_scale(float* g, int64_t n, float c) {
    for (int64_t i = 0; i < n; ++i) g[i] = g[i] * c;
}

/* ------------------------------------------------------------------------ */
/* One rank's sharded step and the unsharded comparator                     */
/* ------------------------------------------------------------------------ */

/* grads[w]: replica w's gradient for this rank's owned elements (owned
 * order, n_owned bf16).  master/m/v: this rank's fp32 state (owned order).
 * param_out: the full bf16 buffer (global layout); only this rank's segments
 * are written.  clip_coef: pass 1.0f for no clipping (g * 1 == g exactly) or
 * the coefficient from oracle_clip_coef().  g_scratch: n_owned floats. */
void oracle_rank_step(int32_t world_size, int32_t rank, const oracle_segment* segs, int64_t n_segs,
                      const uint16_t* const* grads, int64_t n_owned,
                      float* master, float* m, float* v, uint16_t* param_out,
                      const oracle_hp* hp, int64_t t, float clip_coef, int use_clip,
                      float* g_scratch) {
    oracle_scalars s;
    oracle_adamw_scalars(hp, t, &s);
    oracle_reduce(world_size, grads, n_owned, g_scratch);
    if (use_clip) oracle_scale(g_scratch, n_owned, clip_coef);
    oracle_adamw(&s, g_scratch, n_owned, master, m, v);
    for (int64_t k = 0; k < n_segs; ++k) {
        if (segs[k].owner != rank) continue;
        for (int64_t j = 0; j < segs[k].length; ++j)
            param_out[segs[k].global_offset + j] =
                oracle_f32_to_bf16(master[segs[k].owned_offset + j]);
    }
}

/* Plain data-parallel step: every replica's full gradient (global layout,
 * length n) averaged in rank order, AdamW over all n elements, bf16 copy. */
void oracle_ddp_step(int32_t world_size, const uint16_t* const* full_grads, int64_t n,
                     float* master, float* m, float* v, uint16_t* param_out,
                     const oracle_hp* hp, int64_t t, float clip_coef, int use_clip,
                     float* g_scratch) {
    oracle_scalars s;
    oracle_adamw_scalars(hp, t, &s);
    oracle_reduce(world_size, full_grads, n, g_scratch);
    if (use_clip) oracle_scale(g_scratch, n, clip_coef);
    oracle_adamw(&s, g_scratch, n, master, m, v);
    oracle_f32_to_bf16_array(master, n, param_out);
}

/* ------------------------------------------------------------------------ */
/* Flat pad / unpad                                                          */
/* ------------------------------------------------------------------------ */

/* Concatenate n_tensors bf16 tensors (pointers + element counts) into a
 * buffer of padded_numel elements, zero filling the tail. */
void oracle_pad(int32_t n_tensors, const uint16_t* const* tensors, const int64_t* numels,
                int64_t padded_numel, uint16_t* out) {
    int64_t pos = 0;
    for (int32_t t = 0; t < n_tensors; ++t)
        for (int64_t j = 0; j < numels[t]; ++j) out[pos++] = tensors[t][j];
    while (pos < padded_numel) out[pos++] = 0;
}

void oracle_unpad(int32_t n_tensors, const uint16_t* flat, const int64_t* numels,
                  uint16_t* const* tensors) {
    int64_t pos = 0;
    for (int32_t t = 0; t < n_tensors; ++t)
        for (int64_t j = 0; j < numels[t]; ++j) tensors[t][j] = flat[pos++];
}
