/*
 * CPU oracle for the dropless sparse Mixture-of-Experts feed-forward block.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load this library.  It shares no code with the CUDA
 * implementation and is deliberately plain and slow: scalar loops, float64
 * accumulation, no blocking and no reordering beyond what the definitions
 * below state.  The only parallelism is an OpenMP loop over independent tokens.
 *
 * What the block computes (one token t, hidden vector x_t of size H):
 *   1. router logits   l_e = sum_h x_t[h] * Wr[e][h] + b[e]     (e < E)
 *      "PhiMoE in Transformers", section 6: the top-k router is a bias-free
 *      nn.Linear hidden_size -> num_local_experts; the optional per-expert bias
 *      b is the input that skews expert load.
 *   2. selection: greedy top-1, mask it, take the next, ... k times; the k
 *      selected logits are soft-maxed and concatenated ("PhiMoE in
 *      Transformers", section 6, sparsemixer in eval mode, generalised from
 *      k = 2 to any k).  Ties go to the lower expert index.
 *   3. each selected expert e runs its SwiGLU FFN on x_t with the packed
 *      weights gate_up[e] = [gate (I rows); up (I rows)] x H and down[e] = H x I:
 *      g = gate x, u = up x, a = SiLU(g) * u, o = down a, SiLU(z) = z/(1+e^-z)
 *      ("PhiMoE in Transformers", section 2 item 3: gate_up_proj of shape
 *      (num_experts, 2*intermediate, hidden) chunked into gate then up;
 *      "Mixture of Experts in Transformers", WeightConverter section: w1 (gate)
 *      and w3 (up) concatenated in that order, down_proj stacked per expert).
 *   4. y_t = s * sum_j w_j o_j + sum over shared experts of their SwiGLU FFN
 *      on x_t (Instella-MoE walk-through, FarSkipMoE: routed + shared, routed
 *      scale 2.5; GraniteMoeSWA page, decoder layer: moe + shared_mlp).
 *   5. dropless dispatch: the slots (t, j) are grouped by expert with a stable
 *      counting sort (expert ascending, then slot id t*k+j ascending); every
 *      slot is kept ("Mixture of Experts in Transformers", grouped_mm backend:
 *      sort and group tokens by expert id; "PhiMoE in Transformers", section 2
 *      item 4: no token is dropped).
 *
 * Storage: activations and expert weights are float32 or bf16 bit patterns
 * (flag per tensor); bf16 is widened exactly to float before use.  The router
 * weight and bias are always float32.  All arithmetic is float64.  The expert
 * selection compares the logits rounded to float32, the precision in which the
 * CUDA path takes the same decision; the softmax uses the float64 logits.
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int64_t T;
    int32_t H, I, E, k;
    int32_t n_shared, I_shared;
    double routed_scale;
    int32_t act_bf16;   /* x is bf16 bits (uint16) instead of float32 */
    int32_t w_bf16;     /* expert weights are bf16 bits */
} oracle_shape;

static double widen(const void* p, int64_t i, int bf16)
{
    if (bf16) {
        uint32_t bits = (uint32_t)((const uint16_t*)p)[i] << 16;
        float f;
        memcpy(&f, &bits, sizeof f);
        return (double)f;
    }
    return (double)((const float*)p)[i];
}

/* Step 1 for one token. */
static void router_one(const oracle_shape* s, const void* x, int64_t t, const float* wr,
                       const float* b, double* logits)
{
    for (int32_t e = 0; e < s->E; ++e) {
        double acc = 0.0;
        for (int32_t h = 0; h < s->H; ++h)
            acc += widen(x, t * s->H + h, s->act_bf16) * (double)wr[(int64_t)e * s->H + h];
        logits[e] = acc + (b ? (double)b[e] : 0.0);
    }
}

/* Step 2 for one token: greedy masked argmax k times, then softmax over those k. */
static void topk_one(int32_t E, int32_t k, const double* logits, int32_t* idx, double* w)
{
    unsigned char taken[1024];
    memset(taken, 0, sizeof taken);
    for (int32_t j = 0; j < k; ++j) {
        int32_t best = -1;
        float best_v = 0.0f;
        for (int32_t e = 0; e < E; ++e) {
            if (taken[e]) continue;
            float v = (float)logits[e];
            if (best < 0 || v > best_v) { best = e; best_v = v; }
        }
        taken[best] = 1;
        idx[j] = best;
    }
    double mx = logits[idx[0]];
    for (int32_t j = 1; j < k; ++j)
        if (logits[idx[j]] > mx) mx = logits[idx[j]];
    double den = 0.0;
    for (int32_t j = 0; j < k; ++j) den += exp(logits[idx[j]] - mx);
    for (int32_t j = 0; j < k; ++j) w[j] = exp(logits[idx[j]] - mx) / den;
}

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* Step 3: one SwiGLU expert.  gate_up is [2I, H], down is [H, I], both row-major. */
static void expert_ffn(int32_t H, int32_t I, const void* gate_up, const void* down, int w_bf16,
                       const double* x, double* a, double* out)
{
    for (int32_t i = 0; i < I; ++i) {
        double g = 0.0, u = 0.0;
        for (int32_t h = 0; h < H; ++h) {
            g += widen(gate_up, (int64_t)i * H + h, w_bf16) * x[h];
            u += widen(gate_up, (int64_t)(I + i) * H + h, w_bf16) * x[h];
        }
        a[i] = silu(g) * u;
    }
    for (int32_t h = 0; h < H; ++h) {
        double acc = 0.0;
        for (int32_t i = 0; i < I; ++i) acc += widen(down, (int64_t)h * I + i, w_bf16) * a[i];
        out[h] = acc;
    }
}

static int shape_ok(const oracle_shape* s)
{
    return s && s->T >= 0 && s->H > 0 && s->I > 0 && s->E > 0 && s->E <= 1024 && s->k > 0 &&
           s->k <= s->E && s->n_shared >= 0 && (s->n_shared == 0 || s->I_shared > 0);
}

/* Exported: router logits for n tokens (tokens == NULL means 0..n-1). */
int oracle_router(const oracle_shape* s, const void* x, const float* wr, const float* b,
                  const int64_t* tokens, int64_t n, double* logits)
{
    if (!shape_ok(s)) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; ++r)
        router_one(s, x, tokens ? tokens[r] : r, wr, b, logits + r * s->E);
    return 0;
}

/* Exported: selection + softmax for n rows of logits. */
int oracle_topk_softmax(int64_t n, int32_t E, int32_t k, const double* logits, int32_t* idx,
                        double* w)
{
    if (E <= 0 || E > 1024 || k <= 0 || k > E) return -1;
    for (int64_t r = 0; r < n; ++r) topk_one(E, k, logits + r * E, idx + r * k, w + r * k);
    return 0;
}

/* Exported: step 5, the stable counting sort of the T*k slots by expert.
 * counts[E], offsets[E+1] (exclusive scan), perm[T*k] = slot id at sorted
 * position p, inv[T*k] = sorted position of slot id.  Returns -2 on an expert
 * index outside [0, E). */
int oracle_permute(int64_t T, int32_t E, int32_t k, const int32_t* idx, int32_t* counts,
                   int32_t* offsets, int32_t* perm, int32_t* inv)
{
    int64_t n = T * k;
    for (int32_t e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t q = 0; q < n; ++q) {
        if (idx[q] < 0 || idx[q] >= E) return -2;
        counts[idx[q]] += 1;
    }
    offsets[0] = 0;
    for (int32_t e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int32_t* fill = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
    if (!fill) return -3;
    for (int32_t e = 0; e < E; ++e) fill[e] = offsets[e];
    for (int64_t q = 0; q < n; ++q) {
        int32_t p = fill[idx[q]]++;
        perm[p] = (int32_t)q;
        inv[q] = p;
    }
    free(fill);
    return 0;
}

/* Exported: one expert FFN on one float64 hidden vector (used by the pins). */
int oracle_expert(int32_t H, int32_t I, const void* gate_up, const void* down, int32_t w_bf16,
                  const double* x, double* out)
{
    double* a = (double*)malloc(sizeof(double) * (size_t)I);
    if (!a) return -3;
    expert_ffn(H, I, gate_up, down, w_bf16, x, a, out);
    free(a);
    return 0;
}

/* Shared experts of one token added onto y (weight 1, no routed scale). */
static void add_shared(const oracle_shape* s, const void* sh_gate_up, const void* sh_down,
                       const double* xv, double* a, double* o, double* y)
{
    int64_t gu_stride = (int64_t)2 * s->I_shared * s->H, d_stride = (int64_t)s->H * s->I_shared;
    for (int32_t sh = 0; sh < s->n_shared; ++sh) {
        const void* gu = s->w_bf16 ? (const void*)((const uint16_t*)sh_gate_up + sh * gu_stride)
                                   : (const void*)((const float*)sh_gate_up + sh * gu_stride);
        const void* dn = s->w_bf16 ? (const void*)((const uint16_t*)sh_down + sh * d_stride)
                                   : (const void*)((const float*)sh_down + sh * d_stride);
        expert_ffn(s->H, s->I_shared, gu, dn, s->w_bf16, xv, a, o);
        for (int32_t h = 0; h < s->H; ++h) y[h] += o[h];
    }
}

static const void* expert_ptr(const void* base, int64_t e, int64_t stride, int bf16)
{
    return bf16 ? (const void*)((const uint16_t*)base + e * stride)
                : (const void*)((const float*)base + e * stride);
}

/* Exported: the sparse block (steps 1-4) for n tokens (tokens == NULL: 0..n-1).
 * y is [n, H] float64; idx_out [n, k] and w_out [n, k] may be NULL. */
int oracle_moe_block(const oracle_shape* s, const void* x, const float* wr, const float* b,
                     const void* gate_up, const void* down, const void* sh_gate_up,
                     const void* sh_down, const int64_t* tokens, int64_t n, double* y,
                     int32_t* idx_out, double* w_out)
{
    if (!shape_ok(s)) return -1;
    if (s->n_shared > 0 && (!sh_gate_up || !sh_down)) return -1;
    int64_t gu_stride = (int64_t)2 * s->I * s->H, d_stride = (int64_t)s->H * s->I;
    int32_t maxI = s->I > s->I_shared ? s->I : s->I_shared;
    int err = 0;
#pragma omp parallel
    {
        double* logits = (double*)malloc(sizeof(double) * (size_t)s->E);
        double* xv = (double*)malloc(sizeof(double) * (size_t)s->H);
        double* a = (double*)malloc(sizeof(double) * (size_t)maxI);
        double* o = (double*)malloc(sizeof(double) * (size_t)s->H);
        int32_t idx[1024];
        double w[1024];
        if (!logits || !xv || !a || !o) {
#pragma omp atomic write
            err = -3;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < n; ++r) {
                int64_t t = tokens ? tokens[r] : r;
                double* yr = y + r * s->H;
                router_one(s, x, t, wr, b, logits);
                topk_one(s->E, s->k, logits, idx, w);
                for (int32_t h = 0; h < s->H; ++h) {
                    xv[h] = widen(x, t * s->H + h, s->act_bf16);
                    yr[h] = 0.0;
                }
                for (int32_t j = 0; j < s->k; ++j) {
                    int64_t e = idx[j];
                    expert_ffn(s->H, s->I, expert_ptr(gate_up, e, gu_stride, s->w_bf16),
                               expert_ptr(down, e, d_stride, s->w_bf16), s->w_bf16, xv, a, o);
                    for (int32_t h = 0; h < s->H; ++h) yr[h] += s->routed_scale * w[j] * o[h];
                }
                add_shared(s, sh_gate_up, sh_down, xv, a, o, yr);
                for (int32_t j = 0; j < s->k; ++j) {
                    if (idx_out) idx_out[r * s->k + j] = idx[j];
                    if (w_out) w_out[r * s->k + j] = w[j];
                }
            }
        }
        free(logits); free(xv); free(a); free(o);
    }
    return err;
}

/* Exported: the same block by brute force, for all T tokens: every expert runs
 * on every token and its output is weighted by W[t][e], which is w_j when e is
 * the j-th selected expert of t and 0 otherwise.  This is the "standard MoE
 * with no token dropped" that the dropless sparse dispatch must equal. */
int oracle_moe_dense(const oracle_shape* s, const void* x, const float* wr, const float* b,
                     const void* gate_up, const void* down, const void* sh_gate_up,
                     const void* sh_down, double* y)
{
    if (!shape_ok(s)) return -1;
    if (s->n_shared > 0 && (!sh_gate_up || !sh_down)) return -1;
    int64_t gu_stride = (int64_t)2 * s->I * s->H, d_stride = (int64_t)s->H * s->I;
    int32_t maxI = s->I > s->I_shared ? s->I : s->I_shared;
    int err = 0;
#pragma omp parallel
    {
        double* logits = (double*)malloc(sizeof(double) * (size_t)s->E);
        double* dense_w = (double*)malloc(sizeof(double) * (size_t)s->E);
        double* xv = (double*)malloc(sizeof(double) * (size_t)s->H);
        double* a = (double*)malloc(sizeof(double) * (size_t)maxI);
        double* o = (double*)malloc(sizeof(double) * (size_t)s->H);
        int32_t idx[1024];
        double w[1024];
        if (!logits || !dense_w || !xv || !a || !o) {
#pragma omp atomic write
            err = -3;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t t = 0; t < s->T; ++t) {
                double* yr = y + t * s->H;
                router_one(s, x, t, wr, b, logits);
                topk_one(s->E, s->k, logits, idx, w);
                for (int32_t e = 0; e < s->E; ++e) dense_w[e] = 0.0;
                for (int32_t j = 0; j < s->k; ++j) dense_w[idx[j]] = w[j];
                for (int32_t h = 0; h < s->H; ++h) {
                    xv[h] = widen(x, t * s->H + h, s->act_bf16);
                    yr[h] = 0.0;
                }
                for (int64_t e = 0; e < s->E; ++e) {
                    expert_ffn(s->H, s->I, expert_ptr(gate_up, e, gu_stride, s->w_bf16),
                               expert_ptr(down, e, d_stride, s->w_bf16), s->w_bf16, xv, a, o);
                    for (int32_t h = 0; h < s->H; ++h)
                        yr[h] += s->routed_scale * dense_w[e] * o[h];
                }
                add_shared(s, sh_gate_up, sh_down, xv, a, o, yr);
            }
        }
        free(logits); free(dense_w); free(xv); free(a); free(o);
    }
    return err;
}

/* Exported: number of OpenMP threads a parallel region uses. */
int oracle_threads(void)
{
    int n = 1;
#pragma omp parallel
    {
#pragma omp single
        n = omp_get_num_threads();
    }
    return n;
}
