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

/* DeepSeek-V3 routing, "noaux_tc" (named by the Instella-MoE walk-through,
 * "config at a glance"; the pages do not define it, so this follows the
 * DeepSeek-V3 technical report, section 2.1: sigmoid affinities, a per-expert
 * bias that enters the selection only, node/group-limited routing, and gating
 * weights normalised over the selected affinities), for one token:
 *   1. s_e = 1 / (1 + exp(-l_e))                      affinity (l: bias-free logits)
 *   2. c_e = s_e + b_e                                 selection score
 *   3. the E experts form n_group contiguous groups of E / n_group; a group's
 *      score is the sum of its two largest c_e (its only one if a group has
 *      one expert); the topk_group groups with the largest scores are kept
 *      (greedy, ties to the lower group index);
 *   4. the k experts of the kept groups with the largest c_e, in descending
 *      order (ties to the lower expert index);
 *   5. w_j = s_(idx_j) / sum_i s_(idx_i).
 * The selection compares c and the group scores rounded to float32, the
 * precision in which the CUDA path takes the same decisions (the group score
 * is the float32 sum of two float32 values); the weights use float64. */
static void noaux_one(int32_t E, int32_t k, int32_t n_group, int32_t topk_group,
                      const double* logits, const float* bias, int32_t* idx, double* w)
{
    double aff[1024];
    float c[1024], gscore[1024];
    unsigned char gkeep[1024], taken[1024];
    int32_t gsize = E / n_group;
    for (int32_t e = 0; e < E; ++e) {
        aff[e] = 1.0 / (1.0 + exp(-logits[e]));
        c[e] = (float)(aff[e] + (bias ? (double)bias[e] : 0.0));
    }
    for (int32_t g = 0; g < n_group; ++g) {
        int32_t b1 = -1, b2 = -1;
        for (int32_t e = g * gsize; e < (g + 1) * gsize; ++e) {
            if (b1 < 0 || c[e] > c[b1]) { b2 = b1; b1 = e; }
            else if (b2 < 0 || c[e] > c[b2]) b2 = e;
        }
        gscore[g] = b2 < 0 ? c[b1] : (float)((double)c[b1] + (double)c[b2]);
        gkeep[g] = 0;
    }
    for (int32_t r = 0; r < topk_group; ++r) {
        int32_t best = -1;
        for (int32_t g = 0; g < n_group; ++g)
            if (!gkeep[g] && (best < 0 || gscore[g] > gscore[best])) best = g;
        gkeep[best] = 1;
    }
    memset(taken, 0, sizeof taken);
    for (int32_t j = 0; j < k; ++j) {
        int32_t best = -1;
        for (int32_t e = 0; e < E; ++e) {
            if (taken[e] || !gkeep[e / gsize]) continue;
            if (best < 0 || c[e] > c[best]) best = e;
        }
        taken[best] = 1;
        idx[j] = best;
    }
    double den = 0.0;
    for (int32_t j = 0; j < k; ++j) den += aff[idx[j]];
    for (int32_t j = 0; j < k; ++j) w[j] = aff[idx[j]] / den;
}

/* Exported: noaux_tc selection and weights for n rows of bias-free logits.
 * -1 unless E % n_group == 0, 1 <= topk_group <= n_group and
 * k <= topk_group * E / n_group. */
int oracle_route_noaux_tc(int64_t n, int32_t E, int32_t k, int32_t n_group, int32_t topk_group,
                          const double* logits, const float* bias, int32_t* idx, double* w)
{
    if (E <= 0 || E > 1024 || k <= 0 || n_group <= 0 || E % n_group != 0 || topk_group <= 0 ||
        topk_group > n_group || k > topk_group * (E / n_group))
        return -1;
    for (int64_t r = 0; r < n; ++r)
        noaux_one(E, k, n_group, topk_group, logits + r * E, bias, idx + r * k, w + r * k);
    return 0;
}

/* Exported: the block for n tokens given their routing (steps 3-4 with the
 * selection idx [n, k] and weights w [n, k] of each listed token row):
 * y_r = routed_scale * sum_j w_rj FFN_(idx_rj)(x_t) + the shared experts. */
int oracle_moe_block_routed(const oracle_shape* s, const void* x, const void* gate_up,
                            const void* down, const void* sh_gate_up, const void* sh_down,
                            const int64_t* tokens, int64_t n, const int32_t* idx,
                            const double* w, double* y)
{
    if (!shape_ok(s)) return -1;
    if (s->n_shared > 0 && (!sh_gate_up || !sh_down)) return -1;
    int64_t gu_stride = (int64_t)2 * s->I * s->H, d_stride = (int64_t)s->H * s->I;
    int32_t maxI = s->I > s->I_shared ? s->I : s->I_shared;
    int err = 0;
#pragma omp parallel
    {
        double* xv = (double*)malloc(sizeof(double) * (size_t)s->H);
        double* a = (double*)malloc(sizeof(double) * (size_t)maxI);
        double* o = (double*)malloc(sizeof(double) * (size_t)s->H);
        if (!xv || !a || !o) {
#pragma omp atomic write
            err = -3;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < n; ++r) {
                int64_t t = tokens ? tokens[r] : r;
                double* yr = y + r * s->H;
                for (int32_t h = 0; h < s->H; ++h) {
                    xv[h] = widen(x, t * s->H + h, s->act_bf16);
                    yr[h] = 0.0;
                }
                for (int32_t j = 0; j < s->k; ++j) {
                    int64_t e = idx[r * s->k + j];
                    if (e < 0 || e >= s->E) continue;
                    expert_ffn(s->H, s->I, expert_ptr(gate_up, e, gu_stride, s->w_bf16),
                               expert_ptr(down, e, d_stride, s->w_bf16), s->w_bf16, xv, a, o);
                    for (int32_t h = 0; h < s->H; ++h)
                        yr[h] += s->routed_scale * w[r * s->k + j] * o[h];
                }
                add_shared(s, sh_gate_up, sh_down, xv, a, o, yr);
            }
        }
        free(xv); free(a); free(o);
    }
    return err;
}

/* ------------------------------------------------------------------------
 * Backward pass.  For an upstream gradient dy[T, H] of the block output y,
 * by the chain rule through the forward steps above (float64 throughout):
 *   routed slot (t, j), expert e = idx_tj, weight w_j:
 *     g = Wg_e x_t, u = Wu_e x_t, a = SiLU(g) * u, f = Wd_e a
 *     dw_j   = s <dy_t, f>                        (y_t holds s * w_j * f)
 *     da     = s w_j Wd_e^T dy_t
 *     dWd_e += s w_j dy_t a^T
 *     dg     = da * u * SiLU'(g),  SiLU'(g) = sig(g) (1 + g (1 - sig(g)))
 *     du     = da * SiLU(g)
 *     dWg_e += dg x_t^T,  dWu_e += du x_t^T,  dx_t += Wg_e^T dg + Wu_e^T du
 *   shared expert: the same with weight 1 and no routing;
 *   router: the selection is piecewise constant, so only the k selected
 *     logits carry gradient, through the softmax over them:
 *     dl_j = w_j (dw_j - sum_i w_i dw_i); dWr[e] += dl_e x_t; db[e] += dl_e;
 *     dx_t += sum_e dl_e Wr[e].
 * The weight gradients are summed over all tokens (sequential in token
 * order); every output is float64. */
static double dsilu(double z)
{
    double sg = 1.0 / (1.0 + exp(-z));
    return sg * (1.0 + z * (1.0 - sg));
}

/* One expert's backward for one token: adds into dgu ([2I, H]) and dd
 * ([H, I]) and dx ([H]); scale = the factor on its output (s w_j, or 1). */
static void expert_bwd(int32_t H, int32_t I, const void* gate_up, const void* down, int w_bf16,
                       const double* x, const double* dy, double scale, double* g, double* u,
                       double* da, double* dgu, double* dd, double* dx)
{
    for (int32_t i = 0; i < I; ++i) {
        double gi = 0.0, ui = 0.0, di = 0.0;
        for (int32_t h = 0; h < H; ++h) {
            gi += widen(gate_up, (int64_t)i * H + h, w_bf16) * x[h];
            ui += widen(gate_up, (int64_t)(I + i) * H + h, w_bf16) * x[h];
        }
        for (int32_t h = 0; h < H; ++h) di += widen(down, (int64_t)h * I + i, w_bf16) * dy[h];
        g[i] = gi;
        u[i] = ui;
        da[i] = scale * di;
    }
    for (int32_t h = 0; h < H; ++h)
        for (int32_t i = 0; i < I; ++i) dd[(int64_t)h * I + i] += scale * dy[h] * silu(g[i]) * u[i];
    for (int32_t i = 0; i < I; ++i) {
        double dg = da[i] * u[i] * dsilu(g[i]);
        double du = da[i] * silu(g[i]);
        for (int32_t h = 0; h < H; ++h) {
            dgu[(int64_t)i * H + h] += dg * x[h];
            dgu[(int64_t)(I + i) * H + h] += du * x[h];
            dx[h] += widen(gate_up, (int64_t)i * H + h, w_bf16) * dg +
                     widen(gate_up, (int64_t)(I + i) * H + h, w_bf16) * du;
        }
    }
}

/* Exported: the block's gradients for all T tokens.
 *   dy [T, H] float64; outputs (float64, zeroed here):
 *   dx [T, H], d_gate_up [E, 2I, H], d_down [E, H, I], d_wr [E, H], d_b [E],
 *   d_sh_gate_up [S, 2Is, H] and d_sh_down [S, H, Is] (NULL when S == 0),
 *   dw [T, k] (the routing weights' gradient), dl [T, E] (the logits').
 * Single-threaded: the weight gradients sum over tokens in token order. */
int oracle_moe_backward(const oracle_shape* s, const void* x, const float* wr, const float* b,
                        const void* gate_up, const void* down, const void* sh_gate_up,
                        const void* sh_down, const double* dy, double* dx, double* d_gate_up,
                        double* d_down, double* d_wr, double* d_b, double* d_sh_gate_up,
                        double* d_sh_down, double* dw_out, double* dl_out)
{
    if (!shape_ok(s)) return -1;
    if (s->n_shared > 0 && (!sh_gate_up || !sh_down || !d_sh_gate_up || !d_sh_down)) return -1;
    const int64_t T = s->T;
    const int32_t H = s->H, I = s->I, E = s->E, k = s->k, S = s->n_shared, Is = s->I_shared;
    const int64_t gu_stride = (int64_t)2 * I * H, d_stride = (int64_t)H * I;
    const int64_t sgu_stride = (int64_t)2 * Is * H, sd_stride = (int64_t)H * Is;
    int32_t maxI = I > Is ? I : Is;
    memset(dx, 0, sizeof(double) * (size_t)(T * H));
    memset(d_gate_up, 0, sizeof(double) * (size_t)(E * gu_stride));
    memset(d_down, 0, sizeof(double) * (size_t)(E * d_stride));
    memset(d_wr, 0, sizeof(double) * (size_t)E * H);
    memset(d_b, 0, sizeof(double) * (size_t)E);
    if (S > 0) {
        memset(d_sh_gate_up, 0, sizeof(double) * (size_t)(S * sgu_stride));
        memset(d_sh_down, 0, sizeof(double) * (size_t)(S * sd_stride));
    }
    double* logits = (double*)malloc(sizeof(double) * (size_t)E);
    double* xv = (double*)malloc(sizeof(double) * (size_t)H);
    double* a = (double*)malloc(sizeof(double) * (size_t)maxI);
    double* o = (double*)malloc(sizeof(double) * (size_t)H);
    double* g = (double*)malloc(sizeof(double) * (size_t)maxI);
    double* u = (double*)malloc(sizeof(double) * (size_t)maxI);
    double* da = (double*)malloc(sizeof(double) * (size_t)maxI);
    int err = 0;
    if (!logits || !xv || !a || !o || !g || !u || !da) err = -3;
    for (int64_t t = 0; t < T && !err; ++t) {
        int32_t idx[1024];
        double w[1024], dw[1024];
        const double* dyt = dy + t * H;
        double* dxt = dx + t * H;
        router_one(s, x, t, wr, b, logits);
        topk_one(E, k, logits, idx, w);
        for (int32_t h = 0; h < H; ++h) xv[h] = widen(x, t * H + h, s->act_bf16);
        for (int32_t j = 0; j < k; ++j) {
            int64_t e = idx[j];
            const void* gu = expert_ptr(gate_up, e, gu_stride, s->w_bf16);
            const void* dn = expert_ptr(down, e, d_stride, s->w_bf16);
            expert_ffn(H, I, gu, dn, s->w_bf16, xv, a, o);
            double acc = 0.0;
            for (int32_t h = 0; h < H; ++h) acc += dyt[h] * o[h];
            dw[j] = s->routed_scale * acc;
            expert_bwd(H, I, gu, dn, s->w_bf16, xv, dyt, s->routed_scale * w[j], g, u, da,
                       d_gate_up + e * gu_stride, d_down + e * d_stride, dxt);
        }
        for (int32_t sh = 0; sh < S; ++sh)
            expert_bwd(H, Is, expert_ptr(sh_gate_up, sh, sgu_stride, s->w_bf16),
                       expert_ptr(sh_down, sh, sd_stride, s->w_bf16), s->w_bf16, xv, dyt, 1.0,
                       g, u, da, d_sh_gate_up + sh * sgu_stride, d_sh_down + sh * sd_stride, dxt);
        double wdw = 0.0;
        for (int32_t j = 0; j < k; ++j) wdw += w[j] * dw[j];
        if (dl_out)
            for (int32_t e = 0; e < E; ++e) dl_out[t * E + e] = 0.0;
        for (int32_t j = 0; j < k; ++j) {
            int64_t e = idx[j];
            double dl = w[j] * (dw[j] - wdw);
            if (dw_out) dw_out[t * k + j] = dw[j];
            if (dl_out) dl_out[t * E + e] = dl;
            d_b[e] += dl;
            for (int32_t h = 0; h < H; ++h) {
                d_wr[e * H + h] += dl * xv[h];
                dxt[h] += dl * (double)wr[e * H + h];
            }
        }
    }
    free(logits); free(xv); free(a); free(o); free(g); free(u); free(da);
    return err;
}

/* Exported: the load-balancing auxiliary loss the PhiMoE page attaches to the
 * router ("load_balancing_loss_func", Switch Transformer eqs. (4)-(6), times
 * router_aux_loss_coef), and its gradient with respect to the logits:
 *   p_t   = softmax over all E of the logits of token t
 *   P_e   = (1/T) sum_t p_te                   (router probability, eq. 6)
 *   f_e   = (1/T) #{(t, j): idx_tj = e}        (dispatch fraction, eq. 5, top-k)
 *   loss  = coef * E * sum_e f_e P_e           (eq. 4)
 *   dl_te = coef * E / T * p_te (f_e - sum_c p_tc f_c)   (f is piecewise constant)
 * logits [T, E] float64, idx [T, k]; dl [T, E] float64 output (may be NULL). */
int oracle_aux_loss(int64_t T, int32_t E, int32_t k, const double* logits, const int32_t* idx,
                    double coef, double* loss, double* dl)
{
    if (T <= 0 || E <= 0 || E > 1024 || k <= 0 || k > E) return -1;
    double f[1024], P[1024], p[1024];
    for (int32_t e = 0; e < E; ++e) { f[e] = 0.0; P[e] = 0.0; }
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t j = 0; j < k; ++j) {
            int32_t e = idx[t * k + j];
            if (e < 0 || e >= E) return -2;
            f[e] += 1.0;
        }
    }
    for (int32_t e = 0; e < E; ++e) f[e] /= (double)T;
    for (int64_t t = 0; t < T; ++t) {
        const double* l = logits + t * E;
        double mx = l[0], den = 0.0, pf = 0.0;
        for (int32_t e = 1; e < E; ++e) if (l[e] > mx) mx = l[e];
        for (int32_t e = 0; e < E; ++e) { p[e] = exp(l[e] - mx); den += p[e]; }
        for (int32_t e = 0; e < E; ++e) { p[e] /= den; P[e] += p[e]; pf += p[e] * f[e]; }
        if (dl)
            for (int32_t e = 0; e < E; ++e)
                dl[t * E + e] = coef * (double)E / (double)T * p[e] * (f[e] - pf);
    }
    double acc = 0.0;
    for (int32_t e = 0; e < E; ++e) acc += f[e] * (P[e] / (double)T);
    *loss = coef * (double)E * acc;
    return 0;
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
