// The backward pass of the block around the expert GEMMs (gemm_sm100_bwd.cu).
//
// For the upstream gradient dy of y_t = s sum_j w_tj FFN_e(x_t) + shared(x_t)
// (routing: top-k with a softmax over the selected k, "PhiMoE in
// Transformers", section 6; routed scale and shared experts, Instella-MoE
// walk-through, FarSkipMoE), by the chain rule:
//   dO_p  = s w_p dy_t                 the output gradient of routed slot p
//   dw_p  = s <dy_t, FFN_e(x_t)>       the routing weight's (from the down
//                                      dgrad epilogue: <dh_p, a_p> / w_p)
//   dl_tj = w_tj (dw_tj - sum_i w_ti dw_ti)   softmax over the selected k; the
//                                      selection itself carries no gradient
//   + the load-balancing auxiliary loss ("PhiMoE in Transformers", section 6:
//     load_balancing_loss_func after Switch Transformer eqs. 4-6, times
//     router_aux_loss_coef): loss = coef E sum_e f_e P_e with f_e the tokens
//     dispatched to e over T and P_e the mean router probability;
//     dl_te += coef E / T p_te (f_e - sum_c p_tc f_c)
//   dWr   = dl^T x, db = sum_t dl_t, dx_t += dl_t Wr
//   dx_t  = sum_j dX_(t,j) + sum_s dX_shared(s,t) + dl_t Wr.
// Expert rows of the backward buffers are kept in the sorted order with each
// expert padded to a multiple of 128 rows (zero rows), which the weight
// gradient GEMMs need (see gemm_sm100_bwd.cu).
#include "common.cuh"

namespace moe {

constexpr int kBwdPad = 128;
constexpr int kBwdThreads = 256;
constexpr int kRouterTokens = 64;      // tokens per step of the router weight gradient

// poff[e] = sum over experts before e of round_up(count, 128).  One thread.
__global__ void pad_offsets_kernel(const int32_t* __restrict__ offsets,
                                   int32_t* __restrict__ poffsets, int E) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    int32_t acc = 0;
    poffsets[0] = 0;
    for (int e = 0; e < E; ++e) {
        const int32_t c = offsets[e + 1] - offsets[e];
        acc += (c + kBwdPad - 1) / kBwdPad * kBwdPad;
        poffsets[e + 1] = acc;
    }
}

// dO rows in the padded sorted order: row poff_e + m (m < count_e) is
// s * w(slot) * dy(token of the slot); the padding rows are zero.  One CTA
// per row (grid-stride), 16-byte vectors.
__global__ void __launch_bounds__(kBwdThreads) gather_scale_pad_kernel(
    const uint4* __restrict__ dy, const int32_t* __restrict__ offsets,
    const int32_t* __restrict__ poffsets, const int32_t* __restrict__ perm,
    const float* __restrict__ topk_w, uint4* __restrict__ dO, int E, int k, int vec_per_row,
    float routed_scale) {
    __shared__ int32_t offs[kMaxExperts + 1], poffs[kMaxExperts + 1];
    for (int e = threadIdx.x; e <= E; e += kBwdThreads) {
        offs[e] = offsets[e];
        poffs[e] = poffsets[e];
    }
    __syncthreads();
    const int64_t P = poffs[E];
    for (int64_t r = blockIdx.x; r < P; r += gridDim.x) {
        int lo = 0, hi = E - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (poffs[mid] <= r) lo = mid;
            else hi = mid - 1;
        }
        const int64_t m = r - poffs[lo];
        uint4* dst = dO + r * vec_per_row;
        if (m < offs[lo + 1] - offs[lo]) {
            const int32_t q = perm[offs[lo] + m];
            const float f = routed_scale * topk_w[q];
            const uint4* src = dy + static_cast<int64_t>(q / k) * vec_per_row;
            for (int v = threadIdx.x; v < vec_per_row; v += kBwdThreads) {
                const uint4 u = src[v];
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
                uint32_t o[4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    o[i] = pack_bf16x2(f * bf16_to_f32(static_cast<uint16_t>(w[i] & 0xffffu)),
                                       f * bf16_to_f32(static_cast<uint16_t>(w[i] >> 16)));
                dst[v] = make_uint4(o[0], o[1], o[2], o[3]);
            }
        } else {
            for (int v = threadIdx.x; v < vec_per_row; v += kBwdThreads)
                dst[v] = make_uint4(0, 0, 0, 0);
        }
    }
}

// Router backward, one warp per token: dw = dw_raw / w, dl over the selected
// experts, plus the auxiliary loss's term over all E when coef != 0 (logits
// and per-expert counts given).  Writes dl [T, E] and, when asked, dw [T, k]
// and the loss (added atomically: coef E sum_e f_e p_te / T per token).
__global__ void __launch_bounds__(kBwdThreads) router_backward_kernel(
    const float* __restrict__ dw_raw, const float* __restrict__ topk_w,
    const int32_t* __restrict__ topk_idx, const float* __restrict__ logits,
    const int32_t* __restrict__ counts, float* __restrict__ dl, float* __restrict__ dw_out,
    float* __restrict__ loss, int64_t T, int E, int k, float coef, int dw_tiles) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * (kBwdThreads / 32) + warp;
    if (t >= T) return;
    // selected experts: lane j < k
    float w = 0.f, dw = 0.f;
    int e_sel = -1;
    if (lane < k) {
        w = topk_w[t * k + lane];
        float raw = 0.f;
        for (int i = 0; i < dw_tiles; ++i) raw += dw_raw[(t * k + lane) * dw_tiles + i];
        dw = raw / w;
        e_sel = topk_idx[t * k + lane];
        if (dw_out) dw_out[t * k + lane] = dw;
    }
    float wdw = w * dw;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) wdw += __shfl_xor_sync(0xffffffffu, wdw, off);
    const float dl_sel = w * (dw - wdw);
    const bool aux = coef != 0.f && logits != nullptr && counts != nullptr;
    float mx = -3.402823466e38f, den = 0.f, pf = 0.f;
    const float invT = 1.f / static_cast<float>(T);
    if (aux) {
        for (int e = lane; e < E; e += 32) mx = fmaxf(mx, logits[t * E + e]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        for (int e = lane; e < E; e += 32) {
            const float pe = expf(logits[t * E + e] - mx);
            den += pe;
            pf += pe * static_cast<float>(counts[e]) * invT;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            den += __shfl_xor_sync(0xffffffffu, den, off);
            pf += __shfl_xor_sync(0xffffffffu, pf, off);
        }
        pf /= den;
        if (loss && lane == 0) atomicAdd(loss, coef * static_cast<float>(E) * pf * invT);
    }
    // every lane learns the k selected experts and their terms (all lanes
    // take part in each shuffle), then writes its experts' row entries
    int ej[kMaxK];
    float dj[kMaxK];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
        ej[j] = __shfl_sync(0xffffffffu, e_sel, j);
        dj[j] = __shfl_sync(0xffffffffu, dl_sel, j);
    }
    for (int e = lane; e < E; e += 32) {
        float g = 0.f;
        if (aux) {
            const float pe = expf(logits[t * E + e] - mx) / den;
            g = coef * static_cast<float>(E) * invT * pe *
                (static_cast<float>(counts[e]) * invT - pf);
        }
#pragma unroll
        for (int j = 0; j < kMaxK; ++j)
            if (j < k && ej[j] == e) g += dj[j];
        dl[t * E + e] = g;
    }
}

// Router weight gradient, first pass: part[c][e][h] = sum over the tokens of
// chunk c of dl[t][e] * x[t][h]; partb[c][e] = sum of dl[t][e].  Block (h
// chunk of 256, token chunk c); each thread owns one column h and EB experts
// at a time (EB accumulators, EB >= E where E <= 32).  Chunks are sized so
// that the grid holds several CTAs per SM (router_wgrad_tokens_per_chunk).
template <typename XT, int EB>
__global__ void __launch_bounds__(kBwdThreads) router_wgrad_partial_kernel(
    const XT* __restrict__ x, const float* __restrict__ dl, float* __restrict__ part,
    float* __restrict__ partb, int64_t T, int H, int E, int tokens_per_chunk) {
    __shared__ float dl_sh[kRouterTokens][EB + 1];
    const int h = blockIdx.x * kBwdThreads + threadIdx.x;
    const int c = blockIdx.y;
    const int64_t t0 = static_cast<int64_t>(c) * tokens_per_chunk;
    const int64_t t1 = t0 + tokens_per_chunk < T ? t0 + tokens_per_chunk : T;
    for (int e0 = 0; e0 < E; e0 += EB) {
        const int ne = E - e0 < EB ? E - e0 : EB;
        float acc[EB];
#pragma unroll
        for (int j = 0; j < EB; ++j) acc[j] = 0.f;
        float accb = 0.f;
        for (int64_t ts = t0; ts < t1; ts += kRouterTokens) {
            const int nt = t1 - ts < kRouterTokens ? static_cast<int>(t1 - ts) : kRouterTokens;
            __syncthreads();
            for (int i = threadIdx.x; i < kRouterTokens * EB; i += kBwdThreads) {
                const int tt = i / EB, j = i % EB;
                dl_sh[tt][j] = (tt < nt && j < ne) ? dl[(ts + tt) * E + e0 + j] : 0.f;
            }
            __syncthreads();
            if (threadIdx.x < EB && blockIdx.x == 0)
                for (int tt = 0; tt < nt; ++tt) accb += dl_sh[tt][threadIdx.x];
            if (h < H) {
                int tt = 0;
                // four token rows' loads in flight at a time
                for (; tt + 4 <= nt; tt += 4) {
                    float xv[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) xv[u] = ElemIO<XT>::load(x, (ts + tt + u) * H + h);
#pragma unroll
                    for (int u = 0; u < 4; ++u)
#pragma unroll
                        for (int j = 0; j < EB; ++j) acc[j] = fmaf(dl_sh[tt + u][j], xv[u], acc[j]);
                }
                for (; tt < nt; ++tt) {
                    const float xv = ElemIO<XT>::load(x, (ts + tt) * H + h);
#pragma unroll
                    for (int j = 0; j < EB; ++j) acc[j] = fmaf(dl_sh[tt][j], xv, acc[j]);
                }
            }
        }
        if (h < H)
            for (int j = 0; j < ne; ++j)
                part[(static_cast<int64_t>(c) * E + e0 + j) * H + h] = acc[j];
        if (threadIdx.x < ne && blockIdx.x == 0) partb[static_cast<int64_t>(c) * E + e0 + threadIdx.x] = accb;
    }
}

// Second pass: d_wr[e][h] = sum over chunks in order; d_b[e] likewise.
__global__ void __launch_bounds__(kBwdThreads) router_wgrad_reduce_kernel(
    const float* __restrict__ part, const float* __restrict__ partb, float* __restrict__ d_wr,
    float* __restrict__ d_b, int H, int E, int nchunks) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * kBwdThreads + threadIdx.x;
    const int64_t n = static_cast<int64_t>(E) * H;
    if (i < n) {
        float acc = 0.f;
        for (int c = 0; c < nchunks; ++c) acc += part[static_cast<int64_t>(c) * n + i];
        d_wr[i] = acc;
    }
    if (d_b && i < E) {
        float acc = 0.f;
        for (int c = 0; c < nchunks; ++c) acc += partb[static_cast<int64_t>(c) * E + i];
        d_b[i] = acc;
    }
}

// dx_t = sum_j dX[padded row of slot (t, j)] + sum_s dX_sh[s*T + t] + sum_e dl[t][e] Wr[e],
// float32 in that order, rounded once.  One CTA per token (grid-stride); each
// thread owns 8 consecutive columns.
__global__ void __launch_bounds__(kBwdThreads) dx_combine_kernel(
    const uint4* __restrict__ dX, const uint4* __restrict__ dX_sh, const int32_t* __restrict__ inv,
    const int32_t* __restrict__ topk_idx, const int32_t* __restrict__ offsets,
    const int32_t* __restrict__ poffsets, const float* __restrict__ dl,
    const float* __restrict__ w_router, uint4* __restrict__ dx, int64_t T, int H, int E, int k,
    int S) {
    __shared__ int64_t rows_sh[kMaxK];
    __shared__ float dl_sh[kMaxExperts];
    const int vpr = H / 8;
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        __syncthreads();
        if (threadIdx.x < k) {
            const int64_t q = t * k + threadIdx.x;
            const int e = topk_idx[q];
            rows_sh[threadIdx.x] = static_cast<int64_t>(inv[q]) - offsets[e] + poffsets[e];
        }
        for (int e = threadIdx.x; e < E; e += kBwdThreads) dl_sh[e] = dl[t * E + e];
        __syncthreads();
        for (int v = threadIdx.x; v < vpr; v += kBwdThreads) {
            float acc[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = 0.f;
            auto add_row = [&](const uint4 u) {
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    acc[2 * i] += bf16_to_f32(static_cast<uint16_t>(w[i] & 0xffffu));
                    acc[2 * i + 1] += bf16_to_f32(static_cast<uint16_t>(w[i] >> 16));
                }
            };
            for (int j = 0; j < k; ++j) add_row(dX[rows_sh[j] * vpr + v]);
            for (int s = 0; s < S; ++s) add_row(dX_sh[(static_cast<int64_t>(s) * T + t) * vpr + v]);
            for (int e = 0; e < E; ++e) {
                const float g = dl_sh[e];
                if (g == 0.f) continue;
                const float4* wr = reinterpret_cast<const float4*>(w_router + static_cast<int64_t>(e) * H) + 2 * v;
                const float4 a = wr[0], b = wr[1];
                acc[0] = fmaf(g, a.x, acc[0]); acc[1] = fmaf(g, a.y, acc[1]);
                acc[2] = fmaf(g, a.z, acc[2]); acc[3] = fmaf(g, a.w, acc[3]);
                acc[4] = fmaf(g, b.x, acc[4]); acc[5] = fmaf(g, b.y, acc[5]);
                acc[6] = fmaf(g, b.z, acc[6]); acc[7] = fmaf(g, b.w, acc[7]);
            }
            dx[t * vpr + v] = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                                         pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
        }
    }
}

cudaError_t launch_expert_backward(const moe_shape&, int64_t, const int32_t*, const int32_t*,
                                   const int32_t*, const void*, const void*, const void*,
                                   const void*, const void*, const void*, const void*, const void*,
                                   const void*, const void*, const void*, const void*, void*, void*,
                                   void*, void*, float*, float*, float*, float*, float*, int32_t*,
                                   int, cudaStream_t);

// n-tiles (256 columns of I) of the down-projection dgrad: the per-slot parts
// of the routing weight's gradient.
// routing-weight partials per slot: one per (256-column tile, half of it)
int backward_dw_tiles(const moe_shape& s) { return 2 * ((s.I + 255) / 256); }

size_t backward_pad_rows(const moe_shape& s) {
    return static_cast<size_t>(s.T * s.k) + static_cast<size_t>(kBwdPad - 1) * s.E;
}

// Tokens per chunk of the router weight gradient: enough chunks that the
// (H/256) x chunks grid holds about 600 CTAs, at least 64 tokens a chunk,
// and the float32 partials within 64 MB.
int router_wgrad_tokens_per_chunk(const moe_shape& s) {
    const int64_t hb = (s.H + kBwdThreads - 1) / kBwdThreads;
    int64_t chunks = (600 + hb - 1) / hb;
    const int64_t max_by_tokens = (s.T + kRouterTokens - 1) / kRouterTokens;
    const int64_t max_by_bytes = (64ll << 20) / (static_cast<int64_t>(s.E) * s.H * 4);
    if (chunks > max_by_tokens) chunks = max_by_tokens;
    if (chunks > max_by_bytes) chunks = max_by_bytes;
    if (chunks < 1) chunks = 1;
    int64_t per = (s.T + chunks - 1) / chunks;
    per = (per + kRouterTokens - 1) / kRouterTokens * kRouterTokens;
    return static_cast<int>(per > 0 ? per : kRouterTokens);
}

int router_wgrad_chunks(const moe_shape& s) {
    const int64_t per = router_wgrad_tokens_per_chunk(s);
    const int64_t n = (s.T + per - 1) / per;
    return static_cast<int>(n > 0 ? n : 1);
}

cudaError_t launch_backward(const moe_shape& s, const void* x, const float* w_router,
                            const int32_t* topk_idx, const float* topk_w, const int32_t* counts,
                            const int32_t* offsets, const int32_t* perm, const int32_t* inv,
                            const void* gate_up, const void* down, const void* sh_gate_up,
                            const void* sh_down, const void* gu, const void* gu_sh, const void* h,
                            const void* h_sh, const void* x_perm, const float* logits,
                            float aux_coef, const void* dy, void* dx, float* d_gate_up,
                            float* d_down, float* d_sh_gate_up, float* d_sh_down,
                            float* d_w_router, float* d_router_bias, float* d_topk_w,
                            float* aux_loss, const BackwardBuffers& b, int32_t* err_flag,
                            int num_sms, cudaStream_t st) {
    const int S = s.n_shared;
    cudaError_t e;
    pad_offsets_kernel<<<1, 32, 0, st>>>(offsets, b.poffsets, s.E);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int64_t P = static_cast<int64_t>(backward_pad_rows(s));
    const int grid_rows = static_cast<int>(P < int64_t(num_sms) * 8 ? P : int64_t(num_sms) * 8);
    gather_scale_pad_kernel<<<grid_rows, kBwdThreads, 0, st>>>(
        static_cast<const uint4*>(dy), offsets, b.poffsets, perm, topk_w,
        static_cast<uint4*>(b.dO), s.E, s.k, s.H / 8, s.routed_scale);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (aux_loss && (e = cudaMemsetAsync(aux_loss, 0, sizeof(float), st)) != cudaSuccess) return e;
    e = launch_expert_backward(s, P, offsets, b.poffsets, perm, x, dy, gate_up, down, sh_gate_up,
                               sh_down, gu, gu_sh, h, h_sh, x_perm, b.dO, b.dgu, b.dgu_sh, b.dO,
                               b.dX_sh, b.dw_raw, d_gate_up, d_down, d_sh_gate_up, d_sh_down,
                               err_flag, num_sms, st);
    if (e != cudaSuccess) return e;
    const unsigned tok_blocks = static_cast<unsigned>((s.T + kBwdThreads / 32 - 1) / (kBwdThreads / 32));
    router_backward_kernel<<<tok_blocks, kBwdThreads, 0, st>>>(
        b.dw_raw, topk_w, topk_idx, logits, counts, b.dl, d_topk_w, aux_loss, s.T, s.E, s.k,
        aux_coef, backward_dw_tiles(s));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int chunks = router_wgrad_chunks(s);
    const int tpc = router_wgrad_tokens_per_chunk(s);
    dim3 g1(static_cast<unsigned>((s.H + kBwdThreads - 1) / kBwdThreads), static_cast<unsigned>(chunks));
    if (s.dtype == MOE_BF16) {
        const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
        if (s.E <= 8)
            router_wgrad_partial_kernel<__nv_bfloat16, 8><<<g1, kBwdThreads, 0, st>>>(
                xb, b.dl, b.part, b.partb, s.T, s.H, s.E, tpc);
        else if (s.E <= 16)
            router_wgrad_partial_kernel<__nv_bfloat16, 16><<<g1, kBwdThreads, 0, st>>>(
                xb, b.dl, b.part, b.partb, s.T, s.H, s.E, tpc);
        else
            router_wgrad_partial_kernel<__nv_bfloat16, 32><<<g1, kBwdThreads, 0, st>>>(
                xb, b.dl, b.part, b.partb, s.T, s.H, s.E, tpc);
    } else {
        router_wgrad_partial_kernel<float, 32><<<g1, kBwdThreads, 0, st>>>(
            static_cast<const float*>(x), b.dl, b.part, b.partb, s.T, s.H, s.E, tpc);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int64_t n = static_cast<int64_t>(s.E) * s.H;
    router_wgrad_reduce_kernel<<<static_cast<unsigned>((n + kBwdThreads - 1) / kBwdThreads),
                                 kBwdThreads, 0, st>>>(b.part, b.partb, d_w_router, d_router_bias,
                                                       s.H, s.E, chunks);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int grid_t = static_cast<int>(s.T < int64_t(num_sms) * 8 ? s.T : int64_t(num_sms) * 8);
    dx_combine_kernel<<<grid_t, kBwdThreads, 0, st>>>(
        static_cast<const uint4*>(b.dO), static_cast<const uint4*>(b.dX_sh), inv, topk_idx,
        offsets, b.poffsets, b.dl, w_router, static_cast<uint4*>(dx), s.T, s.H, s.E, s.k, S);
    return cudaGetLastError();
}

}  // namespace moe
