// Router linear + top-k selection + softmax over the selected k, fused.
//
// "PhiMoE in Transformers (Phi-3.5-MoE)", section 6: the router is a bias-free
// nn.Linear hidden -> num_local_experts; in eval mode the experts are chosen
// greedily (top-1, mask it, take the next) and the chosen logits are soft-maxed.
// The optional per-expert bias is added to the logits before selection.
//
// One CTA of 8 warps handles 32 tokens; warp w owns tokens 4w..4w+3 and lane l
// owns experts l, l+32, ... (EPL per lane).  x and Wr are staged through shared
// memory in chunks of 128 hidden columns; each lane accumulates its 4 x EPL
// logits in float32, sequentially within a chunk, then chunk by chunk.  Selection runs as k rounds of a warp
// arg-max (ties to the lower expert index) over the register-resident logits.
#include "common.cuh"

namespace moe {

constexpr int kRouteTokens = 32;
constexpr int kRouteHC = 128;              // hidden columns per chunk
constexpr int kRouteLd = kRouteHC + 4;     // padded smem row (floats)

template <typename T, int EPL>
__global__ void __launch_bounds__(256) route_topk_kernel(
    const T* __restrict__ x, const float* __restrict__ wr, const float* __restrict__ bias,
    float* __restrict__ logits, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
    int64_t n_tokens, int H, int E, int k) {
    extern __shared__ float4 smem_f4[];
    float* xs = reinterpret_cast<float*>(smem_f4);          // [32][kRouteLd]
    float* ws = xs + kRouteTokens * kRouteLd;               // [32*EPL][kRouteLd]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t tok0 = static_cast<int64_t>(blockIdx.x) * kRouteTokens;
    const int n_exp_rows = 32 * EPL;

    float acc[4][EPL];
#pragma unroll
    for (int t = 0; t < 4; ++t)
#pragma unroll
        for (int j = 0; j < EPL; ++j) acc[t][j] = 0.f;

    for (int h0 = 0; h0 < H; h0 += kRouteHC) {
        const int hc = min(kRouteHC, H - h0);
        __syncthreads();
        for (int i = tid; i < kRouteTokens * kRouteHC; i += 256) {
            int r = i / kRouteHC, c = i % kRouteHC;
            int64_t tok = tok0 + r;
            float v = 0.f;
            if (tok < n_tokens && c < hc) v = ElemIO<T>::load(x, tok * H + h0 + c);
            xs[r * kRouteLd + c] = v;
        }
        for (int i = tid; i < n_exp_rows * kRouteHC; i += 256) {
            int r = i / kRouteHC, c = i % kRouteHC;
            float v = 0.f;
            if (r < E && c < hc) v = wr[static_cast<int64_t>(r) * H + h0 + c];
            ws[r * kRouteLd + c] = v;
        }
        __syncthreads();
        // per-chunk partial sums keep the float32 rounding error near
        // (sqrt(128) + sqrt(H/128)) ulp instead of sqrt(H) ulp
        float part[4][EPL];
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int j = 0; j < EPL; ++j) part[t][j] = 0.f;
        for (int c = 0; c < hc; c += 4) {
            float4 xv[4];
#pragma unroll
            for (int t = 0; t < 4; ++t)
                xv[t] = *reinterpret_cast<const float4*>(&xs[(warp * 4 + t) * kRouteLd + c]);
#pragma unroll
            for (int j = 0; j < EPL; ++j) {
                float4 wv = *reinterpret_cast<const float4*>(&ws[(lane + 32 * j) * kRouteLd + c]);
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    part[t][j] = fmaf(xv[t].x, wv.x, part[t][j]);
                    part[t][j] = fmaf(xv[t].y, wv.y, part[t][j]);
                    part[t][j] = fmaf(xv[t].z, wv.z, part[t][j]);
                    part[t][j] = fmaf(xv[t].w, wv.w, part[t][j]);
                }
            }
        }
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int j = 0; j < EPL; ++j) acc[t][j] += part[t][j];
    }

#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const int64_t tok = tok0 + warp * 4 + t;
        if (tok >= n_tokens) continue;   // warp-uniform
        float l[EPL];
        unsigned taken = 0;
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
            const int e = lane + 32 * j;
            l[j] = acc[t][j] + ((bias && e < E) ? bias[e] : 0.f);
            if (logits && e < E) logits[tok * E + e] = l[j];
        }
        float sel_v[kMaxK];
        int sel_e[kMaxK];
        for (int r = 0; r < k; ++r) {
            float best = -INFINITY;
            int best_e = 0x7fffffff;
#pragma unroll
            for (int j = 0; j < EPL; ++j) {
                const int e = lane + 32 * j;
                if (e < E && !(taken >> j & 1u) && (l[j] > best || best_e == 0x7fffffff)) {
                    best = l[j];
                    best_e = e;
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                float ov = __shfl_xor_sync(0xffffffffu, best, off);
                int oe = __shfl_xor_sync(0xffffffffu, best_e, off);
                if (ov > best || (ov == best && oe < best_e)) {
                    best = ov;
                    best_e = oe;
                }
            }
            if ((best_e & 31) == lane) taken |= 1u << (best_e >> 5);
            sel_v[r] = best;
            sel_e[r] = best_e;
        }
        if (lane == 0) {
            // softmax over the selected logits; sel_v[0] is their maximum
            float den = 0.f;
            for (int r = 0; r < k; ++r) den += expf(sel_v[r] - sel_v[0]);
            for (int r = 0; r < k; ++r) {
                topk_idx[tok * k + r] = sel_e[r];
                topk_w[tok * k + r] = expf(sel_v[r] - sel_v[0]) / den;
            }
        }
    }
}

// One warp: writes the token's logits lg[0..E) (if `logits`), then selects the
// top k (k rounds of a warp arg-max, ties to the lower expert index) and
// writes their indices and the softmax over the selected logits.
__device__ __forceinline__ void select_topk_warp(const float* lg, int E, int k, int64_t tok,
                                                 float* __restrict__ logits,
                                                 int32_t* __restrict__ topk_idx,
                                                 float* __restrict__ topk_w,
                                                 int32_t* sel_copy = nullptr) {
    const int lane = threadIdx.x & 31;
    if (logits)
        for (int e = lane; e < E; e += 32) logits[tok * E + e] = lg[e];
    float sel_v[kMaxK];
    int sel_e[kMaxK];
    for (int r = 0; r < k; ++r) {
        float best = -INFINITY;
        int best_e = 0x7fffffff;
        for (int e = lane; e < E; e += 32) {
            bool taken = false;
            for (int q = 0; q < r; ++q) taken |= (sel_e[q] == e);
            if (!taken && (lg[e] > best || best_e == 0x7fffffff)) {
                best = lg[e];
                best_e = e;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, best, off);
            const int oe = __shfl_xor_sync(0xffffffffu, best_e, off);
            if (ov > best || (ov == best && oe < best_e)) {
                best = ov;
                best_e = oe;
            }
        }
        sel_v[r] = best;
        sel_e[r] = best_e;
    }
    if (lane == 0) {
        float den = 0.f;
        for (int r = 0; r < k; ++r) den += expf(sel_v[r] - sel_v[0]);
        for (int r = 0; r < k; ++r) {
            topk_idx[tok * k + r] = sel_e[r];
            topk_w[tok * k + r] = expf(sel_v[r] - sel_v[0]) / den;
            if (sel_copy) sel_copy[r] = sel_e[r];   // (shared memory, for the plan)
        }
    }
}

// Few tokens (decode): one CTA per token, 8 warps over the experts.  The token
// row is staged in shared memory as float32; warp w computes the logits of
// experts w, w+8, ...: each lane reads 4 consecutive weights per step (16-byte
// loads, 8 steps unrolled so many loads are in flight), then the warp sums the
// lane partials with a butterfly.  Warp 0 then selects as above.
template <typename T>
__global__ void __launch_bounds__(256) route_small_kernel(
    const T* __restrict__ x, const float* __restrict__ wr, const float* __restrict__ bias,
    float* __restrict__ logits, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
    int H, int E, int k) {
    extern __shared__ float4 smem_f4[];
    float* xs = reinterpret_cast<float*>(smem_f4);     // [H]
    float* lg = xs + ((H + 3) & ~3);                   // [E]
    const int64_t tok = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int h = tid; h < H; h += 256) xs[h] = ElemIO<T>::load(x, tok * H + h);
    __syncthreads();
    const bool vec = (H % 4) == 0;
    for (int e = warp; e < E; e += 8) {
        const float* w = wr + static_cast<int64_t>(e) * H;
        float acc = 0.f;
        if (vec) {
            const int n4 = H >> 2;
            int i = lane;
            for (; i + 7 * 32 < n4; i += 8 * 32) {
                float4 wv[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) wv[u] = __ldg(reinterpret_cast<const float4*>(w) + i + u * 32);
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const float4 xv = *reinterpret_cast<const float4*>(&xs[4 * (i + u * 32)]);
                    acc = fmaf(wv[u].x, xv.x, acc);
                    acc = fmaf(wv[u].y, xv.y, acc);
                    acc = fmaf(wv[u].z, xv.z, acc);
                    acc = fmaf(wv[u].w, xv.w, acc);
                }
            }
            for (; i < n4; i += 32) {
                const float4 wv = __ldg(reinterpret_cast<const float4*>(w) + i);
                const float4 xv = *reinterpret_cast<const float4*>(&xs[4 * i]);
                acc = fmaf(wv.x, xv.x, acc);
                acc = fmaf(wv.y, xv.y, acc);
                acc = fmaf(wv.z, xv.z, acc);
                acc = fmaf(wv.w, xv.w, acc);
            }
        } else {
            for (int h = lane; h < H; h += 32) acc = fmaf(w[h], xs[h], acc);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) lg[e] = acc + (bias ? bias[e] : 0.f);
    }
    __syncthreads();
    if (warp != 0) return;
    select_topk_warp(lg, E, k, tok, logits, topk_idx, topk_w);
}

// Decode batches (at most kRouteClusterTokens tokens per cluster): a cluster
// of kRouteCluster CTAs per block of tokens, CTA r owning hidden columns
// [r HS, (r+1) HS).  Each CTA stages its slice of the tokens' rows and of the
// router weights in shared memory (16-byte cp.async, all in flight at once)
// and computes the partial logits of every (token, expert) over its slice
// (warp w: experts w, w+8, ...; one pass over a weight slice for all the
// block's tokens, lane partials summed by a butterfly).  TBM is the block's
// token capacity: 1 for a single token (no per-token guards), else
// kRouteClusterTokens.  After a cluster barrier, CTA 0 adds
// the kRouteCluster partials of each logit in rank order through distributed
// shared memory, adds the bias and selects as above; a second barrier keeps
// the other CTAs' shared memory alive until it has read it.  The router
// weights are read once per token block, spread over kRouteCluster SMs.
constexpr int kRouteCluster = 8;
constexpr int kRouteClusterTokens = 16;

// Volatile (kept in order with the cluster barriers) but without a memory
// clobber, so that a thread's loads are all in flight before their first use.
__device__ __forceinline__ float ld_shared_cluster_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ void cp_async16_route(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
                 : "memory");
}

template <typename T, int TBM>
__global__ void __launch_bounds__(256) route_cluster_kernel(
    const T* __restrict__ x, const float* __restrict__ wr, const float* __restrict__ bias,
    float* __restrict__ logits, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
    int32_t* __restrict__ counts, int32_t* __restrict__ offsets, int32_t* __restrict__ perm,
    int32_t* __restrict__ inv, int64_t n_tokens, int H, int E, int k, int HS, int stage_w,
    int vec_x) {
    extern __shared__ float4 smem_f4[];
    // the selected experts of the block's slots and the plan's counts and
    // offsets, when this launch also builds the dispatch plan (perm != NULL)
    __shared__ int32_t plan_idx[kRouteClusterTokens * kMaxK];
    __shared__ int32_t plan_cnt[kMaxExperts];
    __shared__ int32_t plan_off[kMaxExperts];
    float* part = reinterpret_cast<float*>(smem_f4);              // [TB][E] partial logits
    float* xs = part + ((kRouteClusterTokens * E + 3) & ~3);      // [TB][HS]
    float* ws = xs + kRouteClusterTokens * HS;                    // [E][HS] if stage_w
    // bf16 token rows as loaded, [TB][HS], when vec_x (float rows load into xs)
    T* xb = sizeof(T) == 4 ? reinterpret_cast<T*>(xs)
                           : reinterpret_cast<T*>(stage_w ? ws + E * HS : ws);
    const uint32_t rank = cluster_ctarank();
    const int64_t tok0 = static_cast<int64_t>(cluster_id_x()) * kRouteClusterTokens;
    const int tb = static_cast<int>(n_tokens - tok0 < kRouteClusterTokens ? n_tokens - tok0
                                                                          : kRouteClusterTokens);
    const int h0 = static_cast<int>(rank) * HS;
    const int hs = H - h0 < HS ? (H - h0 > 0 ? H - h0 : 0) : HS;   // columns of this slice
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // HS is a multiple of 4 and the slice starts on a 16-byte boundary of
    // each weight row when H % 4 == 0 (the launcher's condition)
    const int n4 = hs >> 2;
    // launched as a programmatic dependent: the router weights (written by
    // no kernel) start loading before pdl_wait, the token rows after it
    pdl_launch_dependents();
    if (stage_w) {
        // the slice of every router row, all in flight at once (one memory
        // latency instead of one per expert a warp handles)
        const int q = HS >> 2;
        for (int i = tid; i < E * q; i += 256) {
            const int e = i / q, c = i - e * q;
            if (c < n4) cp_async16_route(ws + e * HS + 4 * c, wr + static_cast<int64_t>(e) * H + h0 + 4 * c);
        }
    }
    pdl_wait();
    if (vec_x) {
        // the tokens' slices in 16-byte chunks, all in flight at once (H and
        // HS are multiples of the chunk, so the slice is whole chunks); the
        // columns past H read as zero
        constexpr int EPC = 16 / static_cast<int>(sizeof(T));
        const int cpr = HS / EPC, valid = hs / EPC;
        for (int i = tid; i < tb * cpr; i += 256) {
            const int t = i / cpr, c = i - t * cpr;
            T* dst = xb + t * HS + c * EPC;
            if (c < valid)
                cp_async16_route(dst, x + (tok0 + t) * H + h0 + c * EPC);
            else
                *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
        __syncthreads();
        if (sizeof(T) != 4)
            for (int i = tid; i < tb * HS; i += 256) xs[i] = ElemIO<T>::load(xb, i);
    } else {
        for (int i = tid; i < tb * HS; i += 256) {
            const int t = i / HS, h = i - t * HS;
            xs[i] = h < hs ? ElemIO<T>::load(x, (tok0 + t) * H + h0 + h) : 0.f;
        }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
    for (int e = warp; e < E; e += 8) {
        const float4* wg = reinterpret_cast<const float4*>(wr + static_cast<int64_t>(e) * H + h0);
        // (points into xs when the slice is not staged, so that even a
        // speculated load stays inside the allocation)
        const float4* wsv = reinterpret_cast<const float4*>(stage_w ? ws + e * HS : xs);
        // one pass over the expert's slice for all the block's tokens (a
        // weight chunk is read once and used tb times); per logit the lane
        // order of the products and the butterfly are those of one token
        float acc[TBM];
#pragma unroll
        for (int t = 0; t < TBM; ++t) acc[t] = 0.f;
        for (int i = lane; i < n4; i += 32) {
            const float4 a = stage_w ? wsv[i] : __ldg(wg + i);
#pragma unroll
            for (int t = 0; t < TBM; ++t) {
                if (TBM == 1 || t < tb) {
                    const float4 b = reinterpret_cast<const float4*>(xs + t * HS)[i];
                    acc[t] = fmaf(a.x, b.x, acc[t]);
                    acc[t] = fmaf(a.y, b.y, acc[t]);
                    acc[t] = fmaf(a.z, b.z, acc[t]);
                    acc[t] = fmaf(a.w, b.w, acc[t]);
                }
            }
        }
#pragma unroll
        for (int t = 0; t < TBM; ++t) {
            if (TBM == 1 || t < tb) {
                float v = acc[t];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
                if (lane == 0) part[t * E + e] = v;
            }
        }
    }
    cluster_sync();
    if (rank == 0) {
        // logits = sum of the ranks' partials in rank order (+ bias), kept in
        // this CTA's xs (no longer needed)
        float* lg = xs;
        const uint32_t base = smem_u32(part);
        for (int i = tid; i < tb * E; i += 256) {
            float pv[kRouteCluster];
#pragma unroll
            for (int r = 0; r < kRouteCluster; ++r)
                pv[r] = ld_shared_cluster_f32(mapa_shared(base + 4u * static_cast<uint32_t>(i),
                                                          static_cast<uint32_t>(r)));
            float v = 0.f;
#pragma unroll
            for (int r = 0; r < kRouteCluster; ++r) v += pv[r];
            lg[i] = v + (bias ? bias[i % E] : 0.f);
        }
        __syncthreads();
        for (int t = warp; t < tb; t += 8)
            select_topk_warp(lg + t * E, E, k, tok0 + t, logits, topk_idx, topk_w,
                             perm ? plan_idx + t * k : nullptr);
        if (perm) {
            // the one block holds every token: its dispatch plan as
            // moe_permute defines it (counts, their exclusive prefix sum,
            // slots in (expert, slot id) order), built here in one pass
            __syncthreads();
            const int n = tb * k;
            for (int e = tid; e < E; e += 256) {
                int c = 0;
                for (int q = 0; q < n; ++q) c += plan_idx[q] == e;
                plan_cnt[e] = c;
                counts[e] = c;
            }
            __syncthreads();
            if (warp == 0) {
                const int per = (E + 31) / 32;      // consecutive experts per lane
                int own = 0;
                for (int j = 0; j < per; ++j) {
                    const int e = lane * per + j;
                    if (e < E) own += plan_cnt[e];
                }
                int incl = own;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const int v = __shfl_up_sync(0xffffffffu, incl, off);
                    if (lane >= off) incl += v;
                }
                int run = incl - own;
                for (int j = 0; j < per; ++j) {
                    const int e = lane * per + j;
                    if (e < E) {
                        plan_off[e] = run;
                        offsets[e] = run;
                        run += plan_cnt[e];
                    }
                }
                if (lane == 31) offsets[E] = incl;
            }
            __syncthreads();
            for (int q = tid; q < n; q += 256) {
                const int e = plan_idx[q];
                int before = 0;
                for (int q2 = 0; q2 < q; ++q2) before += plan_idx[q2] == e;
                const int p = plan_off[e] + before;
                perm[p] = q;
                inv[q] = p;
            }
        }
    }
    cluster_sync();
}

// The cluster kernel when its shared memory fits (decode batches); returns
// cudaErrorNotSupported otherwise so that the caller takes route_small.  With
// `perm` non-NULL it also writes the dispatch plan (counts, offsets, perm,
// inv), which needs every token in one block: more than kRouteClusterTokens
// tokens return cudaErrorNotSupported.
cudaError_t launch_route_cluster(const moe_shape& s, const void* x, const float* wr,
                                 const float* bias, float* logits, int32_t* idx, float* w,
                                 int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv,
                                 cudaStream_t st) {
    if (s.H % 4 != 0 || s.T > 64 * kRouteClusterTokens) return cudaErrorNotSupported;
    if (perm && (s.T > kRouteClusterTokens || s.k > kMaxK || s.E > kMaxExperts))
        return cudaErrorNotSupported;
    // slices of whole 16-byte chunks of the token rows (8 bf16 or 4 floats)
    const int HS = ((s.H + kRouteCluster - 1) / kRouteCluster + 7) & ~7;
    size_t smem = sizeof(float) * (((kRouteClusterTokens * s.E + 3) & ~3) +
                                   static_cast<size_t>(kRouteClusterTokens) * HS);
    if (smem > 96 * 1024 || static_cast<size_t>(kRouteClusterTokens) * s.E >
                                static_cast<size_t>(kRouteClusterTokens) * HS)
        return cudaErrorNotSupported;
    // stage the router slice in shared memory too when it fits
    const size_t w_bytes = sizeof(float) * static_cast<size_t>(s.E) * HS;
    const int stage_w = smem + w_bytes <= 160 * 1024 ? 1 : 0;
    if (stage_w) smem += w_bytes;
    // bf16 rows load in 16-byte chunks into a staging area behind the slice
    // (float rows straight into theirs) when every row starts on 16 bytes
    const int vec_x = (reinterpret_cast<uintptr_t>(x) % 16 == 0) &&
                      (s.dtype == MOE_BF16 ? s.H % 8 == 0 : true);
    if (vec_x && s.dtype == MOE_BF16) smem += 2 * static_cast<size_t>(kRouteClusterTokens) * HS;
    const int blocks = static_cast<int>((s.T + kRouteClusterTokens - 1) / kRouteClusterTokens);
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(blocks * kRouteCluster));
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kRouteCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (s.dtype == MOE_BF16) {
        auto kern = s.T == 1 ? route_cluster_kernel<__nv_bfloat16, 1>
                             : route_cluster_kernel<__nv_bfloat16, kRouteClusterTokens>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        return cudaLaunchKernelEx(&cfg, kern, static_cast<const __nv_bfloat16*>(x), wr, bias, logits,
                                  idx, w, counts, offsets, perm, inv, static_cast<int64_t>(s.T),
                                  s.H, s.E, s.k, HS, stage_w, vec_x);
    }
    auto kern = s.T == 1 ? route_cluster_kernel<float, 1>
                         : route_cluster_kernel<float, kRouteClusterTokens>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<const float*>(x), wr, bias, logits, idx, w,
                              counts, offsets, perm, inv, static_cast<int64_t>(s.T), s.H, s.E, s.k,
                              HS, stage_w, vec_x);
}

cudaError_t launch_route_small(const moe_shape& s, const void* x, const float* wr,
                               const float* bias, float* logits, int32_t* idx, float* w,
                               cudaStream_t st) {
    const size_t smem = sizeof(float) * (((s.H + 3) & ~3) + s.E);
    if (smem > 200 * 1024) return cudaErrorInvalidValue;
    if (s.dtype == MOE_BF16) {
        auto kern = route_small_kernel<__nv_bfloat16>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        kern<<<static_cast<unsigned>(s.T), 256, smem, st>>>(
            static_cast<const __nv_bfloat16*>(x), wr, bias, logits, idx, w, s.H, s.E, s.k);
    } else {
        auto kern = route_small_kernel<float>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        kern<<<static_cast<unsigned>(s.T), 256, smem, st>>>(static_cast<const float*>(x), wr,
                                                            bias, logits, idx, w, s.H, s.E, s.k);
    }
    return cudaGetLastError();
}

template <typename T, int EPL>
static cudaError_t launch_route_t(const moe_shape& s, const void* x, const float* wr,
                                  const float* bias, float* logits, int32_t* idx, float* w,
                                  cudaStream_t st) {
    const size_t smem = sizeof(float) * (kRouteTokens + 32 * EPL) * kRouteLd;
    auto kern = route_topk_kernel<T, EPL>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    const int64_t blocks = (s.T + kRouteTokens - 1) / kRouteTokens;
    kern<<<static_cast<unsigned>(blocks), 256, smem, st>>>(static_cast<const T*>(x), wr, bias,
                                                           logits, idx, w, s.T, s.H, s.E, s.k);
    return cudaGetLastError();
}

cudaError_t launch_route(const moe_shape& s, const void* x, const float* wr, const float* bias,
                         float* logits, int32_t* idx, float* w, cudaStream_t st) {
    const bool bf = s.dtype == MOE_BF16;
    if (s.E <= 32)
        return bf ? launch_route_t<__nv_bfloat16, 1>(s, x, wr, bias, logits, idx, w, st)
                  : launch_route_t<float, 1>(s, x, wr, bias, logits, idx, w, st);
    if (s.E <= 64)
        return bf ? launch_route_t<__nv_bfloat16, 2>(s, x, wr, bias, logits, idx, w, st)
                  : launch_route_t<float, 2>(s, x, wr, bias, logits, idx, w, st);
    if (s.E <= 128)
        return bf ? launch_route_t<__nv_bfloat16, 4>(s, x, wr, bias, logits, idx, w, st)
                  : launch_route_t<float, 4>(s, x, wr, bias, logits, idx, w, st);
    return bf ? launch_route_t<__nv_bfloat16, 8>(s, x, wr, bias, logits, idx, w, st)
              : launch_route_t<float, 8>(s, x, wr, bias, logits, idx, w, st);
}

}  // namespace moe
