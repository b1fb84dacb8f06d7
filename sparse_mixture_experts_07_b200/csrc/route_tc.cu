// Router on the tensor cores, with top-k and softmax fused into the epilogue.
//
// "PhiMoE in Transformers (Phi-3.5-MoE)", section 6: router = bias-free
// nn.Linear hidden -> num_local_experts, then greedy top-1 / mask / next and a
// softmax over the selected logits.  The per-expert bias joins the logits
// before selection.
//
// x is bf16; the router weight is float32.  Each float32 weight w is split
// into three bf16 terms, w = hi + mid + lo to within one float32 ulp (8 + 8 +
// 8 significant bits against float32's 24), so that one kind::f16 MMA over B = [hi; mid; lo]
// (3 E_PAD rows) with float32 accumulation yields x.hi, x.mid and x.lo, whose
// sum is the float32-weight logit.  x and the float32 weight tile of each
// k-block come in by TMA; the split into the bf16 B tile happens in shared
// memory (the weight is tiny and L2-resident).
//
// One CTA per 128 tokens, 5 warps: warp 0 streams the x tiles by TMA up to 5-6
// k-blocks ahead, warp 1 issues the MMAs (128 x N x 16, N = round_up(3 E_PAD,
// 16)), warps 2..4 split the staged weight tile of each k-block into the
// swizzled B tile.  In the epilogue thread t < 128 owns TMEM lane t = token m0+t: it sums
// its three partial logits per expert, adds the bias, and runs the k rounds
// of arg-max (ties to the lower index) and the softmax in registers.
#include "common.cuh"

namespace moe {

namespace rtc {
constexpr int BM = 128;
constexpr int BK = 64;
constexpr int CONVERTERS = 96;            // warps 2..4
constexpr int THREADS = 64 + CONVERTERS;  // + producer warp, MMA warp
constexpr int A_BYTES = BM * BK * 2;
}  // namespace rtc

template <int E_PAD>
struct RouteTcCfg {
    static constexpr int N = ((3 * E_PAD + 15) / 16) * 16;
    static constexpr int B_BYTES = N * rtc::BK * 2;
    static constexpr int W_BYTES = E_PAD * rtc::BK * 4;     // float32 weight tile (staging)
    static constexpr int STAGE_BYTES = rtc::A_BYTES + B_BYTES + W_BYTES;
    static constexpr int TMEM_COLS = N <= 32 ? 32 : N <= 64 ? 64 : N <= 128 ? 128 : 256;
    static constexpr int STAGES = (220 * 1024) / STAGE_BYTES < 6 ? (220 * 1024) / STAGE_BYTES : 6;
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
};

// Splits the staged float32 weight tile w32 [E_PAD][64] into the [hi; mid; lo; 0]
// bf16 B tile (128-byte swizzle: 16-byte chunk c of row r stored at chunk
// position c ^ (r & 7)).  Thread t handles chunks t, t + CONVERTERS, ...
template <int E_PAD>
__device__ __forceinline__ void split_weight_tile(uint8_t* sb, const float* w32, int t) {
    using C = RouteTcCfg<E_PAD>;
    for (int i = t; i < E_PAD * 8; i += rtc::CONVERTERS) {
        const int e = i >> 3, c = i & 7;
        const float4 u = *reinterpret_cast<const float4*>(w32 + e * rtc::BK + c * 8);
        const float4 v = *reinterpret_cast<const float4*>(w32 + e * rtc::BK + c * 8 + 4);
        const float a8[8] = {u.x, u.y, u.z, u.w, v.x, v.y, v.z, v.w};
        uint32_t hi[4], mid[4], lo[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float hv[2], mv[2], lv[2];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const float a = a8[2 * q + j];
                hv[j] = __bfloat162float(__float2bfloat16_rn(a));
                const float b = a - hv[j];                        // exact
                mv[j] = __bfloat162float(__float2bfloat16_rn(b));
                lv[j] = b - mv[j];   // exact; rounding it to bf16 below costs < 1 fp32 ulp of a
            }
            hi[q] = pack_bf16x2(hv[0], hv[1]);
            mid[q] = pack_bf16x2(mv[0], mv[1]);
            lo[q] = pack_bf16x2(lv[0], lv[1]);
        }
        const int r0 = e, r1 = E_PAD + e, r2 = 2 * E_PAD + e;
        *reinterpret_cast<uint4*>(sb + (r0 >> 3) * 1024 + (r0 & 7) * 128 + ((c ^ (r0 & 7)) << 4)) =
            make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(sb + (r1 >> 3) * 1024 + (r1 & 7) * 128 + ((c ^ (r1 & 7)) << 4)) =
            make_uint4(mid[0], mid[1], mid[2], mid[3]);
        *reinterpret_cast<uint4*>(sb + (r2 >> 3) * 1024 + (r2 & 7) * 128 + ((c ^ (r2 & 7)) << 4)) =
            make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
    for (int i = t; i < (C::N - 3 * E_PAD) * 8; i += rtc::CONVERTERS) {
        const int r = 3 * E_PAD + (i >> 3), c = i & 7;
        *reinterpret_cast<uint4*>(sb + (r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4)) =
            make_uint4(0u, 0u, 0u, 0u);
    }
}

// Epilogue pieces of the tensor-core routers.  The calling thread owns one
// token, whose TMEM lane holds x.hi, x.mid and x.lo for every expert (columns
// [0,E_PAD), [E_PAD,2E_PAD), [2E_PAD,3E_PAD)).
//
// lg[e] += hi, then mid, then lo (column order).  Every lane of the warp must
// call it (tcgen05.ld is warp-wide).
template <int E_PAD>
__device__ __forceinline__ void add_tmem_terms(uint32_t lane_addr, float (&lg)[E_PAD]) {
    constexpr int NCH = (3 * E_PAD + 31) / 32;
#pragma unroll
    for (int ch = 0; ch < NCH; ++ch) {
        float v[32];
        tmem_ld32(lane_addr + ch * 32, v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int col = ch * 32 + j;
            if (col < 3 * E_PAD) lg[col % E_PAD] += v[j];
        }
    }
}

// Writes the float32 logits (if requested), then the k rounds of arg-max (ties
// to the lower index) and the softmax over the selected logits of token `tok`.
template <int E_PAD>
__device__ __forceinline__ void select_topk(const float (&lg)[E_PAD], int64_t tok, int E, int k,
                                            float* __restrict__ logits,
                                            int32_t* __restrict__ topk_idx,
                                            float* __restrict__ topk_w) {
    if (logits) {
#pragma unroll
        for (int e = 0; e < E_PAD; ++e)
            if (e < E) logits[tok * E + e] = lg[e];
    }
    uint32_t taken[(E_PAD + 31) / 32];
#pragma unroll
    for (int q = 0; q < (E_PAD + 31) / 32; ++q) taken[q] = 0u;
    float sel0 = 0.f, den = 0.f;
    float sel_v[kMaxK];
    for (int r = 0; r < k; ++r) {
        int best = -1;
        float bv = 0.f;
#pragma unroll
        for (int e = 0; e < E_PAD; ++e) {
            if (e < E && !((taken[e >> 5] >> (e & 31)) & 1u) && (best < 0 || lg[e] > bv)) {
                best = e;
                bv = lg[e];
            }
        }
        taken[best >> 5] |= 1u << (best & 31);
        if (r == 0) sel0 = bv;
        sel_v[r] = bv;
        topk_idx[tok * k + r] = best;
        den += expf(bv - sel0);
    }
    for (int r = 0; r < k; ++r) topk_w[tok * k + r] = expf(sel_v[r] - sel0) / den;
}

// logit = ((bias + hi) + mid) + lo, then the selection.
template <int E_PAD>
__device__ __forceinline__ void topk_epilogue(uint32_t lane_addr, int64_t tok, bool ok,
                                              const float* __restrict__ bias,
                                              float* __restrict__ logits,
                                              int32_t* __restrict__ topk_idx,
                                              float* __restrict__ topk_w, int64_t n_tokens, int E,
                                              int k) {
    float lg[E_PAD];
#pragma unroll
    for (int e = 0; e < E_PAD; ++e) lg[e] = (bias && e < E) ? bias[e] : 0.f;
    add_tmem_terms<E_PAD>(lane_addr, lg);
    if (tok < n_tokens && ok) select_topk<E_PAD>(lg, tok, E, k, logits, topk_idx, topk_w);
}

template <int E_PAD>
__global__ void __launch_bounds__(rtc::THREADS, 1) route_tc_kernel(
    const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
    const float* __restrict__ bias, float* __restrict__ logits, int32_t* __restrict__ topk_idx,
    float* __restrict__ topk_w, int64_t n_tokens, int H, int E, int k, int32_t* err_flag,
    uint64_t timeout_ns) {
    using C = RouteTcCfg<E_PAD>;
    using namespace rtc;
    constexpr int STAGES = C::STAGES;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ uint32_t tmem_base_sh;
    __shared__ int fail_sh;
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * C::STAGE_BYTES);
    uint64_t* full = bars;                  // TMA of A landed                 [STAGES]
    uint64_t* bready = bars + STAGES;       // B tile written (CONVERTERS arr.) [STAGES]
    uint64_t* empty = bars + 2 * STAGES;    // MMAs of the stage done          [STAGES]
    uint64_t* done = bars + 3 * STAGES;     // all MMAs done                   [1]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t m0 = static_cast<int64_t>(blockIdx.x) * BM;
    const uint64_t deadline = global_ns() + timeout_ns;

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&bready[s], CONVERTERS);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
        fail_sh = 0;
        fence_barrier_init();
        tma_prefetch_desc(&map_x);
        tma_prefetch_desc(&map_w);
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base_sh, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;
    const int nkb = (H + BK - 1) / BK;

    if (warp == 0) {
        // ---- producer: x tiles, running up to STAGES k-blocks ahead
        if (lane == 0) {
            for (int kb = 0; kb < nkb; ++kb) {
                const int s = kb % STAGES;
                const uint32_t ph = static_cast<uint32_t>(kb / STAGES) & 1u;
                if (!mbar_wait(&empty[s], ph ^ 1u, deadline)) { atomicExch(&fail_sh, 1); break; }
                uint8_t* st = smem + s * C::STAGE_BYTES;
                mbar_arrive_expect_tx(&full[s], A_BYTES + C::W_BYTES);
                tma_load_2d(st, &map_x, &full[s], kb * BK, static_cast<int32_t>(m0));
                tma_load_2d(st + A_BYTES + C::B_BYTES, &map_w, &full[s], kb * BK, 0);
            }
        }
    } else if (warp == 1) {
        // ---- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(BM, C::N);
            for (int kb = 0; kb < nkb; ++kb) {
                const int s = kb % STAGES;
                const uint32_t ph = static_cast<uint32_t>(kb / STAGES) & 1u;
                if (!mbar_wait(&full[s], ph, deadline) || !mbar_wait(&bready[s], ph, deadline)) {
                    atomicExch(&fail_sh, 1);
                    break;
                }
                tc_fence_after();
                const uint32_t a0 = smem_u32(smem + s * C::STAGE_BYTES), b0 = a0 + A_BYTES;
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk)
                    umma_bf16(tmem, smem_desc_sw128(a0 + kk * 32), smem_desc_sw128(b0 + kk * 32),
                              idesc, (kb | kk) != 0 ? 1u : 0u);
                umma_commit(&empty[s]);
            }
            umma_commit(done);
        }
    } else {
        // ---- converters: the B tile of each k-block
        // split each staged float32 weight tile once its TMA has landed (the
        // producer only issues it after the stage was released by the MMA)
        const int t = tid - 64;
        for (int kb = 0; kb < nkb; ++kb) {
            const int s = kb % STAGES;
            const uint32_t ph = static_cast<uint32_t>(kb / STAGES) & 1u;
            if (!mbar_wait(&full[s], ph, deadline)) { atomicExch(&fail_sh, 1); break; }
            uint8_t* st = smem + s * C::STAGE_BYTES;
            split_weight_tile<E_PAD>(st + A_BYTES,
                                     reinterpret_cast<const float*>(st + A_BYTES + C::B_BYTES), t);
            fence_proxy_async_smem();   // generic-proxy writes -> visible to the MMA
            mbar_arrive(&bready[s]);
        }
    }

    bool ok = mbar_wait(done, 0, deadline + 1000000000ull);
    __syncthreads();
    ok = ok && fail_sh == 0;
    if (tid == 0 && !ok) raise_error(err_flag, MOE_ERR_TIMEOUT);
    tc_fence_after();

    // ---- epilogue (warps 0..3): thread tid owns token m0 + tid (TMEM lane tid)
    if (warp < 4)
        topk_epilogue<E_PAD>(tmem + (static_cast<uint32_t>(warp * 32) << 16), m0 + tid, ok, bias,
                             logits, topk_idx, topk_w, n_tokens, E, k);

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// Router with the weight split ahead of time.  The split of the float32
// weight into its three bf16 terms depends on the weight only, so it can be
// done once when the weights are loaded ("Mixture of Experts in
// Transformers", WeightConverter section: conversions run in the
// weight-loading pipeline) instead of in every CTA of every call.

// w_split [N][H] bf16: row e < E_PAD is hi(W[e]), row E_PAD + e is mid(W[e]),
// row 2 E_PAD + e is lo(W[e]) (zero for e >= E), rows >= 3 E_PAD are zero.
// One thread per (row, 8 consecutive columns); H % 8 == 0.
__global__ void __launch_bounds__(256) router_split_kernel(const float* __restrict__ w,
                                                           uint4* __restrict__ out, int E,
                                                           int E_PAD, int N, int H) {
    const int chunks = H / 8;
    const int64_t total = static_cast<int64_t>(N) * chunks;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * 256) {
        const int r = static_cast<int>(i / chunks);
        const int c = static_cast<int>(i - static_cast<int64_t>(r) * chunks);
        const int term = r / E_PAD, e = r - term * E_PAD;
        uint32_t packed[4] = {0u, 0u, 0u, 0u};
        if (term < 3 && e < E) {
            const float4 u = *reinterpret_cast<const float4*>(w + static_cast<int64_t>(e) * H + c * 8);
            const float4 v =
                *reinterpret_cast<const float4*>(w + static_cast<int64_t>(e) * H + c * 8 + 4);
            const float a8[8] = {u.x, u.y, u.z, u.w, v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float t2[2];
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const float a = a8[2 * q + j];
                    const float hi = __bfloat162float(__float2bfloat16_rn(a));
                    const float b = a - hi;                                  // exact
                    const float mid = __bfloat162float(__float2bfloat16_rn(b));
                    t2[j] = term == 0 ? hi : term == 1 ? mid : b - mid;      // b - mid exact
                }
                packed[q] = pack_bf16x2(t2[0], t2[1]);
            }
        }
        out[i] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    }
}

namespace rts {
constexpr int THREADS = 128;   // warp 0 TMA, warp 1 MMA; all four run the epilogue
}

template <int E_PAD>
struct RouteSplitCfg {
    static constexpr int N = RouteTcCfg<E_PAD>::N;
    static constexpr int B_BYTES = N * rtc::BK * 2;
    static constexpr int STAGE_BYTES = rtc::A_BYTES + B_BYTES;
    static constexpr int TMEM_COLS = RouteTcCfg<E_PAD>::TMEM_COLS;
    static constexpr int STAGES = (200 * 1024) / STAGE_BYTES < 8 ? (200 * 1024) / STAGE_BYTES : 8;
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
};

// A cluster of `ks` CTAs per 128 tokens, CTA c of the cluster taking the c-th
// of ks contiguous slices of the k-blocks (split-K, so that few tokens still
// keep many SMs streaming x).  In each CTA warp 0 streams the x tile and the
// split-weight tile of each k-block by TMA, STAGES k-blocks ahead, and warp 1
// issues 128 x N x 16 MMAs.  Thread t < 128 then owns token m0 + t:
//   ks == 1: logit = ((bias + hi) + mid) + lo (topk_epilogue);
//   ks > 1:  each CTA forms its partial (hi + mid) + lo, CTAs 1..ks-1 store
//            theirs into CTA 0's shared memory, and CTA 0 sums
//            bias + p_0 + p_1 + ... in rank order, then selects.
template <int E_PAD>
__global__ void __launch_bounds__(rts::THREADS, 1) route_tc_split_kernel(
    const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_ws,
    const float* __restrict__ bias, float* __restrict__ logits, int32_t* __restrict__ topk_idx,
    float* __restrict__ topk_w, int64_t n_tokens, int H, int E, int k, int ks, int32_t* err_flag,
    uint64_t timeout_ns) {
    using C = RouteSplitCfg<E_PAD>;
    using namespace rtc;
    constexpr int STAGES = C::STAGES;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ uint32_t tmem_base_sh;
    __shared__ int fail_sh;
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * C::STAGE_BYTES);
    uint64_t* full = bars;                  // x and weight tiles landed  [STAGES]
    uint64_t* empty = bars + STAGES;        // MMAs of the stage done     [STAGES]
    uint64_t* done = bars + 2 * STAGES;     // all MMAs done              [1]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int slice = ks > 1 ? static_cast<int>(cluster_ctarank()) : 0;
    const int64_t m0 = static_cast<int64_t>(blockIdx.x / ks) * BM;
    const uint64_t deadline = global_ns() + timeout_ns;

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
        fail_sh = 0;
        fence_barrier_init();
        tma_prefetch_desc(&map_x);
        tma_prefetch_desc(&map_ws);
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base_sh, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;
    // this CTA's k-blocks [kb0, kb1); the host makes every slice non-empty
    const int nkb_all = (H + BK - 1) / BK;
    const int kb0 = slice * nkb_all / ks, kb1 = (slice + 1) * nkb_all / ks;
    const int nkb = kb1 - kb0;

    if (warp == 0 && lane == 0) {
        for (int i = 0; i < nkb; ++i) {
            const int s = i % STAGES;
            const uint32_t ph = static_cast<uint32_t>(i / STAGES) & 1u;
            if (!mbar_wait(&empty[s], ph ^ 1u, deadline)) { atomicExch(&fail_sh, 1); break; }
            uint8_t* st = smem + s * C::STAGE_BYTES;
            mbar_arrive_expect_tx(&full[s], C::STAGE_BYTES);
            tma_load_2d(st, &map_x, &full[s], (kb0 + i) * BK, static_cast<int32_t>(m0));
            tma_load_2d(st + A_BYTES, &map_ws, &full[s], (kb0 + i) * BK, 0);
        }
    } else if (warp == 1 && lane == 0) {
        constexpr uint32_t idesc = idesc_bf16_f32(BM, C::N);
        for (int i = 0; i < nkb; ++i) {
            const int s = i % STAGES;
            const uint32_t ph = static_cast<uint32_t>(i / STAGES) & 1u;
            if (!mbar_wait(&full[s], ph, deadline)) { atomicExch(&fail_sh, 1); break; }
            tc_fence_after();
            const uint32_t a0 = smem_u32(smem + s * C::STAGE_BYTES), b0 = a0 + A_BYTES;
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
                umma_bf16(tmem, smem_desc_sw128(a0 + kk * 32), smem_desc_sw128(b0 + kk * 32), idesc,
                          (i | kk) != 0 ? 1u : 0u);
            umma_commit(&empty[s]);
        }
        umma_commit(done);
    }
    __syncwarp();

    bool ok = mbar_wait(done, 0, deadline + 1000000000ull);
    __syncthreads();
    ok = ok && fail_sh == 0;
    if (tid == 0 && !ok) raise_error(err_flag, MOE_ERR_TIMEOUT);
    tc_fence_after();
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    if (ks == 1) {
        topk_epilogue<E_PAD>(lane_addr, m0 + tid, ok, bias, logits, topk_idx, topk_w, n_tokens,
                             E, k);
    } else {
        float part[E_PAD];
#pragma unroll
        for (int e = 0; e < E_PAD; ++e) part[e] = 0.f;
        add_tmem_terms<E_PAD>(lane_addr, part);          // (hi + mid) + lo
        // all MMAs of the cluster are complete: CTA 0's stage buffers are free
        cluster_sync();
        // partials of CTA c >= 1 at float offset ((c - 1) E_PAD + e) * 128 + t of
        // CTA 0's first stage buffers (consecutive threads, consecutive words)
        float* red = reinterpret_cast<float*>(smem);
        if (slice > 0) {
            const uint32_t dst = mapa_shared(smem_u32(red), 0) +
                                 static_cast<uint32_t>(((slice - 1) * E_PAD * BM + tid) * 4);
#pragma unroll
            for (int e = 0; e < E_PAD; ++e)
                asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(dst + e * BM * 4),
                             "f"(part[e])
                             : "memory");
        }
        cluster_sync();
        if (slice == 0) {
            const int64_t tok = m0 + tid;
            float lg[E_PAD];
#pragma unroll
            for (int e = 0; e < E_PAD; ++e) lg[e] = ((bias && e < E) ? bias[e] : 0.f) + part[e];
            for (int c = 1; c < ks; ++c) {
#pragma unroll
                for (int e = 0; e < E_PAD; ++e) lg[e] += red[((c - 1) * E_PAD + e) * BM + tid];
            }
            if (tok < n_tokens && ok) select_topk<E_PAD>(lg, tok, E, k, logits, topk_idx, topk_w);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

typedef CUresult (*EncodeTiledFnR)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFnR route_encode_fn() {
    static EncodeTiledFnR fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFnR>(ptr);
    }
    return fn;
}

template <int E_PAD>
static cudaError_t launch_route_tc_t(const moe_shape& s, const void* x, const float* wr,
                                     const float* bias, float* logits, int32_t* idx, float* w,
                                     int32_t* err_flag, cudaStream_t st) {
    using C = RouteTcCfg<E_PAD>;
    EncodeTiledFnR enc = route_encode_fn();
    if (!enc) return cudaErrorInvalidValue;
    CUtensorMap map;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(s.H), static_cast<cuuint64_t>(s.T)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(s.H) * 2};
    cuuint32_t box[2] = {rtc::BK, rtc::BM};
    cuuint32_t estr[2] = {1, 1};
    if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    CUtensorMap map_w;
    cuuint64_t wdims[2] = {static_cast<cuuint64_t>(s.H), static_cast<cuuint64_t>(s.E)};
    cuuint64_t wstrides[1] = {static_cast<cuuint64_t>(s.H) * 4};
    cuuint32_t wbox[2] = {rtc::BK, static_cast<cuuint32_t>(E_PAD)};
    if (enc(&map_w, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(wr), wdims, wstrides,
            wbox, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    auto kern = route_tc_kernel<E_PAD>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const unsigned grid = static_cast<unsigned>((s.T + rtc::BM - 1) / rtc::BM);
    kern<<<grid, rtc::THREADS, C::SMEM_BYTES, st>>>(map, map_w, bias, logits, idx, w, s.T, s.H, s.E,
                                                    s.k, err_flag, 4000000000ull);
    return cudaGetLastError();
}

// Tensor-core router for bf16 activations and E <= 64.
cudaError_t launch_route_tc(const moe_shape& s, const void* x, const float* wr, const float* bias,
                            float* logits, int32_t* idx, float* w, int32_t* err_flag,
                            cudaStream_t st) {
    if (s.E <= 8) return launch_route_tc_t<8>(s, x, wr, bias, logits, idx, w, err_flag, st);
    if (s.E <= 16) return launch_route_tc_t<16>(s, x, wr, bias, logits, idx, w, err_flag, st);
    if (s.E <= 32) return launch_route_tc_t<32>(s, x, wr, bias, logits, idx, w, err_flag, st);
    return launch_route_tc_t<64>(s, x, wr, bias, logits, idx, w, err_flag, st);
}

// Rows of the split router weight for E experts (0 when the tensor-core
// router does not apply).
int router_split_rows(const moe_shape& s) {
    if (s.dtype != MOE_BF16 || s.E > 64) return 0;
    if (s.E <= 8) return RouteTcCfg<8>::N;
    if (s.E <= 16) return RouteTcCfg<16>::N;
    if (s.E <= 32) return RouteTcCfg<32>::N;
    return RouteTcCfg<64>::N;
}

static int router_e_pad(int E) { return E <= 8 ? 8 : E <= 16 ? 16 : E <= 32 ? 32 : 64; }

cudaError_t launch_router_split(const moe_shape& s, const float* wr, void* w_split, int num_sms,
                                cudaStream_t st) {
    const int N = router_split_rows(s);
    const int64_t total = static_cast<int64_t>(N) * (s.H / 8);
    int64_t grid = (total + 255) / 256;
    if (grid > static_cast<int64_t>(num_sms) * 8) grid = static_cast<int64_t>(num_sms) * 8;
    if (grid < 1) return cudaSuccess;
    router_split_kernel<<<static_cast<unsigned>(grid), 256, 0, st>>>(
        wr, static_cast<uint4*>(w_split), s.E, router_e_pad(s.E), N, s.H);
    return cudaGetLastError();
}

template <int E_PAD>
static cudaError_t launch_route_tc_split_t(const moe_shape& s, const void* x, const void* w_split,
                                           const float* bias, float* logits, int32_t* idx,
                                           float* w, int32_t* err_flag, int num_sms,
                                           cudaStream_t st) {
    using C = RouteSplitCfg<E_PAD>;
    EncodeTiledFnR enc = route_encode_fn();
    if (!enc) return cudaErrorInvalidValue;
    CUtensorMap map, map_ws;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(s.H), static_cast<cuuint64_t>(s.T)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(s.H) * 2};
    cuuint32_t box[2] = {rtc::BK, rtc::BM};
    cuuint32_t estr[2] = {1, 1};
    if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    cuuint64_t wdims[2] = {static_cast<cuuint64_t>(s.H), static_cast<cuuint64_t>(C::N)};
    cuuint32_t wbox[2] = {rtc::BK, static_cast<cuuint32_t>(C::N)};
    if (enc(&map_ws, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(w_split), wdims,
            strides, wbox, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    auto kern = route_tc_split_kernel<E_PAD>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    // split K over a cluster of ks CTAs while the m-tiles alone leave SMs idle;
    // each slice keeps >= 4 k-blocks and CTA 0's stage buffers hold the
    // partials of the other ks - 1 CTAs
    const int64_t m_tiles = (s.T + rtc::BM - 1) / rtc::BM;
    const int nkb = (s.H + rtc::BK - 1) / rtc::BK;
    int ks = 1;
    while (ks < 8 && m_tiles * ks * 2 <= num_sms && nkb >= 8 * ks &&
           (2 * ks - 1) * E_PAD * rtc::BM * 4 <= C::STAGES * C::STAGE_BYTES)
        ks *= 2;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(m_tiles * ks), 1, 1);
    cfg.blockDim = dim3(rts::THREADS, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(ks);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, map, map_ws, bias, logits, idx, w, s.T, s.H, s.E, s.k,
                              ks, err_flag, static_cast<uint64_t>(4000000000ull));
}

// Tensor-core router on a weight split by launch_router_split.
cudaError_t launch_route_tc_split(const moe_shape& s, const void* x, const void* w_split,
                                  const float* bias, float* logits, int32_t* idx, float* w,
                                  int32_t* err_flag, int num_sms, cudaStream_t st) {
    if (s.E <= 8)
        return launch_route_tc_split_t<8>(s, x, w_split, bias, logits, idx, w, err_flag, num_sms,
                                          st);
    if (s.E <= 16)
        return launch_route_tc_split_t<16>(s, x, w_split, bias, logits, idx, w, err_flag,
                                           num_sms, st);
    if (s.E <= 32)
        return launch_route_tc_split_t<32>(s, x, w_split, bias, logits, idx, w, err_flag,
                                           num_sms, st);
    return launch_route_tc_split_t<64>(s, x, w_split, bias, logits, idx, w, err_flag, num_sms,
                                       st);
}

}  // namespace moe
