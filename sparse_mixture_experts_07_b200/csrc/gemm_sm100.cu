// Grouped GEMMs of the expert FFNs on the 5th-generation tensor cores.
//
// "Mixture of Experts in Transformers", expert backends: the grouped_mm
// backend sorts the tokens by expert and runs one grouped GEMM over all
// experts instead of a per-expert loop.  "PhiMoE in Transformers", section 2
// item 3: the gate and up projections are packed as gate_up_proj (E, 2I, H),
// rows [0, I) gate and [I, 2I) up, and the FFN applies act(gate) * up.
//
// Two epilogues share one mainloop:
//   kSwiGLU  (GEMM 1): B tile = 128 gate rows + the 128 matching up rows of
//            gate_up, so one N=256 MMA yields gate and up for 128 columns;
//            the epilogue writes h = SiLU(gate) * up in bf16.
//   kScaled  (GEMM 2): B tile = 256 rows of down; the epilogue multiplies each
//            row by its weight (routed_scale * topk_w of the slot, or 1 for a
//            shared expert) and writes the slot output in bf16.
//
// Structure (one persistent CTA per SM, 192 threads):
//   warp 0      TMA producer: A tile 128x64 and B tile 256x64 (bf16, 128-byte
//               swizzle) per k-block into a 4-stage shared-memory ring;
//   warp 1      allocates 512 TMEM columns; one thread issues
//               tcgen05.mma.cta_group::1.kind::f16 128x256x16 into one of two
//               256-column fp32 accumulators and commits stage releases;
//   warps 2..5  epilogue: tcgen05.ld of their 32 TMEM lanes (rows), fused
//               epilogue math, bf16 stores; frees the accumulator.
// The epilogue of tile i overlaps the mainloop of tile i+1.  Tiles come from
// a group table every CTA rebuilds from the device offsets: group g < E is
// routed expert g (rows [offsets[g], offsets[g+1]) of the sorted slot space),
// group E+s is shared expert s (the T token rows).  Within a group the tiles
// are rasterised in bands of `group_m` m-tiles with n outer, so a band of A
// rows and the B panel stay in L2.
//
// Every wait is bounded by a deadline on %globaltimer; on expiry the kernel
// sets MOE_ERR_TIMEOUT in err_flag, leaves its loops, drains its MMAs and
// frees its tensor memory.
#include "gemm_common.cuh"

namespace moe {

namespace sm100 {
constexpr int BM = 128;
constexpr int BN = 256;     // MMA N (GEMM 1: 128 gate + 128 up)
constexpr int BK = 64;      // one 128-byte swizzle row of bf16
constexpr int UMMA_K = 16;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;          // 16 KB
constexpr int B_BYTES = BN * BK * 2;          // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TMEM_COLS = 512;                // two 256-column accumulators
constexpr int THREADS = 192;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
}  // namespace sm100

template <int EPI>
__global__ void __launch_bounds__(sm100::THREADS, 1) grouped_gemm_sm100(
    const __grid_constant__ CUtensorMap map_a_routed, const __grid_constant__ CUtensorMap map_a_shared,
    const __grid_constant__ CUtensorMap map_b_routed, const __grid_constant__ CUtensorMap map_b_shared,
    const GemmParams p) {
    using namespace sm100;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ GroupTable gt;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;

    // 1024-byte aligned stage ring (128-byte swizzle atoms are 1024 bytes)
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
    uint64_t* full = bars;                 // [STAGES]  TMA -> MMA
    uint64_t* empty = bars + STAGES;       // [STAGES]  MMA -> TMA
    uint64_t* tfull = bars + 2 * STAGES;   // [2]       MMA -> epilogue
    uint64_t* tempty = tfull + 2;          // [2]       epilogue -> MMA
    uint64_t* drain = tempty + 2;          // [1]       final MMA completion

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint64_t deadline = global_ns() + p.timeout_ns;
    constexpr int n_cols_per_tile = (EPI == kSwiGLU) ? BN / 2 : BN;

    stage_offsets(gt.tile_start, p.offsets, p.E);
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 128);
        }
        mbar_init(drain, 1);
        abort_sh = 0;
        fence_barrier_init();
        build_group_table(gt, p.E, p.S, p.T, BM, p.n_tiles_routed, p.n_tiles_shared);
        tma_prefetch_desc(&map_a_routed);
        tma_prefetch_desc(&map_b_routed);
        if (p.S > 0) {
            tma_prefetch_desc(&map_a_shared);
            tma_prefetch_desc(&map_b_shared);
        }
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base_sh, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_sh;
    const int total = gt.total_tiles;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                const TileCoord c = decode_tile(gt, p, tile, n_cols_per_tile, BM);
                const CUtensorMap* ma = c.routed ? &map_a_routed : &map_a_shared;
                const CUtensorMap* mb = c.routed ? &map_b_routed : &map_b_shared;
                const int K = c.routed ? p.K_routed : p.K_shared;
                const int eidx = c.routed ? c.g : c.g - p.E;
                // A rows: routed -> sorted slot rows; shared GEMM 1 -> token rows;
                // shared GEMM 2 -> rows of that shared expert's h block.
                int a_row = gt.row0[c.g] + c.m0;
                if (EPI == kSwiGLU && !c.routed) a_row = c.m0;
                const int b_rows = c.routed ? p.b_rows_routed : p.b_rows_shared;
                const int b_row = eidx * b_rows + c.n0;
                const int half = c.routed ? p.half_routed : p.half_shared;
                const int num_kb = (K + BK - 1) / BK;
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, deadline)) { ok = false; break; }
                    uint8_t* sa = smem + stage * STAGE_BYTES;
                    uint8_t* sb = sa + A_BYTES;
                    mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
                    tma_load_2d(sa, ma, &full[stage], kb * BK, a_row);
                    if (EPI == kSwiGLU) {
                        tma_load_2d(sb, mb, &full[stage], kb * BK, b_row);
                        tma_load_2d(sb + B_BYTES / 2, mb, &full[stage], kb * BK, b_row + half);
                    } else {
                        tma_load_2d(sb, mb, &full[stage], kb * BK, b_row);
                    }
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            if (!ok) {
                raise_error(p.err_flag, MOE_ERR_TIMEOUT);
                atomicExch(&abort_sh, 1);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(BM, BN);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                const TileCoord c = decode_tile(gt, p, tile, n_cols_per_tile, BM);
                const int K = c.routed ? p.K_routed : p.K_shared;
                const int num_kb = (K + BK - 1) / BK;
                if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, deadline)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(&full[stage], phase, deadline)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
                    const uint32_t sb = sa + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / UMMA_K; ++kk) {
                        const uint64_t da = smem_desc_sw128(sa + kk * UMMA_K * 2);
                        const uint64_t db = smem_desc_sw128(sb + kk * UMMA_K * 2);
                        umma_bf16(d_tmem, da, db, idesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    umma_commit(&empty[stage]);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                umma_commit(&tfull[acc]);
                if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
            }
            if (!ok) {
                raise_error(p.err_flag, MOE_ERR_TIMEOUT);
                atomicExch(&abort_sh, 1);
            }
            // all issued MMAs complete before the tensor memory is released
            umma_commit(drain);
            if (!mbar_wait(drain, 0, deadline + 1000000000ull))
                raise_error(p.err_flag, MOE_ERR_TIMEOUT);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int quarter = warp & 3;               // TMEM lane quarter of this warp
        const int row_in_tile = quarter * 32 + lane;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
            const TileCoord c = decode_tile(gt, p, tile, n_cols_per_tile, BM);
            if (!mbar_wait(&tfull[acc], acc_phase, deadline)) {
                raise_error(p.err_flag, MOE_ERR_TIMEOUT);
                break;
            }
            tc_fence_after();
            const int m = c.m0 + row_in_tile;
            const bool valid = m < c.rows;
            const int N = c.routed ? p.N_routed : p.N_shared;
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                   static_cast<uint32_t>(acc * BN);
            if (EPI == kSwiGLU) {
                __nv_bfloat16* out = static_cast<__nv_bfloat16*>(c.routed ? p.out_routed : p.out_shared);
                const int64_t ld = c.routed ? p.ld_routed : p.ld_shared;
                const int64_t orow = static_cast<int64_t>(gt.row0[c.g]) + m;
#pragma unroll 1
                for (int cc = 0; cc < BN / 2; cc += 32) {
                    float gv[32], uv[32];
                    tmem_ld32(taddr + cc, gv);
                    tmem_ld32(taddr + BN / 2 + cc, uv);
                    tmem_ld_wait();
                    uint32_t packed[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float g0 = gv[2 * j], g1 = gv[2 * j + 1];
                        const float h0 = g0 / (1.f + __expf(-g0)) * uv[2 * j];
                        const float h1 = g1 / (1.f + __expf(-g1)) * uv[2 * j + 1];
                        packed[j] = pack_bf16x2(h0, h1);
                    }
                    if (valid) {
                        const int n = c.n0 + cc;
                        uint4* dst = reinterpret_cast<uint4*>(out + orow * ld + n);
#pragma unroll
                        for (int v = 0; v < 4; ++v)
                            if (n + 8 * v < N)
                                dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1],
                                                    packed[4 * v + 2], packed[4 * v + 3]);
                        __nv_bfloat16* gu = static_cast<__nv_bfloat16*>(c.routed ? p.gu_routed
                                                                                  : p.gu_shared);
                        if (gu) store_gu32(gu + orow * 2 * N, n, N, gv, uv);
                    }
                }
            } else {
                __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out_routed);
                int64_t orow;
                float scale = 1.f;
                if (c.routed) {
                    orow = static_cast<int64_t>(gt.row0[c.g]) + m;
                    if (valid) scale = p.routed_scale * p.topk_w[p.perm[orow]];
                } else {
                    orow = p.out_row0_shared + gt.row0[c.g] + m;
                }
                const int64_t ld = p.ld_routed;
#pragma unroll 1
                for (int cc = 0; cc < BN; cc += 32) {
                    float v[32];
                    tmem_ld32(taddr + cc, v);
                    tmem_ld_wait();
                    uint32_t packed[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        packed[j] = pack_bf16x2(scale * v[2 * j], scale * v[2 * j + 1]);
                    if (valid) {
                        const int n = c.n0 + cc;
                        uint4* dst = reinterpret_cast<uint4*>(out + orow * ld + n);
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            if (n + 8 * q < N)
                                dst[q] = make_uint4(packed[4 * q], packed[4 * q + 1],
                                                    packed[4 * q + 2], packed[4 * q + 3]);
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
            if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// GEMM 1 (gate_up + SwiGLU) and GEMM 2 (down + weight) for the bf16 path.
cudaError_t launch_ffn_sm100(const moe_shape& s, const void* x, const void* x_perm,
                             const int32_t* offsets, const int32_t* perm, const float* topk_w,
                             const void* gate_up, const void* down, const void* sh_gate_up,
                             const void* sh_down, void* h_routed, void* h_shared, void* y_slots,
                             int32_t* err_flag, int num_sms, int group_m, cudaStream_t st,
                             void* gu_routed, void* gu_shared) {
    using namespace sm100;
    const int64_t Tk = s.T * s.k;
    const int S = s.n_shared;
    const int Is = S > 0 ? s.I_shared : s.I;

    CUtensorMap a1r, a1s, b1r, b1s, a2r, a2s, b2r, b2s;
    bool ok = true;
    ok &= make_map(&a1r, x_perm, Tk, s.H, BM);
    ok &= make_map(&b1r, gate_up, static_cast<int64_t>(s.E) * 2 * s.I, s.H, BN / 2);
    ok &= make_map(&a2r, h_routed, Tk, s.I, BM);
    ok &= make_map(&b2r, down, static_cast<int64_t>(s.E) * s.H, s.I, BN);
    if (S > 0) {
        ok &= make_map(&a1s, x, s.T, s.H, BM);
        ok &= make_map(&b1s, sh_gate_up, static_cast<int64_t>(S) * 2 * Is, s.H, BN / 2);
        ok &= make_map(&a2s, h_shared, static_cast<int64_t>(S) * s.T, Is, BM);
        ok &= make_map(&b2s, sh_down, static_cast<int64_t>(S) * s.H, Is, BN);
    } else {
        a1s = a1r; b1s = b1r; a2s = a2r; b2s = b2r;
    }
    if (!ok) return cudaErrorInvalidValue;

    GemmParams p{};
    p.offsets = offsets;
    p.perm = perm;
    p.topk_w = topk_w;
    p.T = s.T;
    p.E = s.E;
    p.S = S;
    p.k = s.k;
    p.routed_scale = s.routed_scale;
    p.group_m = group_m;
    p.err_flag = err_flag;
    p.timeout_ns = 4000000000ull;
    p.gu_routed = gu_routed;
    p.gu_shared = gu_shared;

    const int64_t mt_bound = ceil_div(Tk, BM) + s.E;
    const int64_t mt_shared = S > 0 ? S * ceil_div(s.T, BM) : 0;

    // GEMM 1
    p.n_tiles_routed = static_cast<int>(ceil_div(s.I, BN / 2));
    p.n_tiles_shared = static_cast<int>(ceil_div(Is, BN / 2));
    p.K_routed = s.H;
    p.K_shared = s.H;
    p.N_routed = s.I;
    p.N_shared = Is;
    p.b_rows_routed = 2 * s.I;
    p.b_rows_shared = 2 * Is;
    p.half_routed = s.I;
    p.half_shared = Is;
    p.out_routed = h_routed;
    p.out_shared = h_shared;
    p.ld_routed = s.I;
    p.ld_shared = Is;
    p.out_row0_shared = 0;
    int64_t tiles = mt_bound * p.n_tiles_routed + mt_shared * p.n_tiles_shared;
    int grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
    auto k1 = grouped_gemm_sm100<kSwiGLU>;
    cudaError_t e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    k1<<<grid, THREADS, SMEM_BYTES, st>>>(a1r, a1s, b1r, b1s, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    // GEMM 2
    p.gu_routed = nullptr;
    p.gu_shared = nullptr;
    p.n_tiles_routed = static_cast<int>(ceil_div(s.H, BN));
    p.n_tiles_shared = p.n_tiles_routed;
    p.K_routed = s.I;
    p.K_shared = Is;
    p.N_routed = s.H;
    p.N_shared = s.H;
    p.b_rows_routed = s.H;
    p.b_rows_shared = s.H;
    p.half_routed = 0;
    p.half_shared = 0;
    p.out_routed = y_slots;
    p.out_shared = y_slots;
    p.ld_routed = s.H;
    p.ld_shared = s.H;
    p.out_row0_shared = Tk;
    tiles = mt_bound * p.n_tiles_routed + mt_shared * p.n_tiles_shared;
    grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
    auto k2 = grouped_gemm_sm100<kScaled>;
    e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    k2<<<grid, THREADS, SMEM_BYTES, st>>>(a2r, a2s, b2r, b2s, p);
    return cudaGetLastError();
}

}  // namespace moe
