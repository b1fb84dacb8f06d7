// The grouped GEMMs of the expert FFNs on CTA pairs (tcgen05 cta_group::2).
//
// Same computation as the one-CTA kernel ("Mixture of Experts in
// Transformers", expert backends: one grouped GEMM over all experts after
// sorting the tokens by expert; "PhiMoE in Transformers", section 2 item 3:
// packed gate_up_proj, act(gate) * up), with tiles of 256 rows x 256 MMA
// columns computed by two CTAs of a cluster:
//   - each CTA loads its 128 rows of A and 128 of the 256 B rows (GEMM 1:
//     CTA 0 the gate rows, CTA 1 the matching up rows; GEMM 2: the two halves
//     of the down panel), so per MMA each SM streams a third less operand data
//     than with 128 x 256 tiles on one SM;
//   - both CTAs' TMA loads complete on the even CTA's full barrier; the even
//     CTA alone issues tcgen05.mma.cta_group::2 (M=256, N=256, K=16) and its
//     commits arrive on both CTAs' barriers (stage free, accumulator full);
//   - each CTA's epilogue reads its own 128 TMEM lanes (= its 128 rows) and
//     reports the accumulator free on the even CTA's barrier;
//   - the last m-tile of a group with at most 128 real rows runs as an M=128
//     pair MMA (64 rows per CTA), which the hardware stores folded: TMEM lanes
//     0-63 hold the first half of the columns, lanes 64-127 the second half.
//     For GEMM 1 each CTA then loads 64 gate rows and the matching 64 up rows,
//     so every lane still holds gate and up of the same output columns.
// No TMA multicast is used: each CTA fetches its own operand halves.
// Waits are bounded as in the one-CTA kernel.
#include "gemm_common.cuh"

namespace moe {

namespace pair {
constexpr int BM = 256;                       // tile rows (128 per CTA)
constexpr int BM_CTA = 128;
constexpr int BN = 256;                       // MMA N
constexpr int BN_CTA = 128;                   // B rows per CTA
constexpr int BK = 64;
constexpr int UMMA_K = 16;
constexpr int A_BYTES = BM_CTA * BK * 2;      // 16 KB
constexpr int B_BYTES = BN_CTA * BK * 2;      // 16 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TMEM_COLS = 512;                // two 256-column accumulators
constexpr int THREADS = 192;
constexpr int EPI_WARPS = 4;
constexpr uint16_t BOTH = 0x3;                // cluster ranks 0 and 1
}  // namespace pair

constexpr int kSmallGroups = 72;              // E + S of every shape measured here

// Tile of the pair kernel.  The last m-tile of a group is a "half" tile when
// at most 128 of its rows are real: it runs as an M=128 pair MMA (64 rows per
// CTA) instead of M=256, which halves the padding of that tile.
template <int MAXG>
__device__ __forceinline__ TileCoord decode_pair_tile(const GroupTableT<MAXG>& gt, const GemmParams& p,
                                                      int tile, int n_cols_per_tile, bool& half) {
    const TileCoord c = decode_tile(gt, p, tile, n_cols_per_tile, pair::BM);
    half = c.rows - c.m0 <= pair::BM / 2;
    return c;
}

// STAGES: depth of the shared-memory ring (7 fits next to a group table of at
// most 72 groups, 6 next to the full 264).
template <int EPI, int STAGES, int MAXG>
__global__ void __launch_bounds__(pair::THREADS, 1) grouped_gemm_pair(
    const __grid_constant__ CUtensorMap map_a_routed, const __grid_constant__ CUtensorMap map_a_shared,
    const __grid_constant__ CUtensorMap map_b_routed, const __grid_constant__ CUtensorMap map_b_shared,
    const __grid_constant__ CUtensorMap map_bh_routed,
    const __grid_constant__ CUtensorMap map_bh_shared, const GemmParams p) {
    using namespace pair;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ GroupTableT<MAXG> gt;
    __shared__ uint32_t tmem_base_sh;

    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
    uint64_t* full = bars;                 // [STAGES] even CTA: both CTAs' TMA bytes
    uint64_t* empty = bars + STAGES;       // [STAGES] both CTAs: stage consumed
    uint64_t* tfull = bars + 2 * STAGES;   // [2]      both CTAs: accumulator ready
    uint64_t* tempty = tfull + 2;          // [2]      even CTA: accumulator freed (8 warps)
    uint64_t* drain = tempty + 2;          // [1]      even CTA: all MMAs complete

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int cluster = static_cast<int>(cluster_id_x());
    const int n_clusters = static_cast<int>(n_clusters_x());
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
            mbar_init(&tempty[b], 2 * EPI_WARPS);
        }
        mbar_init(drain, 1);
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
        tmem_alloc_pair(&tmem_base_sh, TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();        // both CTAs' barriers initialised before any remote use
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_sh;
    const int total = gt.total_tiles;
    const uint32_t full_leader = mapa_shared(smem_u32(full), 0);
    const uint32_t tempty_leader = mapa_shared(smem_u32(tempty), 0);

    if (warp == 0) {
        // ------------------------------------------------------------ producer (both CTAs)
        if (lane == 0) {
            // L2 priorities: activation rows are reused by every n-tile of their
            // group (evict-last); weight panels keep the normal policy
            // (evict-first on them measured 8-15 % slower)
            const uint64_t pol_a = l2_policy_evict_last();
            const uint64_t pol_b = l2_policy_evict_normal();
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = cluster; tile < total && ok; tile += n_clusters) {
                bool half;
                const TileCoord c = decode_pair_tile(gt, p, tile, n_cols_per_tile, half);
                const CUtensorMap* ma = c.routed ? &map_a_routed : &map_a_shared;
                const CUtensorMap* mb = c.routed ? &map_b_routed : &map_b_shared;
                const CUtensorMap* mbh = c.routed ? &map_bh_routed : &map_bh_shared;
                const int K = c.routed ? p.K_routed : p.K_shared;
                const int eidx = c.routed ? c.g : c.g - p.E;
                const int up_off = c.routed ? p.half_routed : p.half_shared;
                // this CTA's A rows (128 of a full tile, the first 64 used of a half
                // tile): routed -> sorted slot rows; shared GEMM 1 -> token rows;
                // shared GEMM 2 -> that expert's block of h
                const int rows_cta = half ? BM_CTA / 2 : BM_CTA;
                int a_row = gt.row0[c.g] + c.m0 + static_cast<int>(rank) * rows_cta;
                if (EPI == kSwiGLU && !c.routed) a_row = c.m0 + static_cast<int>(rank) * rows_cta;
                // this CTA's 128 B rows.  GEMM 1, full tile: gate (rank 0) or up
                // (rank 1) of the 128 columns; GEMM 1, half tile: 64 gate rows then
                // the matching 64 up rows of columns n0 + 64 rank; GEMM 2: its half
                const int b_rows = c.routed ? p.b_rows_routed : p.b_rows_shared;
                int b_row = eidx * b_rows + c.n0;
                if (EPI == kSwiGLU) b_row += half ? static_cast<int>(rank) * 64 : (rank ? up_off : 0);
                else b_row += static_cast<int>(rank) * BN_CTA;
                const int num_kb = (K + BK - 1) / BK;
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, deadline)) { ok = false; break; }
                    uint8_t* sa = smem + stage * STAGE_BYTES;
                    if (leader) mbar_arrive_expect_tx(&full[stage], 2 * STAGE_BYTES);
                    const uint32_t bar = full_leader + stage * 8;
                    tma_load_2d_pair_hint(sa, ma, bar, kb * BK, a_row, pol_a);
                    if (EPI == kSwiGLU && half) {
                        tma_load_2d_pair_hint(sa + A_BYTES, mbh, bar, kb * BK, b_row, pol_b);
                        tma_load_2d_pair_hint(sa + A_BYTES + B_BYTES / 2, mbh, bar, kb * BK,
                                              b_row + up_off, pol_b);
                    } else {
                        tma_load_2d_pair_hint(sa + A_BYTES, mb, bar, kb * BK, b_row, pol_b);
                    }
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            if (!ok) raise_error(p.err_flag, MOE_ERR_TIMEOUT);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA (even CTA)
        if (lane == 0 && leader) {
            constexpr uint32_t idesc_full = idesc_bf16_f32(BM, BN);
            constexpr uint32_t idesc_half = idesc_bf16_f32(BM / 2, BN);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int tile = cluster; tile < total && ok; tile += n_clusters) {
                bool half;
                const TileCoord c = decode_pair_tile(gt, p, tile, n_cols_per_tile, half);
                const uint32_t idesc = half ? idesc_half : idesc_full;
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
                    for (int kk = 0; kk < BK / UMMA_K; ++kk)
                        umma_bf16_pair(d_tmem, smem_desc_sw128(sa + kk * UMMA_K * 2),
                                       smem_desc_sw128(sb + kk * UMMA_K * 2), idesc,
                                       (kb | kk) != 0 ? 1u : 0u);
                    umma_commit_pair(&empty[stage], BOTH);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                umma_commit_pair(&tfull[acc], BOTH);
                if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
            }
            if (!ok) raise_error(p.err_flag, MOE_ERR_TIMEOUT);
            // every issued MMA completes before the tensor memory is released
            umma_commit_pair(drain, 0x1);
            if (!mbar_wait(drain, 0, deadline + 1000000000ull))
                raise_error(p.err_flag, MOE_ERR_TIMEOUT);
        }
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        // TMEM lane l of this CTA holds, for a full tile, row 128 rank + l and all
        // 256 columns; for a half tile (64 rows per CTA, folded), row 64 rank +
        // (l mod 64) and columns [0,128) (l < 64) or [128,256) (l >= 64).
        const int quarter = warp & 3;               // TMEM lane quarter of this warp
        const int lane_in_cta = quarter * 32 + lane;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = cluster; tile < total; tile += n_clusters) {
            bool half;
            const TileCoord c = decode_pair_tile(gt, p, tile, n_cols_per_tile, half);
            if (!mbar_wait(&tfull[acc], acc_phase, deadline)) {
                raise_error(p.err_flag, MOE_ERR_TIMEOUT);
                break;
            }
            tc_fence_after();
            const int m = c.m0 + (half ? static_cast<int>(rank) * 64 + (lane_in_cta & 63)
                                       : static_cast<int>(rank) * BM_CTA + lane_in_cta);
            const bool valid = m < c.rows;
            const int N = c.routed ? p.N_routed : p.N_shared;
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                   static_cast<uint32_t>(acc * BN);
            if (EPI == kSwiGLU) {
                __nv_bfloat16* out = static_cast<__nv_bfloat16*>(c.routed ? p.out_routed : p.out_shared);
                const int64_t ld = c.routed ? p.ld_routed : p.ld_shared;
                const int64_t orow = static_cast<int64_t>(gt.row0[c.g]) + m;
                // full: gate at columns [0,128), up at [128,256) for output columns
                // n0 + [0,128); half: gate [0,64), up [64,128) for columns
                // n0 + 64 (l >= 64) + [0,64)
                const int ncols = half ? 64 : BN / 2;
                const int col0 = c.n0 + (half && lane_in_cta >= 64 ? 64 : 0);
#pragma unroll 1
                for (int cc = 0; cc < ncols; cc += 32) {
                    float gv[32], uv[32];
                    tmem_ld32(taddr + cc, gv);
                    tmem_ld32(taddr + ncols + cc, uv);
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
                        const int n = col0 + cc;
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
                // full: columns n0 + [0,256); half: n0 + 128 (l >= 64) + [0,128)
                const int ncols = half ? BN / 2 : BN;
                const int col0 = c.n0 + (half && lane_in_cta >= 64 ? BN / 2 : 0);
#pragma unroll 1
                for (int cc = 0; cc < ncols; cc += 32) {
                    float v[32];
                    tmem_ld32(taddr + cc, v);
                    tmem_ld_wait();
                    uint32_t packed[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        packed[j] = pack_bf16x2(scale * v[2 * j], scale * v[2 * j + 1]);
                    if (valid) {
                        const int n = col0 + cc;
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
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(tempty_leader + acc * 8);
            if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        }
    }

    // both CTAs are done with the pair's tensor memory and barriers
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
}

constexpr int pair_smem_bytes(int stages) { return stages * pair::STAGE_BYTES + 1024 + 256; }

static cudaError_t launch_pair(void (*kern)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap,
                                            CUtensorMap, CUtensorMap, GemmParams),
                               int smem_bytes, int grid, cudaStream_t st, const CUtensorMap& a_r,
                               const CUtensorMap& a_s, const CUtensorMap& b_r,
                               const CUtensorMap& b_s, const CUtensorMap& bh_r,
                               const CUtensorMap& bh_s, const GemmParams& p) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         smem_bytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(pair::THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem_bytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a_r, a_s, b_r, b_s, bh_r, bh_s, p);
}

// GEMM 1 (gate_up + SwiGLU) and GEMM 2 (down + weight) on CTA pairs.
cudaError_t launch_ffn_sm100_pair(const moe_shape& s, const void* x, const void* x_perm,
                                  const int32_t* offsets, const int32_t* perm,
                                  const float* topk_w, const void* gate_up, const void* down,
                                  const void* sh_gate_up, const void* sh_down, void* h_routed,
                                  void* h_shared, void* y_slots, int32_t* err_flag, int num_sms,
                                  int group_m, cudaStream_t st, void* gu_routed, void* gu_shared) {
    using namespace pair;
    const int64_t Tk = s.T * s.k;
    const int S = s.n_shared;
    const int Is = S > 0 ? s.I_shared : s.I;

    CUtensorMap a1r, a1s, b1r, b1s, h1r, h1s, a2r, a2s, b2r, b2s;
    bool ok = true;
    ok &= make_map(&a1r, x_perm, Tk, s.H, BM_CTA);
    ok &= make_map(&b1r, gate_up, static_cast<int64_t>(s.E) * 2 * s.I, s.H, BN_CTA);
    ok &= make_map(&h1r, gate_up, static_cast<int64_t>(s.E) * 2 * s.I, s.H, BN_CTA / 2);
    ok &= make_map(&a2r, h_routed, Tk, s.I, BM_CTA);
    ok &= make_map(&b2r, down, static_cast<int64_t>(s.E) * s.H, s.I, BN_CTA);
    if (S > 0) {
        ok &= make_map(&a1s, x, s.T, s.H, BM_CTA);
        ok &= make_map(&b1s, sh_gate_up, static_cast<int64_t>(S) * 2 * Is, s.H, BN_CTA);
        ok &= make_map(&h1s, sh_gate_up, static_cast<int64_t>(S) * 2 * Is, s.H, BN_CTA / 2);
        ok &= make_map(&a2s, h_shared, static_cast<int64_t>(S) * s.T, Is, BM_CTA);
        ok &= make_map(&b2s, sh_down, static_cast<int64_t>(S) * s.H, Is, BN_CTA);
    } else {
        a1s = a1r; b1s = b1r; h1s = h1r; a2s = a2r; b2s = b2r;
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
    const int max_clusters = num_sms / 2;

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
    int clusters = static_cast<int>(tiles < max_clusters ? tiles : max_clusters);
    // a deeper ring when the group table is small enough to leave room for it
    const bool deep = s.E + S <= kSmallGroups;
    cudaError_t e = deep ? launch_pair(grouped_gemm_pair<kSwiGLU, 7, kSmallGroups>,
                                       pair_smem_bytes(7), 2 * clusters, st, a1r, a1s, b1r, b1s,
                                       h1r, h1s, p)
                         : launch_pair(grouped_gemm_pair<kSwiGLU, 6, kMaxGroups>,
                                       pair_smem_bytes(6), 2 * clusters, st, a1r, a1s, b1r, b1s,
                                       h1r, h1s, p);
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
    clusters = static_cast<int>(tiles < max_clusters ? tiles : max_clusters);
    return deep ? launch_pair(grouped_gemm_pair<kScaled, 7, kSmallGroups>, pair_smem_bytes(7),
                              2 * clusters, st, a2r, a2s, b2r, b2s, b2r, b2s, p)
                : launch_pair(grouped_gemm_pair<kScaled, 6, kMaxGroups>, pair_smem_bytes(6),
                              2 * clusters, st, a2r, a2s, b2r, b2s, b2r, b2s, p);
}

}  // namespace moe
