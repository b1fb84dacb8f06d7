// Grouped GEMMs of the backward pass of the expert FFNs on the tensor cores.
//
// The forward GEMMs ("Mixture of Experts in Transformers", expert backends:
// one grouped GEMM over the expert-sorted tokens; "PhiMoE in Transformers",
// section 2 item 3: gate_up_proj packed [gate; up], act(gate) * up) read both
// operands K-major.  Their gradients need transposed operands, which this
// kernel reads MN-major straight from the forward's tensors (tcgen05 takes
// bf16 operands in either major): a TMA box of 64 MN-columns x 64 K-rows
// (128-byte swizzle) lands as 8 atoms of 8 K-rows x 128 bytes; the shared
// memory descriptor steps 1 KB between K-atoms (SBO) and 8 KB between the
// 64-column MN blocks of a tile (LBO).
//
// Three modes, one CTA per 128 x 256 output tile at a time (persistent),
// warp-specialised like the forward kernel (TMA producer, single-thread MMA
// issuer with two TMEM accumulators, four epilogue warps):
//   kDgradDown   (per expert rows) A = dO (K-major, rows of the padded sorted
//                order, K = H), B = down_e (MN-major: [H, I] read as I x H):
//                acc = dh = s w Wd^T dy.  Epilogue: the SwiGLU backward with
//                the saved pre-activations g, u: dg = dh u SiLU'(g),
//                du = dh SiLU(g), written as dgu [gate | up]; and the tile's
//                part of the routing weight's gradient, sum_i dh_i SiLU(g_i)
//                u_i over its 256 columns, stored per (slot, n-tile) and summed
//                in order by the router backward (the total is s w <G, a>; the
//                router backward divides by w).
//   kDgradGateUp (per expert rows) A = dgu (K-major, K = 2I), B = gate_up_e
//                (MN-major: [2I, H] read as H x 2I): acc = dx of the slot.
//   kWgrad       (per expert output tile) A = the output gradient rows
//                (MN-major), B = the input rows (MN-major), K = the expert's
//                rows: dW_e = sum_p dout_p^T in_p, written in float32.  The
//                A rows of an expert are padded with zero rows to a multiple of
//                128 (see backward.cu), so a k-block that runs past the
//                expert's rows adds nothing whatever B holds there.
// Shared experts are extra groups with the T token rows.  Every wait is
// bounded; on expiry MOE_ERR_TIMEOUT is raised and the CTA winds down.
#include "gemm_common.cuh"

namespace moe {

enum : int { kDgradDown = 0, kDgradGateUp = 1, kWgrad = 2 };

namespace bwd {
constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int UMMA_K = 16;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;          // 16 KB
constexpr int B_BYTES = BN * BK * 2;          // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int BOX_BYTES = 64 * BK * 2;        // one MN-major box: 64 columns x 64 rows
constexpr int TMEM_COLS = 512;
constexpr int EPI_WARPS = 8;                  // two per TMEM lane quarter, each on half the columns
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
}  // namespace bwd

// Shared-memory descriptor of an MN-major operand tile in the 128-byte
// swizzle: MN blocks of 64 elements (one 128-byte row) 8 KB apart, K-atoms of
// 8 rows 1 KB apart.
__device__ __forceinline__ uint64_t smem_desc_mn_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);   // start address
    d |= static_cast<uint64_t>(bwd::BOX_BYTES >> 4) << 16;  // leading byte offset (MN)
    d |= static_cast<uint64_t>(1024 >> 4) << 32;            // stride byte offset (K)
    d |= static_cast<uint64_t>(1) << 46;                    // descriptor version (sm_100)
    d |= static_cast<uint64_t>(2) << 61;                    // swizzle: 128 B
    return d;
}

// 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16_bwd(uint32_t taddr, float* v) {
    uint32_t* r = reinterpret_cast<uint32_t*>(v);
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

// TMA tensor store of a 3D box from shared memory (coordinates innermost
// first), tracked by the thread's bulk async-group.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, uint32_t src, int32_t c0,
                                             int32_t c1, int32_t c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(src), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}
__device__ __forceinline__ void bulk_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// every committed bulk store of this thread has finished reading shared memory
__device__ __forceinline__ void bulk_wait_read0() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// every committed bulk store of this thread is complete
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// 16-byte load, zero when !ok; volatile so that it is issued where written
// (ahead of the math that consumes it).
__device__ __forceinline__ uint4 ldg16_pred(const __nv_bfloat16* ptr, bool ok) {
    uint4 v;
    asm volatile(
        "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %5, 0;\n\t"
        "mov.b32 %0, 0;\n\tmov.b32 %1, 0;\n\tmov.b32 %2, 0;\n\tmov.b32 %3, 0;\n\t"
        "@q ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];\n\t}"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(ptr), "r"(static_cast<int>(ok)));
    return v;
}

struct BwdParams {
    const int32_t* offsets;    // [E+1] sorted rows of each routed expert
    const int32_t* poffsets;   // [E+1] the same, each expert padded to a multiple of 128
    const int32_t* perm;       // [T*k]
    int64_t T;
    int E, S;
    int n_tiles_routed, n_tiles_shared;   // output column tiles
    int m_tiles_routed, m_tiles_shared;   // kWgrad: output row tiles
    int K_routed, K_shared;               // dgrad: contraction length
    int M_routed, M_shared;               // kWgrad: output rows
    int N_routed, N_shared;               // output columns
    int b_rows_routed, b_rows_shared;     // dgrad: B rows per expert (its K extent)
    int I_routed, I_shared;               // kDgradDown: width of gate (and of up)
    const __nv_bfloat16* gu_routed;       // kDgradDown: saved [g | u] rows [T*k, 2I]
    const __nv_bfloat16* gu_shared;       //                         [S*T, 2Is]
    void* out_routed;
    void* out_shared;
    float* dw_raw;                        // kDgradDown: [T*k, n_tiles] per slot and n-tile
    // kWgrad: a shared expert's A / B rows start at (s * stride): T for the
    // per-expert buffers ([S*T, .]), 0 for the token-row tensors (dy, x)
    int64_t a_sh_stride, b_sh_stride;
    int32_t* err_flag;
    uint64_t timeout_ns;
};

template <int MAXG>
struct BwdTable {
    int32_t n_groups;
    int32_t total_tiles;
    int32_t tile_start[MAXG + 1];
    int32_t rows[MAXG];     // dgrad: valid rows; kWgrad: contraction rows
    int32_t row0[MAXG];     // first row in the unpadded sorted order (shared: s*T)
    int32_t prow0[MAXG];    // first row in the padded order (shared: s*T)
    int32_t prows[MAXG];    // padded rows (shared: T)
};

// One thread; offsets / poffsets staged in shared memory (E+1 entries each).
template <int MODE, int MAXG>
__device__ void build_bwd_table(BwdTable<MAXG>& bt, const int32_t* offs, const int32_t* poffs,
                                const BwdParams& p) {
    int32_t acc = 0;
    bt.n_groups = p.E + p.S;
    for (int g = 0; g < p.E + p.S; ++g) {
        const bool routed = g < p.E;
        int32_t rows, row0, prow0, prows;
        if (routed) {
            row0 = offs[g];
            rows = offs[g + 1] - row0;
            prow0 = poffs[g];
            prows = poffs[g + 1] - prow0;
        } else {
            row0 = prow0 = static_cast<int32_t>((g - p.E) * p.T);
            rows = prows = static_cast<int32_t>(p.T);
        }
        if (rows < 0) rows = 0;
        bt.rows[g] = rows;
        bt.row0[g] = row0;
        bt.prow0[g] = prow0;
        bt.prows[g] = prows;
        bt.tile_start[g] = acc;
        if (MODE == kWgrad) {
            acc += routed ? p.m_tiles_routed * p.n_tiles_routed
                          : p.m_tiles_shared * p.n_tiles_shared;
        } else {
            const int mt = (prows + bwd::BM - 1) / bwd::BM;
            acc += mt * (routed ? p.n_tiles_routed : p.n_tiles_shared);
        }
    }
    bt.tile_start[p.E + p.S] = acc;
    bt.total_tiles = acc;
}

struct BwdTile {
    int g;
    bool routed;
    int m0;      // first output row of the tile (dgrad: within the group)
    int n0;      // first output column
};

// Tile order within a group.  kWgrad: n inner (all of an expert's operand
// rows fit in L2 either way).  dgrad: m inner, so that the CTAs working at
// the same time share the B panel (a slice of the expert's weight, read once
// from memory) and re-read only the expert's small A rows from L2; with n
// inner every m-tile streamed the whole weight again.
template <int MODE, int MAXG>
__device__ __forceinline__ BwdTile decode_bwd_tile(const BwdTable<MAXG>& bt, const BwdParams& p,
                                                   int tile) {
    int lo = 0, hi = bt.n_groups - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (bt.tile_start[mid] <= tile) lo = mid;
        else hi = mid - 1;
    }
    BwdTile c;
    c.g = lo;
    c.routed = lo < p.E;
    const int local = tile - bt.tile_start[lo];
    if (MODE == kWgrad) {
        const int nt = c.routed ? p.n_tiles_routed : p.n_tiles_shared;
        c.m0 = (local / nt) * bwd::BM;
        c.n0 = (local % nt) * bwd::BN;
    } else {
        const int mt = (bt.prows[lo] + bwd::BM - 1) / bwd::BM;
        c.m0 = (local % mt) * bwd::BM;
        c.n0 = (local / mt) * bwd::BN;
    }
    return c;
}

template <int MODE>
__global__ void __launch_bounds__(bwd::THREADS, 1) grouped_gemm_bwd(
    const __grid_constant__ CUtensorMap map_a_routed, const __grid_constant__ CUtensorMap map_a_shared,
    const __grid_constant__ CUtensorMap map_b_routed, const __grid_constant__ CUtensorMap map_b_shared,
    const __grid_constant__ CUtensorMap map_o_routed, const __grid_constant__ CUtensorMap map_o_shared,
    const BwdParams p) {
    using namespace bwd;
    constexpr bool A_MN = MODE == kWgrad;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ BwdTable<kMaxGroups> bt;
    __shared__ int32_t offs_sh[kMaxExperts + 1];
    __shared__ int32_t poffs_sh[kMaxExperts + 1];
    __shared__ uint32_t tmem_base_sh;
    // kWgrad epilogue: per epilogue warp one 32-row x 16-column fp32 block,
    // 64-byte swizzled, that a TMA tensor store writes out
    __shared__ __align__(1024) float wg_out[MODE == kWgrad ? EPI_WARPS : 1][32 * 16];

    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
    uint64_t* full = bars;
    uint64_t* empty = bars + STAGES;
    uint64_t* tfull = bars + 2 * STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint64_t deadline = global_ns() + p.timeout_ns;

    for (int g = static_cast<int>(threadIdx.x); g <= p.E; g += static_cast<int>(blockDim.x)) {
        offs_sh[g] = p.offsets[g];
        poffs_sh[g] = p.poffsets[g];
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 32 * EPI_WARPS);
        }
        mbar_init(drain, 1);
        fence_barrier_init();
        build_bwd_table<MODE>(bt, offs_sh, poffs_sh, p);
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
    const int total = bt.total_tiles;

    // k-blocks of a tile
    auto num_kb = [&](const BwdTile& c) -> int {
        if (MODE == kWgrad) {
            const int rows = c.routed ? bt.prows[c.g] : bt.rows[c.g];
            return (rows + BK - 1) / BK;
        }
        const int K = c.routed ? p.K_routed : p.K_shared;
        return (K + BK - 1) / BK;
    };

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                const BwdTile c = decode_bwd_tile<MODE>(bt, p, tile);
                const CUtensorMap* ma = c.routed ? &map_a_routed : &map_a_shared;
                const CUtensorMap* mb = c.routed ? &map_b_routed : &map_b_shared;
                const int eidx = c.routed ? c.g : c.g - p.E;
                const int nkb = num_kb(c);
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, deadline)) { ok = false; break; }
                    uint8_t* sa = smem + stage * STAGE_BYTES;
                    uint8_t* sb = sa + A_BYTES;
                    mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
                    if (MODE == kWgrad) {
                        // A: output-gradient rows (padded order for routed experts),
                        // columns m0..m0+127; B: input rows (unpadded order),
                        // columns n0..n0+255; K runs over the rows
                        const int64_t sh = c.g - p.E;
                        const int ka = static_cast<int>(
                            (c.routed ? bt.prow0[c.g] : sh * p.a_sh_stride) + kb * BK);
                        const int kbr = static_cast<int>(
                            (c.routed ? bt.row0[c.g] : sh * p.b_sh_stride) + kb * BK);
#pragma unroll
                        for (int b = 0; b < BM / 64; ++b)
                            tma_load_2d(sa + b * BOX_BYTES, ma, &full[stage], c.m0 + 64 * b, ka);
#pragma unroll
                        for (int b = 0; b < BN / 64; ++b)
                            tma_load_2d(sb + b * BOX_BYTES, mb, &full[stage], c.n0 + 64 * b, kbr);
                    } else {
                        // A: K-major rows of the group (padded order for routed
                        // experts; the shared experts' rows start at s*T, or at 0
                        // when A is dy itself); B: expert eidx's weight rows
                        // [eidx * b_rows + k] read MN-major
                        const int a_row = (c.routed ? bt.prow0[c.g]
                                                    : (MODE == kDgradDown ? 0 : bt.prow0[c.g])) +
                                          c.m0;
                        const int b_rows = c.routed ? p.b_rows_routed : p.b_rows_shared;
                        const int krow = eidx * b_rows + kb * BK;
                        tma_load_2d(sa, ma, &full[stage], kb * BK, a_row);
#pragma unroll
                        for (int b = 0; b < BN / 64; ++b)
                            tma_load_2d(sb + b * BOX_BYTES, mb, &full[stage], c.n0 + 64 * b, krow);
                    }
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            if (!ok) raise_error(p.err_flag, MOE_ERR_TIMEOUT);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(BM, BN) | (A_MN ? (1u << 15) : 0u) |
                                       (1u << 16);   // B is MN-major in every mode
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                const BwdTile c = decode_bwd_tile<MODE>(bt, p, tile);
                const int nkb = num_kb(c);
                if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, deadline)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(&full[stage], phase, deadline)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
                    const uint32_t sb = sa + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / UMMA_K; ++kk) {
                        const uint64_t da = A_MN ? smem_desc_mn_sw128(sa + kk * UMMA_K * 128)
                                                 : smem_desc_sw128(sa + kk * UMMA_K * 2);
                        const uint64_t db = smem_desc_mn_sw128(sb + kk * UMMA_K * 128);
                        umma_bf16(d_tmem, da, db, idesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    umma_commit(&empty[stage]);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                umma_commit(&tfull[acc]);        // also when the tile had no k-blocks
                if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
            }
            if (!ok) raise_error(p.err_flag, MOE_ERR_TIMEOUT);
            umma_commit(drain);
            if (!mbar_wait(drain, 0, deadline + 1000000000ull))
                raise_error(p.err_flag, MOE_ERR_TIMEOUT);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int quarter = warp & 3;
        const int r_in_tile = quarter * 32 + lane;
        const int ch = (warp - 2) >> 2;              // which half of the columns
        const int c_begin = ch * (BN / 2), c_end = c_begin + BN / 2;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
            const BwdTile c = decode_bwd_tile<MODE>(bt, p, tile);
            if (!mbar_wait(&tfull[acc], acc_phase, deadline)) {
                raise_error(p.err_flag, MOE_ERR_TIMEOUT);
                break;
            }
            tc_fence_after();
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                   static_cast<uint32_t>(acc * BN);
            const int N = c.routed ? p.N_routed : p.N_shared;
            if (MODE == kWgrad) {
                const int M = c.routed ? p.M_routed : p.M_shared;
                const int eidx = c.routed ? c.g : c.g - p.E;
                const bool has_k = num_kb(c) > 0;
                // the warp's 32 rows x 16 columns are staged in shared memory
                // (row = lane, 64-byte swizzle: 16-byte chunk q of row r at
                // q ^ ((r >> 1) & 3), conflict-free) and written by one TMA
                // store; rows past M and columns past N fall outside the
                // tensor map and are not written
                const CUtensorMap* mo = c.routed ? &map_o_routed : &map_o_shared;
                float* buf = wg_out[warp - 2];
                const uint32_t sbuf = smem_u32(buf);
                (void)M;
#pragma unroll 1
                for (int cc = c_begin; cc < c_end; cc += 16) {
                    float v[16];
                    if (has_k) {
                        tmem_ld16_bwd(taddr + cc, v);
                        tmem_ld_wait();
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; ++j) v[j] = 0.f;
                    }
                    // the previous store of this warp has read the buffer
                    if (lane == 0) bulk_wait_read0();
                    __syncwarp();
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        *reinterpret_cast<float4*>(buf + lane * 16 + ((q ^ ((lane >> 1) & 3)) * 4)) =
                            make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_3d(mo, sbuf, c.n0 + cc, c.m0 + quarter * 32, eidx);
                        bulk_commit();
                    }
                }
            } else if (MODE == kDgradDown) {
                // rows: routed -> padded row prow0 + m (dgu) and sorted row row0 + m
                // (saved g, u; slot perm[row0 + m]); rows past the expert's own
                // up to the padding write zeros.  Shared -> row s*T + m.
                const int m = c.m0 + r_in_tile;
                const bool valid = m < bt.rows[c.g];
                const bool pad = c.routed && !valid && m < bt.prows[c.g];
                const int I2 = c.routed ? p.I_routed : p.I_shared;
                const int64_t grow = static_cast<int64_t>(bt.row0[c.g]) + m;
                const int64_t orow = static_cast<int64_t>(bt.prow0[c.g]) + m;
                const __nv_bfloat16* gu = (c.routed ? p.gu_routed : p.gu_shared) + grow * 2 * I2;
                __nv_bfloat16* dgu = static_cast<__nv_bfloat16*>(c.routed ? p.out_routed
                                                                          : p.out_shared) +
                                     orow * 2 * I2;
                float dwp = 0.f;
                // g and u of the next 32 columns are requested before this
                // chunk's tensor-memory load and math, so their latency hides
                uint4 gcur[4], ucur[4], gnxt[4], unxt[4];
                auto load_gu = [&](int cc, uint4 (&g4)[4], uint4 (&u4)[4]) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int nq = c.n0 + cc + 8 * q;
                        const bool in = valid && nq < N;
                        g4[q] = ldg16_pred(gu + nq, in);
                        u4[q] = ldg16_pred(gu + I2 + nq, in);
                    }
                };
                load_gu(c_begin, gcur, ucur);
#pragma unroll 1
                for (int cc = c_begin; cc < c_end; cc += 32) {
                    float v[32];
                    tmem_ld32(taddr + cc, v);
                    if (cc + 32 < c_end) load_gu(cc + 32, gnxt, unxt);
                    tmem_ld_wait();
                    const int n = c.n0 + cc;
                    if (valid) {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const int nq = n + 8 * q;
                            if (nq >= N) break;
                            const uint4 gv = gcur[q];
                            const uint4 uv = ucur[q];
                            const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
                            const uint32_t uw[4] = {uv.x, uv.y, uv.z, uv.w};
                            uint32_t og[4], ou[4];
#pragma unroll
                            for (int h = 0; h < 4; ++h) {
                                float dgo[2], duo[2];
#pragma unroll
                                for (int e2 = 0; e2 < 2; ++e2) {
                                    const float gg = bf16_to_f32(static_cast<uint16_t>(
                                        e2 ? gw[h] >> 16 : gw[h] & 0xffffu));
                                    const float uu = bf16_to_f32(static_cast<uint16_t>(
                                        e2 ? uw[h] >> 16 : uw[h] & 0xffffu));
                                    const float dh = v[8 * q + 2 * h + e2];
                                    const float sg = 1.f / (1.f + __expf(-gg));
                                    const float si = gg * sg;
                                    dgo[e2] = dh * uu * sg * (1.f + gg * (1.f - sg));
                                    duo[e2] = dh * si;
                                    dwp = fmaf(dh, si * uu, dwp);
                                }
                                og[h] = pack_bf16x2(dgo[0], dgo[1]);
                                ou[h] = pack_bf16x2(duo[0], duo[1]);
                            }
                            *reinterpret_cast<uint4*>(dgu + nq) = make_uint4(og[0], og[1], og[2], og[3]);
                            *reinterpret_cast<uint4*>(dgu + I2 + nq) =
                                make_uint4(ou[0], ou[1], ou[2], ou[3]);
                        }
                    } else if (pad) {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const int nq = n + 8 * q;
                            if (nq >= N) break;
                            *reinterpret_cast<uint4*>(dgu + nq) = make_uint4(0, 0, 0, 0);
                            *reinterpret_cast<uint4*>(dgu + I2 + nq) = make_uint4(0, 0, 0, 0);
                        }
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        gcur[q] = gnxt[q];
                        ucur[q] = unxt[q];
                    }
                }
                if (valid && c.routed)
                    p.dw_raw[(static_cast<int64_t>(p.perm[grow]) * p.n_tiles_routed + c.n0 / BN) * 2 + ch] = dwp;
            } else {
                // kDgradGateUp: dx of the slot row (routed: padded row prow0 + m;
                // shared: s*T + m), bf16
                const int m = c.m0 + r_in_tile;
                const bool valid = m < bt.rows[c.g];
                const int64_t orow = static_cast<int64_t>(bt.prow0[c.g]) + m;
                __nv_bfloat16* out = static_cast<__nv_bfloat16*>(c.routed ? p.out_routed
                                                                          : p.out_shared) +
                                     orow * N;
#pragma unroll 1
                for (int cc = c_begin; cc < c_end; cc += 32) {
                    float v[32];
                    tmem_ld32(taddr + cc, v);
                    tmem_ld_wait();
                    const int n = c.n0 + cc;
                    if (valid) {
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            if (n + 8 * q < N)
                                *reinterpret_cast<uint4*>(out + n + 8 * q) = make_uint4(
                                    pack_bf16x2(v[8 * q], v[8 * q + 1]),
                                    pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                                    pack_bf16x2(v[8 * q + 4], v[8 * q + 5]),
                                    pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
            if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        }
    }

    // the TMA stores have finished (they read shared memory that the CTA frees)
    if (MODE == kWgrad && warp >= 2 && lane == 0) bulk_wait_all();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// Weight gradient [E, M, N] float32 as a 3D tensor (N, M, E) for the
// epilogue's TMA stores: box 16 columns x 32 rows, 64-byte swizzle.
static bool make_map_out_f32(CUtensorMap* map, void* base, int E, int64_t M, int64_t N) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc || !base || E <= 0 || M <= 0 || N <= 0 || (N * 4) % 16 != 0) return false;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M),
                          static_cast<cuuint64_t>(E)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(N * 4), static_cast<cuuint64_t>(M * N * 4)};
    cuuint32_t box[3] = {16u, 32u, 1u};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
               CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MODE>
static cudaError_t launch_bwd_mode(const CUtensorMap& a_r, const CUtensorMap& a_s,
                                   const CUtensorMap& b_r, const CUtensorMap& b_s,
                                   const CUtensorMap& o_r, const CUtensorMap& o_s,
                                   const BwdParams& p, int64_t tiles_bound, int num_sms,
                                   cudaStream_t st) {
    auto kern = grouped_gemm_bwd<MODE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         bwd::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const int grid = static_cast<int>(tiles_bound < num_sms ? (tiles_bound > 0 ? tiles_bound : 1)
                                                            : num_sms);
    kern<<<grid, bwd::THREADS, bwd::SMEM_BYTES, st>>>(a_r, a_s, b_r, b_s, o_r, o_s, p);
    return cudaGetLastError();
}

// The four GEMMs of the expert backward (see backward.cu for the buffers).
//   dO [P, H], dgu [P, 2I]: rows in the padded sorted order (P rows); dX [P, H]
//   is written over dO after both GEMMs that read dO have run
//   dy [T, H] (shared experts' dO), dgu_sh [S*T, 2Is], dX_sh [S*T, H]
//   gu [T*k, 2I], gu_sh [S*T, 2Is], h [T*k, I], h_sh [S*T, Is], x_perm [T*k, H]:
//   saved by the training forward (unpadded sorted order / s*T + t)
cudaError_t launch_expert_backward(const moe_shape& s, int64_t P, const int32_t* offsets,
                                   const int32_t* poffsets, const int32_t* perm, const void* x,
                                   const void* dy, const void* gate_up, const void* down,
                                   const void* sh_gate_up, const void* sh_down, const void* gu,
                                   const void* gu_sh, const void* h, const void* h_sh,
                                   const void* x_perm, const void* dO, void* dgu, void* dgu_sh,
                                   void* dX, void* dX_sh, float* dw_raw, float* d_gate_up,
                                   float* d_down, float* d_sh_gate_up, float* d_sh_down,
                                   int32_t* err_flag, int num_sms, cudaStream_t st) {
    using namespace bwd;
    const int64_t Tk = s.T * s.k;
    const int S = s.n_shared;
    const int Is = S > 0 ? s.I_shared : s.I;
    const int64_t ST = S > 0 ? static_cast<int64_t>(S) * s.T : 1;
    const int E = s.E, H = s.H, I = s.I;
    BwdParams p{};
    p.offsets = offsets;
    p.poffsets = poffsets;
    p.perm = perm;
    p.T = s.T;
    p.E = E;
    p.S = S;
    p.I_routed = I;
    p.I_shared = Is;
    p.gu_routed = static_cast<const __nv_bfloat16*>(gu);
    p.gu_shared = static_cast<const __nv_bfloat16*>(gu_sh);
    p.dw_raw = dw_raw;
    p.err_flag = err_flag;
    p.timeout_ns = 4000000000ull;
    const int64_t mt_dgrad = ceil_div(P, BM) + E + (S > 0 ? S * ceil_div(s.T, BM) : 0);

    // ---- 1. dgrad through down + SwiGLU backward: dgu, dw
    {
        CUtensorMap ar, as, br, bs;
        bool ok = make_map(&ar, dO, P, H, BM);
        ok &= make_map(&br, down, static_cast<int64_t>(E) * H, I, 64);
        if (S > 0) {
            ok &= make_map(&as, dy, s.T, H, BM);
            ok &= make_map(&bs, sh_down, static_cast<int64_t>(S) * H, Is, 64);
        } else {
            as = ar;
            bs = br;
        }
        if (!ok) return cudaErrorInvalidValue;
        p.n_tiles_routed = static_cast<int>(ceil_div(I, BN));
        p.n_tiles_shared = static_cast<int>(ceil_div(Is, BN));
        p.K_routed = H;
        p.K_shared = H;
        p.N_routed = I;
        p.N_shared = Is;
        p.b_rows_routed = H;
        p.b_rows_shared = H;
        p.out_routed = dgu;
        p.out_shared = dgu_sh;
        cudaError_t e = launch_bwd_mode<kDgradDown>(
            ar, as, br, bs, ar, ar, p, mt_dgrad * (p.n_tiles_routed > p.n_tiles_shared ? p.n_tiles_routed
                                                                                : p.n_tiles_shared),
            num_sms, st);
        if (e != cudaSuccess) return e;
    }
    // ---- 2. weight gradient of down: dWd_e = sum_p dO_p^T h_p  [H, I]
    {
        CUtensorMap ar, as, br, bs;
        bool ok = make_map(&ar, dO, P, H, 64);
        ok &= make_map(&br, h, Tk, I, 64);
        if (S > 0) {
            ok &= make_map(&as, dy, s.T, H, 64);
            ok &= make_map(&bs, h_sh, ST, Is, 64);
        } else {
            as = ar;
            bs = br;
        }
        if (!ok) return cudaErrorInvalidValue;
        p.M_routed = H;
        p.M_shared = H;
        p.N_routed = I;
        p.N_shared = Is;
        p.m_tiles_routed = static_cast<int>(ceil_div(H, BM));
        p.m_tiles_shared = p.m_tiles_routed;
        p.n_tiles_routed = static_cast<int>(ceil_div(I, BN));
        p.n_tiles_shared = static_cast<int>(ceil_div(Is, BN));
        p.out_routed = d_down;
        p.out_shared = d_sh_down;
        p.a_sh_stride = 0;          // dy rows
        p.b_sh_stride = s.T;        // h_sh rows s*T + t
        const int64_t tiles = static_cast<int64_t>(E) * p.m_tiles_routed * p.n_tiles_routed +
                              static_cast<int64_t>(S) * p.m_tiles_shared * p.n_tiles_shared;
        CUtensorMap orr, os;
        if (!make_map_out_f32(&orr, d_down, E, H, I) ||
            !make_map_out_f32(&os, S > 0 ? d_sh_down : d_down, S > 0 ? S : E, H, S > 0 ? Is : I))
            return cudaErrorInvalidValue;
        cudaError_t e = launch_bwd_mode<kWgrad>(ar, as, br, bs, orr, os, p, tiles, num_sms, st);
        if (e != cudaSuccess) return e;
    }
    // ---- 3. dgrad through gate_up: dX (into dO's buffer, which is dead by now)
    {
        CUtensorMap ar, as, br, bs;
        bool ok = make_map(&ar, dgu, P, 2 * I, BM);
        ok &= make_map(&br, gate_up, static_cast<int64_t>(E) * 2 * I, H, 64);
        if (S > 0) {
            ok &= make_map(&as, dgu_sh, ST, 2 * Is, BM);
            ok &= make_map(&bs, sh_gate_up, static_cast<int64_t>(S) * 2 * Is, H, 64);
        } else {
            as = ar;
            bs = br;
        }
        if (!ok) return cudaErrorInvalidValue;
        p.n_tiles_routed = static_cast<int>(ceil_div(H, BN));
        p.n_tiles_shared = p.n_tiles_routed;
        p.K_routed = 2 * I;
        p.K_shared = 2 * Is;
        p.N_routed = H;
        p.N_shared = H;
        p.b_rows_routed = 2 * I;
        p.b_rows_shared = 2 * Is;
        p.out_routed = dX;
        p.out_shared = dX_sh;
        cudaError_t e = launch_bwd_mode<kDgradGateUp>(ar, as, br, bs, ar, ar, p,
                                                      mt_dgrad * p.n_tiles_routed, num_sms, st);
        if (e != cudaSuccess) return e;
    }
    // ---- 4. weight gradient of gate_up: dWgu_e = sum_p dgu_p^T x_p  [2I, H]
    {
        CUtensorMap ar, as, br, bs;
        bool ok = make_map(&ar, dgu, P, 2 * I, 64);
        ok &= make_map(&br, x_perm, Tk, H, 64);
        if (S > 0) {
            ok &= make_map(&as, dgu_sh, ST, 2 * Is, 64);
            ok &= make_map(&bs, x, s.T, H, 64);
        } else {
            as = ar;
            bs = br;
        }
        if (!ok) return cudaErrorInvalidValue;
        p.M_routed = 2 * I;
        p.M_shared = 2 * Is;
        p.N_routed = H;
        p.N_shared = H;
        p.m_tiles_routed = static_cast<int>(ceil_div(2 * I, BM));
        p.m_tiles_shared = static_cast<int>(ceil_div(2 * Is, BM));
        p.n_tiles_routed = static_cast<int>(ceil_div(H, BN));
        p.n_tiles_shared = p.n_tiles_routed;
        p.out_routed = d_gate_up;
        p.out_shared = d_sh_gate_up;
        p.a_sh_stride = s.T;        // dgu_sh rows s*T + t
        p.b_sh_stride = 0;          // x rows
        const int64_t tiles = static_cast<int64_t>(E) * p.m_tiles_routed * p.n_tiles_routed +
                              static_cast<int64_t>(S) * p.m_tiles_shared * p.n_tiles_shared;
        CUtensorMap orr, os;
        if (!make_map_out_f32(&orr, d_gate_up, E, 2 * I, H) ||
            !make_map_out_f32(&os, S > 0 ? d_sh_gate_up : d_gate_up, S > 0 ? S : E,
                              S > 0 ? 2 * Is : 2 * I, H))
            return cudaErrorInvalidValue;
        return launch_bwd_mode<kWgrad>(ar, as, br, bs, orr, os, p, tiles, num_sms, st);
    }
}

}  // namespace moe
