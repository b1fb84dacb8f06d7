// Expert FFNs of decode batches (T <= 64) with MXFP4 expert weights on the
// block-scaled tensor cores: tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale.
//
// "Mixture of Experts in Transformers", section "from dense to sparse": at
// small batch the layer's time is the bytes of the active experts' weights
// read from memory, and gpt-oss ships its experts in mxfp4.  MXFP4 (OCP
// Microscaling Formats v1.0): 32 consecutive weights along the contraction
// share one E8M0 scale 2^(s-127); each weight is a 4-bit E2M1 code.  Storage
// as in the CUDA-core kernel: q [rows, K/2] bytes (element 2j in the low
// nibble of byte j), s [rows, K/32] bytes.
//
// This path takes H and I multiples of 64 on weights prepared once
// (mx_tc_prepare: the scales in tensor-memory order; codes padded to whole
// 128-weight groups where H or I is not a multiple of 128, the 4-bit
// unpacking tensor maps taking only those), which covers gpt-oss's 2880 as
// well as PhiMoE-, Mixtral- and DeepSeek-shaped layers, and multiples of 128
// on the raw arrays; other shapes take the CUDA-core kernel.  The
// activations' last K-group is zero past K (tensor-map fill), so whatever
// padded weight codes meet there contribute nothing.  Per MMA (M = 128,
// N = 2 CH, K = 32):
//   A  128 weight rows.  TMA reads the packed codes with the 16U4_ALIGN16B
//      element type, which spreads every 16 codes (8 bytes in memory) over
//      16 bytes of shared memory: the layout this MMA kind reads 4-bit
//      operands from.  A stage holds 128 codes of each row (128 bytes in
//      shared memory, 128-byte swizzle).  GEMM 1 stacks 64 gate rows on the
//      64 matching up rows, GEMM 2 takes 128 rows of down.  Scale factors:
//      the weights' own E8M0 bytes.
//   B  the chunk's CH activation rows twice, as E4M3: row n holds
//      hi = e4m3(v 2^-e) and row CH + n holds lo = e4m3((v 2^-e - hi) 2^5),
//      with one E8M0 exponent e per 32 values (e - 5 for lo).  e puts the
//      block's largest magnitude in [128, 256); hi keeps 4 significant bits
//      and lo the next 4, so hi + lo is a bf16 value exactly unless a part
//      underflows E4M3.  Column n plus column CH + n of D is then the dot
//      product with the bf16 activations.
//   D  fp32 in tensor memory, 128 lanes x 2 CH columns, two buffers.
// Scale factors go to tensor memory with tcgen05.cp (32x128b.warpx4): per
// stage one 512-byte atom for A (byte 16 m0 + 4 m1 + kb holds the scale of
// row m0 + 32 m1, K-block kb of the stage) and one for B; the MMA's scale ids
// pick byte kb.
//
// Work item: (active expert, chunk of CH of its rows, 128 weight rows, split
// of the contraction).  The number of splits is chosen on the device, the
// same in every CTA, so that the items fill the grid in whole waves; each
// split writes an fp32 partial [split][slot][output row] and a small kernel
// sums the splits in order (deterministic), then applies SiLU(gate) * up
// (GEMM 1, which also quantises h for GEMM 2) or the routing weight (GEMM 2).
//
// Persistent CTAs of 192 threads, two or three per SM (MxTcCfg): a
// tcgen05 instruction costs its issuing thread a roughly fixed time whatever
// its size, so the SM moves more bytes with more issuing threads.  Stages of
// one K-group, weights as a 4D tensor-map box (the tile's two 64-row halves).
//   warp 0     producer: lane 0 issues the TMA boxes of a stage (the weight
//              tile, the hi and lo activation rows) and the bulk copies of
//              the activation scales and, on prepared weights, of the
//              stage's weight-scale atom; on raw weights all 32 lanes copy
//              the weight scale words with 4-byte cp.async and report them
//              on the stage barrier with cp.async.mbarrier.arrive;
//   warp 1     allocates tensor memory; one thread copies the stage's scale
//              factors to tensor memory and issues its four MMAs;
//   warps 2-5  epilogue: tcgen05.ld of their 32 lanes, hi + lo, fp32 partial
//              stores.
// Waits are bounded (MOE_ERR_TIMEOUT); on expiry the kernel drains its MMAs
// and frees its tensor memory.
#include "decode_common.cuh"
#include "gemm_common.cuh"

#include <cuda_fp8.h>

namespace moe {

namespace mxtc {
constexpr int THREADS = 192;
constexpr int KG = 128;                    // codes per K-group: 4 MMAs of K = 32, one SF word per row
constexpr int A_KG_SMEM = 128 * KG;        // 128 rows x 128 codes, one byte each in smem
constexpr int HALF_ROWS = 64;              // weight rows per half tile (GEMM 1: gate | up)
constexpr int SF_ATOM = 512;               // one scale-factor atom: 128 rows x 4 K-blocks
constexpr int MAX_SPLITS = 8;
constexpr int SPLIT_SLOTS = 128;           // splits x slots <= max(SPLIT_SLOTS, slots)
constexpr int MIN_KG_PER_SPLIT = 8;
constexpr int PREP_THREADS = 256;          // 8 warps, one 32-block each
constexpr int SMEM_BUDGET = 220 * 1024;
constexpr int SF_PAD_ROWS = 16;            // a chunk's copy of CH rows stays in the block
}  // namespace mxtc

// CTAs per SM (CPS) and K-groups per stage (KGS) by chunk size CH: as many
// CTAs as the shared and tensor memory allow while each keeps at least three
// stages (measured, PhiMoE shapes: CH = 8 at 3 CTAs 1.3x faster than 2 and
// 1.15x faster than 4; CH = 16 at 2 CTAs 2 % faster than 3).
template <int CH>
struct MxTcCfg {
    static constexpr int CPS = CH <= 8 ? 3 : 2;
    static constexpr int KGS = 1;
};

// Stage geometry: KGS K-groups (KGS x 128 codes of each of the tile's 128
// rows) per stage, CH activation rows per chunk.
template <int CH, int KGS, int CPS>
struct TcGeo {
    static constexpr int N = 2 * CH;                       // MMA N: hi and lo rows
    static constexpr int A_SMEM = KGS * mxtc::A_KG_SMEM;   // [kg][128 rows][128 B]
    static constexpr int A_TX = A_SMEM / 2;                // bytes TMA reads (and counts)
    static constexpr int B_KG = N * mxtc::KG;              // [hi CH rows | lo CH rows][128 B]
    static constexpr int B_SMEM = KGS * B_KG;
    static constexpr int SF_SMEM = 2 * KGS * mxtc::SF_ATOM;   // [kg] SFA atoms, then [kg] SFB
    static constexpr int STAGE = A_SMEM + B_SMEM + SF_SMEM;  // 1024-multiple
    static constexpr int TX = A_TX + B_SMEM;
    static constexpr int STAGES = (mxtc::SMEM_BUDGET / CPS - 1024 - 256) / STAGE;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE + 256;
    // NACC accumulators per buffer, MMA kb of a K-group adding into
    // accumulator kb % NACC, so that consecutive MMAs do not wait for each
    // other's result; two buffers (the epilogue of one item overlaps the
    // next item's MMAs); two scale-factor slots used by alternate K-groups
    // (as many as fit the tensor memory each of the CPS CTAs of an SM can hold)
    static constexpr int TMEM_LIMIT = CPS == 1 ? 512 : (CPS == 2 ? 256 : 128);
    static constexpr int NACC = 2 * 4 * N + 16 <= TMEM_LIMIT ? 4 : (2 * 2 * N + 16 <= TMEM_LIMIT ? 2 : 1);
    static constexpr int ACC_COLS = NACC * N;              // one buffer
    static constexpr int SF_COL = 2 * ACC_COLS;            // [2 slots][SFA 4 | SFB 4]
    static constexpr int COLS_USED = SF_COL + 16;
    static constexpr int TMEM_COLS = COLS_USED <= 32 ? 32 : COLS_USED <= 64 ? 64
                                   : COLS_USED <= 128 ? 128 : COLS_USED <= 256 ? 256 : 512;
    static_assert(TMEM_COLS <= TMEM_LIMIT, "tensor memory of CPS CTAs per SM");
    static_assert(STAGE % 1024 == 0, "stage must keep the 1024-byte swizzle alignment");
    static_assert(B_KG % 1024 == 0 && A_SMEM % 1024 == 0, "tiles must start on swizzle atoms");
    static_assert(STAGES >= 2 && 2 * STAGES + 5 <= 32, "stage count / barrier space");
};

struct MxTcParams {
    const int32_t* offsets;     // [E+1]
    const uint8_t* w_scales;    // [E * wrows, K/32] E8M0 of the weights (K a multiple of 128)
    const uint8_t* w_tiled;     // or: the weights' E8M0 in tensor-memory order (mx_tc_prepare)
    const uint8_t* act_sf;      // E8M0 of the activation planes, per K-group kg a block of
                                // sf_rows 16-byte rows (hi rows, lo rows at SP, padding):
                                // row r, K-block kb at (kg * sf_rows + r) * 16 + kb
    int sf_rows;                // 2 SP + SF_PAD_ROWS
    float* part;                // [splits][S][n_out] fp32 partial sums
    int32_t* ctl;               // ctl[0]: splits used (written by CTA 0)
    int32_t* err_flag;
    int S;                      // slots (T * k)
    int SP;                     // rows per activation plane (S rounded up to 32)
    int E;
    int K;                      // contraction (H for GEMM 1, I for GEMM 2)
    int I;                      // intermediate size (GEMM 1: offset of the up rows)
    int64_t wrows;              // weight rows per expert (2I or H)
    int n_out;                  // output rows per slot (2I or H)
    int mtiles;                 // 128-row weight tiles per expert (I / 64 or H / 128)
    uint64_t timeout_ns;
};

// D[tmem] (+)= (A . SFA) x (B . SFB)^T: E2M1 A and E4M3 B from shared memory,
// E8M0 scale factors from tensor memory, fp32 accumulation.
__device__ __forceinline__ void umma_mxf8f6f4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                              uint32_t idesc, uint32_t accumulate,
                                              uint32_t sfa_tmem, uint32_t sfb_tmem) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem),
        "r"(sfb_tmem));
}

// 32 rows x 128 bits of shared memory into tensor memory, the same 32 lanes
// repeated in each of the four lane quarters.
__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t src_desc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(src_desc));
}

// Source descriptor of one scale-factor atom: 32 rows of 16 bytes, no
// swizzle, 8-row groups 128 bytes apart.
__device__ __forceinline__ uint64_t smem_desc_sf(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);   // start address
    d |= static_cast<uint64_t>(128 >> 4) << 32;             // stride byte offset
    d |= static_cast<uint64_t>(1) << 46;                    // descriptor version (sm_100)
    return d;                                               // layout type 0: no swizzle
}

// Instruction descriptor, kind::mxf8f6f4 with block scaling: A E2M1, B E4M3,
// K-major both, E8M0 scale factors, M = 128, N = n.  The scale-factor ids
// (bits 4-5 for B, 29-30 for A) are or-ed in per MMA.
__host__ __device__ constexpr uint32_t idesc_mx_e2m1_e4m3(int n) {
    return (5u << 7) | (0u << 10) | (static_cast<uint32_t>(n >> 3) << 17) | (1u << 23) |
           (static_cast<uint32_t>(128 >> 4) << 24);
}

// 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
    uint32_t* r = reinterpret_cast<uint32_t*>(v);
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

__device__ __forceinline__ void cp_async4_tc(void* dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_arrive_noinc_tc(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// TMA tile loads of 3 and 4 dimensions (coordinates innermost first).
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1, int32_t c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}
// `bytes` (a multiple of 16) from a 16-byte aligned global address into this
// CTA's shared memory, counted on bar's transaction bytes.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1, int32_t c2, int32_t c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}
// Splits of the contraction, in whole stages of kgs K-groups: the count s <=
// MAX_SPLITS that minimises the bytes the busiest CTA moves, i.e. the waves
// of items, ceil(units s / grid), times the stages of an item, plus the
// split partials every split writes and the epilogue reads back (8 bytes per
// slot and output row, shared by the grid).  Each split keeps at least
// MIN_KG_PER_SPLIT K-groups and the partial buffer stays within
// max(SPLIT_SLOTS, S) slot rows.  The same in every CTA.
__host__ __device__ inline int mx_tc_splits(int units, int grid, int n_kg, int kgs, int S,
                                            int n_out) {
    const int n_st = (n_kg + kgs - 1) / kgs;
    const double stage_bytes = 128.0 * mxtc::KG / 2 * kgs;
    int best = 1;
    double best_cost = -1.0;
    for (int s = 1; s <= mxtc::MAX_SPLITS; ++s) {
        if (s > 1 && (static_cast<long long>(s) * S > (S > mxtc::SPLIT_SLOTS ? S : mxtc::SPLIT_SLOTS) ||
                      n_kg / s < mxtc::MIN_KG_PER_SPLIT))
            break;
        const long long items = static_cast<long long>(units) * s;
        const long long waves = (items + grid - 1) / grid;
        const long long stages = (n_st + s - 1) / s;
        const double cost = static_cast<double>(waves * stages) * stage_bytes +
                            8.0 * s * S * static_cast<double>(n_out) / grid;
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = s;
        }
    }
    return best;
}

// map_w: the packed codes as a 4D tensor (K codes, R1 rows, R2 row blocks, E
// experts) so that one box brings a K-group of a 128-row tile: per row 64
// contiguous bytes of memory; codes past K and row blocks past R2 read as
// zero.
//   GEMM 1: R1 = I (gate row), R2 = 2 (gate, up): box rows (mt*64.., 0..1)
//   GEMM 2: R1 = 64, R2 = H/64: box rows (0..63, 2mt..2mt+1)
// map_act: the E4M3 planes as a 3D tensor (K bytes, SP rows, 2 planes): box
// (128 bytes of a K-group, CH rows, both planes).
// TILED: the weight scales come as one 512-byte atom per (expert, tile,
// K-group), prepared once (mx_tc_prepare) in the order tensor memory takes
// them, and load with one bulk copy; otherwise (K a multiple of 128) each
// lane copies 4 scale words of the raw [rows, K/32] array.
template <int KIND, int CH, int KGS, int CPS, bool TILED>
__global__ void __launch_bounds__(mxtc::THREADS, CPS) decode_mx_tc_kernel(
    const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_act,
    const MxTcParams p) {
    using G = TcGeo<CH, KGS, CPS>;
    using namespace mxtc;
    static_assert(KGS == 1, "the tensor maps bring one K-group per box");
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ MxUnits act;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int splits_sh;

    uint8_t* ring = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(ring + G::STAGES * G::STAGE);
    uint64_t* empty = full + G::STAGES;
    uint64_t* tfull = empty + G::STAGES;    // [2]
    uint64_t* tempty = tfull + 2;           // [2]
    uint64_t* drain = tempty + 2;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nblk = p.K / 32;                  // raw scale row (not TILED: K % 128 == 0)
    const int n_kg = (p.K + KG - 1) / KG;       // K-groups of a whole contraction (last one
                                                // partial when K % 128 != 0: zero-filled)

    // launched as a programmatic dependent: barriers, descriptor prefetch and
    // tensor memory are set up while the previous kernel finishes; global
    // memory is touched only after pdl_wait
    pdl_launch_dependents();
    if (threadIdx.x == 0) {
        for (int i = 0; i < G::STAGES; ++i) {
            // expect_tx arrival (+ one cp.async arrival per lane for raw weight scales)
            mbar_init(&full[i], TILED ? 1 : 1 + 32);
            mbar_init(&empty[i], 1);        // tcgen05.commit
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 128);
        }
        mbar_init(drain, 1);
        fence_barrier_init();
        tma_prefetch_desc(&map_w);
        tma_prefetch_desc(&map_act);
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base_sh, G::TMEM_COLS);
        tmem_relinquish();
    }
    pdl_wait();
    const uint64_t deadline = global_ns() + p.timeout_ns;
    stage_offsets(act.offs, p.offsets, p.E);
    __syncthreads();
    if (threadIdx.x == 0) {
        build_mx_units(act, p.E, CH, p.mtiles);
        const int s = mx_tc_splits(act.total_units, gridDim.x, n_kg, KGS, p.S, p.n_out);
        splits_sh = s;
        if (blockIdx.x == 0) p.ctl[0] = s;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_sh;
    const int splits = splits_sh;
    const int n_items = act.total_units * splits;

    // item -> expert, chunk, weight tile and K-group range [kg0, kg1); splits
    // cut the contraction at stage boundaries, so only the last stage of a
    // whole contraction can hold fewer than KGS K-groups
    const int n_st = (n_kg + KGS - 1) / KGS;
    auto item_of = [&](int it, int& grp, int& chunk, int& mt, int& kg0, int& kg1) {
        const int u = it / splits, sp = it - (it / splits) * splits;
        const int ai = find_mx_unit(act, u);
        grp = act.gid[ai];
        const int local = u - act.unit_start[ai];
        chunk = local / p.mtiles;
        mt = local - chunk * p.mtiles;
        kg0 = ((sp * n_st) / splits) * KGS;
        kg1 = ((sp + 1) * n_st) / splits * KGS;
        if (kg1 > n_kg) kg1 = n_kg;
    };

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        bool ok = true;
        int f = 0;
        for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
            int grp, chunk, mt, kg0, kg1;
            item_of(it, grp, chunk, mt, kg0, kg1);
            const int brow0 = act.offs[grp] + chunk * CH;     // first slot row of the chunk
            // global rows of the tile: half h, row r -> h0 + h * hstride + r
            const int64_t h0 = static_cast<int64_t>(grp) * p.wrows +
                               (KIND == 0 ? static_cast<int64_t>(mt) * HALF_ROWS
                                          : static_cast<int64_t>(mt) * 128);
            const int64_t hstride = KIND == 0 ? p.I : HALF_ROWS;
            // this lane's scale words: word w = 32 j + lane of an A atom holds
            // row (w / 4) + 32 (w % 4), so each copy instruction fills 32
            // consecutive words (no bank conflicts)
            const uint8_t* wsrc[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int w = 32 * j + lane;
                const int m = (w >> 2) + 32 * (w & 3);
                wsrc[j] = TILED ? nullptr
                                : p.w_scales + (h0 + (m / HALF_ROWS) * hstride + (m % HALF_ROWS)) * nblk;
            }
            // TILED: this tile's scale atoms, one per K-group
            const uint8_t* tsrc = TILED ? p.w_tiled + (static_cast<int64_t>(grp) * p.mtiles + mt) *
                                                         n_kg * SF_ATOM
                                        : nullptr;
            for (int kg = kg0; kg < kg1; kg += KGS, ++f) {
                const int nk = kg1 - kg < KGS ? kg1 - kg : KGS;   // K-groups used in this stage
                const int slot = f % G::STAGES;
                const uint32_t ph = static_cast<uint32_t>(f / G::STAGES) & 1u;
                ok = __all_sync(0xffffffffu, mbar_wait(&empty[slot], ph ^ 1u, deadline));
                if (!ok) break;
                uint8_t* sa = ring + slot * G::STAGE;
                uint8_t* sb = sa + G::A_SMEM;
                uint8_t* sfa = sb + G::B_SMEM;
                uint8_t* sfb = sfa + KGS * SF_ATOM;
                if (lane == 0) {
                    // whole boxes always (codes past K and weight rows past the
                    // expert's are zero filled)
                    mbar_arrive_expect_tx(&full[slot],
                                          G::TX + 2 * CH * 16 + (TILED ? SF_ATOM : 0));
                    if (KIND == 0)
                        tma_load_4d(sa, &map_w, &full[slot], kg * KG, mt * HALF_ROWS, 0, grp);
                    else
                        tma_load_4d(sa, &map_w, &full[slot], kg * KG, 0, 2 * mt, grp);
                    tma_load_3d(sb, &map_act, &full[slot], kg * KG, brow0, 0);
                    if (TILED) bulk_load(sfa, tsrc + static_cast<int64_t>(kg) * SF_ATOM, SF_ATOM, &full[slot]);
                    // the chunk's activation scales: CH hi rows then CH lo rows,
                    // 16 bytes each, row n of the atom at byte 16 n (rows past
                    // the slots feed columns nothing reads)
                    const uint8_t* sfk = p.act_sf + static_cast<int64_t>(kg) * p.sf_rows * 16;
                    bulk_load(sfb, sfk + static_cast<int64_t>(brow0) * 16, CH * 16, &full[slot]);
                    bulk_load(sfb + CH * 16, sfk + static_cast<int64_t>(p.SP + brow0) * 16, CH * 16,
                              &full[slot]);
                }
                if (!TILED) {
                    for (int c = 0; c < nk; ++c) {
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            cp_async4_tc(sfa + c * SF_ATOM + 4 * (32 * j + lane), wsrc[j] + 4 * (kg + c), 4u);
                    }
                    cp_async_arrive_noinc_tc(&full[slot]);
                }
            }
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
        if (!ok && lane == 0) raise_error(p.err_flag, MOE_ERR_TIMEOUT);
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_mx_e2m1_e4m3(G::N);
            int sf_slot = 0;
            bool ok = true;
            int f = 0, acc = 0;
            uint32_t acc_phase = 0;
            for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
                int grp, chunk, mt, kg0, kg1;
                item_of(it, grp, chunk, mt, kg0, kg1);
                if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, deadline)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * G::ACC_COLS);
                for (int kg = kg0; kg < kg1; kg += KGS, ++f) {
                    const int nk = kg1 - kg < KGS ? kg1 - kg : KGS;
                    const int slot = f % G::STAGES;
                    const uint32_t ph = static_cast<uint32_t>(f / G::STAGES) & 1u;
                    if (!mbar_wait(&full[slot], ph, deadline)) { ok = false; break; }
                    tc_fence_after();
                    // the scale words arrived by cp.async (generic proxy); the
                    // copies below read them through the async proxy
                    fence_proxy_async_smem();
                    const uint32_t sa = smem_u32(ring + slot * G::STAGE);
                    const uint32_t sb = sa + G::A_SMEM;
                    const uint32_t sfa = sb + G::B_SMEM;
                    const uint32_t sfb = sfa + KGS * SF_ATOM;
                    for (int c = 0; c < nk; ++c) {
                        const uint32_t sfa_t = tmem_base + G::SF_COL + 8 * sf_slot;
                        const uint32_t sfb_t = sfa_t + 4;
                        sf_slot ^= 1;
                        tmem_cp_32x128b_x4(sfa_t, smem_desc_sf(sfa + c * SF_ATOM));
                        tmem_cp_32x128b_x4(sfb_t, smem_desc_sf(sfb + c * SF_ATOM));
#pragma unroll
                        for (int kb = 0; kb < KG / 32; ++kb) {
                            const uint64_t da = smem_desc_sw128(sa + c * A_KG_SMEM + 32 * kb);
                            const uint64_t db = smem_desc_sw128(sb + c * G::B_KG + 32 * kb);
                            const uint32_t id = idesc | (static_cast<uint32_t>(kb) << 29) |
                                                (static_cast<uint32_t>(kb) << 4);
                            // the first K-group of the item starts every accumulator
                            const bool fresh = kg == kg0 && c == 0 && kb < G::NACC;
                            umma_mxf8f6f4(d_tmem + static_cast<uint32_t>((kb % G::NACC) * G::N), da,
                                          db, id, fresh ? 0u : 1u, sfa_t, sfb_t);
                        }
                    }
                    umma_commit(&empty[slot]);
                }
                if (!ok) break;
                umma_commit(&tfull[acc]);
                if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
            }
            if (!ok) raise_error(p.err_flag, MOE_ERR_TIMEOUT);
            // all issued MMAs complete before the tensor memory is released
            umma_commit(drain);
            if (!mbar_wait(drain, 0, deadline + 1000000000ull))
                raise_error(p.err_flag, MOE_ERR_TIMEOUT);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int quarter = warp & 3;                  // TMEM lane quarter of this warp
        const int m = quarter * 32 + lane;             // weight row within the tile
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
            int grp, chunk, mt, kg0, kg1;
            item_of(it, grp, chunk, mt, kg0, kg1);
            if (!mbar_wait(&tfull[acc], acc_phase, deadline)) {
                raise_error(p.err_flag, MOE_ERR_TIMEOUT);
                break;
            }
            tc_fence_after();
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                   static_cast<uint32_t>(acc * G::ACC_COLS);
            float v[G::N];
#pragma unroll
            for (int c = 0; c < G::N; c += 16) tmem_ld16(taddr + c, v + c);
#pragma unroll
            for (int a = 1; a < G::NACC; ++a) {
                float w[G::N];
#pragma unroll
                for (int c = 0; c < G::N; c += 16)
                    tmem_ld16(taddr + static_cast<uint32_t>(a * G::N + c), w + c);
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < G::N; ++c) v[c] += w[c];
            }
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
            if (++acc == 2) { acc = 0; acc_phase ^= 1u; }

            const int sp = it - (it / splits) * splits;
            const int rows = act.offs[grp + 1] - act.offs[grp] - chunk * CH;
            const int brow0 = act.offs[grp] + chunk * CH;
            int n_o;
            if (KIND == 0)
                n_o = m < HALF_ROWS ? mt * HALF_ROWS + m : p.I + mt * HALF_ROWS + (m - HALF_ROWS);
            else
                n_o = mt * 128 + m;
            float* dst = p.part + (static_cast<int64_t>(sp) * p.S + brow0) * p.n_out + n_o;
            const bool row_in = KIND == 0 || n_o < p.n_out;   // GEMM 2: tile rows past H
#pragma unroll
            for (int c = 0; c < CH; ++c)
                if (c < rows && row_in) dst[static_cast<int64_t>(c) * p.n_out] = v[c] + v[CH + c];
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, G::TMEM_COLS);
    }
}

// ---------------------------------------------------------------- activations

// v (one value of a 32-block whose largest magnitude is bmax) as the E4M3
// pair (hi, lo) and the block's E8M0 exponents: v ~ 2^eh hi + 2^el lo.
__device__ __forceinline__ void e4m3_pair(float v, float bmax, uint8_t& hi, uint8_t& lo,
                                          int& eh, int& el) {
    const int be = static_cast<int>((__float_as_uint(bmax) >> 23) & 0xffu);
    if (be == 0) {            // all-zero (or subnormal) block
        hi = lo = 0;
        eh = el = 0;
        return;
    }
    eh = be - 127 - 7;        // the block maximum lands in [128, 256)
    eh = eh < -127 ? -127 : (eh > 127 ? 127 : eh);
    el = eh - 5 < -127 ? -127 : eh - 5;
    const float a = v * __uint_as_float(static_cast<uint32_t>(127 - eh) << 23);    // exact
    hi = static_cast<uint8_t>(__nv_cvt_float_to_fp8(a, __NV_SATFINITE, __NV_E4M3));
    const float ah = __half2float(__half(__nv_cvt_fp8_to_halfraw(hi, __NV_E4M3)));
    const float r = (a - ah) * __uint_as_float(static_cast<uint32_t>(127 + eh - el) << 23);
    lo = static_cast<uint8_t>(__nv_cvt_float_to_fp8(r, __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ float warp_max_abs(float v) {
    float m = fabsf(v);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    return m;
}

// Byte of activation scale row r, 32-block blk, in the layout the kernel
// copies per K-group (MxTcParams::act_sf).
__device__ __forceinline__ int64_t act_sf_byte(int64_t r, int blk, int sf_rows) {
    return ((static_cast<int64_t>(blk >> 2) * sf_rows) + r) * 16 + (blk & 3);
}

// One warp per (slot row, 32-block): writes the value's hi byte to plane 0
// (row r) and lo byte to plane 1 (row SP + r), and the exponents likewise.
__device__ __forceinline__ void store_e4m3_pair(float v, int64_t r, int blk, int K, int SP,
                                                int sf_rows, uint8_t* q, uint8_t* sf) {
    const int lane = threadIdx.x & 31;
    const float bmax = warp_max_abs(v);
    uint8_t hi, lo;
    int eh, el;
    e4m3_pair(v, bmax, hi, lo, eh, el);
    q[r * K + blk * 32 + lane] = hi;
    q[(SP + r) * K + blk * 32 + lane] = lo;
    if (lane == 0) {
        sf[act_sf_byte(r, blk, sf_rows)] = static_cast<uint8_t>(eh + 127);
        sf[act_sf_byte(SP + r, blk, sf_rows)] = static_cast<uint8_t>(el + 127);
    }
}

// Scale bytes of the blocks past K that fill the last K-group (K % 128 != 0):
// 2^0, a finite factor for codes the tensor map reads as zero.  True when
// `blk` is such a block (written) or past the last K-group (nothing to do).
__device__ __forceinline__ bool pad_scale_block(int64_t r, int blk, int K, int SP, int sf_rows,
                                                uint8_t* sf) {
    if (blk < K / 32) return false;
    if (blk < (K + mxtc::KG - 1) / mxtc::KG * 4 && (threadIdx.x & 31) == 0) {
        sf[act_sf_byte(r, blk, sf_rows)] = 127;
        sf[act_sf_byte(SP + r, blk, sf_rows)] = 127;
    }
    return true;
}

// GEMM 1 operand B: x[perm[r] / k] of every sorted slot row r.
__global__ void __launch_bounds__(mxtc::PREP_THREADS) mx_tc_prep_x_kernel(
    const __nv_bfloat16* __restrict__ x, const int32_t* __restrict__ perm, int k, int K, int SP,
    int sf_rows, uint8_t* __restrict__ q, uint8_t* __restrict__ sf) {
    pdl_launch_dependents();
    pdl_wait();
    const int r = blockIdx.y;
    const int blk = blockIdx.x * (mxtc::PREP_THREADS / 32) + (threadIdx.x >> 5);
    if (pad_scale_block(r, blk, K, SP, sf_rows, sf)) return;
    const int64_t tok = perm[r] / k;
    const float v = __bfloat162float(x[tok * K + blk * 32 + (threadIdx.x & 31)]);
    store_e4m3_pair(v, r, blk, K, SP, sf_rows, q, sf);
}

// GEMM 1 epilogue: gate and up summed over the splits in order, h =
// SiLU(gate) * up rounded to bf16, then quantised as GEMM 2's operand B.
__global__ void __launch_bounds__(mxtc::PREP_THREADS) mx_tc_swiglu_kernel(
    const float* __restrict__ part, const int32_t* __restrict__ ctl, int S, int I, int SP,
    int sf_rows, uint8_t* __restrict__ q, uint8_t* __restrict__ sf) {
    pdl_launch_dependents();
    pdl_wait();
    const int r = blockIdx.y;
    const int blk = blockIdx.x * (mxtc::PREP_THREADS / 32) + (threadIdx.x >> 5);
    if (pad_scale_block(r, blk, I, SP, sf_rows, sf)) return;
    const int i = blk * 32 + (threadIdx.x & 31);
    const int splits = ctl[0];
    float g = 0.f, u = 0.f;
    for (int s = 0; s < splits; ++s) {
        const float* row = part + (static_cast<int64_t>(s) * S + r) * (2 * static_cast<int64_t>(I));
        g += row[i];
        u += row[I + i];
    }
    const float h = __bfloat162float(__float2bfloat16_rn(g / (1.f + __expf(-g)) * u));
    store_e4m3_pair(h, r, blk, I, SP, sf_rows, q, sf);
}

// GEMM 2 epilogue: y_slots[r] = routed_scale * topk_w[perm[r]] * sum over splits.
__global__ void __launch_bounds__(256) mx_tc_down_out_kernel(
    const float* __restrict__ part, const int32_t* __restrict__ ctl, const int32_t* __restrict__ perm,
    const float* __restrict__ topk_w, float routed_scale, int S, int H,
    __nv_bfloat16* __restrict__ y_slots) {
    pdl_launch_dependents();
    pdl_wait();
    const int r = blockIdx.y;
    const int n = blockIdx.x * 256 + threadIdx.x;
    if (n >= H) return;
    const int splits = ctl[0];
    float acc = 0.f;
    for (int s = 0; s < splits; ++s) acc += part[(static_cast<int64_t>(s) * S + r) * H + n];
    const float w = routed_scale * topk_w[perm[r]];
    y_slots[static_cast<int64_t>(r) * H + n] = __float2bfloat16_rn(w * acc);
}

// ------------------------------------------------------------------ launcher

// Packed E2M1 codes [E * wrows, K/2 bytes] read as 16U4_ALIGN16B (each 16
// codes land in 16 bytes of shared memory, 128-byte swizzle) through the 4D
// view described above the kernel; box (128 codes, 64 rows, 2 row blocks, 1
// expert).
static bool make_map_e2m1(CUtensorMap* map, const void* base, int E, int64_t wrows, int64_t K,
                          int64_t r1, int64_t r2, int64_t r1_rows_stride) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc || E <= 0 || K <= 0 || K % 32 != 0) return false;
    const cuuint64_t row_bytes = static_cast<cuuint64_t>(K / 2);
    cuuint64_t dims[4] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(r1),
                          static_cast<cuuint64_t>(r2), static_cast<cuuint64_t>(E)};
    cuuint64_t strides[3] = {row_bytes, row_bytes * static_cast<cuuint64_t>(r1_rows_stride),
                             row_bytes * static_cast<cuuint64_t>(wrows)};
    cuuint32_t box[4] = {static_cast<cuuint32_t>(mxtc::KG), static_cast<cuuint32_t>(mxtc::HALF_ROWS),
                         2u, 1u};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 4, const_cast<void*>(base), dims,
               strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// E4M3 activation planes [2 * SP rows, K bytes] as a 3D tensor (K bytes, SP
// rows, 2 planes); box (128 bytes of a K-group, ch rows, 2 planes), 128-byte
// swizzle; bytes past K read as zero.
static bool make_map_e4m3(CUtensorMap* map, const void* base, int64_t SP, int64_t K, int ch) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc || SP <= 0 || K <= 0 || K % 32 != 0) return false;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(SP), 2u};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(SP * K)};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(mxtc::KG), static_cast<cuuint32_t>(ch), 2u};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Rows of each activation plane: the slots rounded up to 32 (at least one
// box of CH rows for every CH used here).
int64_t mx_tc_plane_rows(int64_t slots) { return (slots + 31) / 32 * 32; }

// Float count of the split partials: max(SPLIT_SLOTS, slots) x max(2I, H).
int64_t mx_tc_part_floats(int64_t slots, int H, int I) {
    const int64_t rows = slots > mxtc::SPLIT_SLOTS ? slots : mxtc::SPLIT_SLOTS;
    const int64_t cols = 2 * static_cast<int64_t>(I) > H ? 2 * static_cast<int64_t>(I) : H;
    return rows * cols;
}

// 32-blocks of a row in whole K-groups (the prep kernels' grid).
static int mx_tc_blocks(int K) { return (K + mxtc::KG - 1) / mxtc::KG * 4; }
// Rows of an activation scale block per K-group.
int mx_tc_sf_rows(int64_t SP) { return static_cast<int>(2 * SP + mxtc::SF_PAD_ROWS); }

// The prepared weights of the tensor-core path (mx_tc_prepare), in this
// order, each part 256-byte aligned:
//   tiled scales, GEMM 1: one SF_ATOM per (expert, I/64 tiles, ceil(H/128)
//     K-groups); GEMM 2: per (expert, ceil(H/128) tiles, ceil(I/128) K-groups)
//   when H % 128 != 0: gate_up codes with rows padded by zero codes to a
//     multiple of 128 weights [E, 2I, Hp/2];  when I % 128 != 0: down codes
//     likewise [E, H, Ip/2]
// (the 4-bit unpacking tensor maps take rows of whole 128-weight K-groups
// only).  0 bytes when the tensor-core kernel cannot take the shape.
static int64_t align256(int64_t v) { return (v + 255) / 256 * 256; }
static int64_t round128(int64_t v) { return (v + 127) / 128 * 128; }
static int64_t mx_tc_tiled_gu_bytes(const moe_shape& s) {
    return static_cast<int64_t>(mxtc::SF_ATOM) * s.E * (s.I / mxtc::HALF_ROWS) *
           ((s.H + mxtc::KG - 1) / mxtc::KG);
}
static int64_t mx_tc_tiled_dn_bytes(const moe_shape& s) {
    return static_cast<int64_t>(mxtc::SF_ATOM) * s.E * ((s.H + 127) / 128) *
           ((s.I + mxtc::KG - 1) / mxtc::KG);
}
static int64_t mx_tc_gu_pad_bytes(const moe_shape& s) {
    return s.H % 128 ? static_cast<int64_t>(s.E) * 2 * s.I * (round128(s.H) / 2) : 0;
}
static int64_t mx_tc_dn_pad_bytes(const moe_shape& s) {
    return s.I % 128 ? static_cast<int64_t>(s.E) * s.H * (round128(s.I) / 2) : 0;
}
int64_t mx_tc_prepared_bytes(const moe_shape& s) {
    if (s.H % 64 != 0 || s.I % 64 != 0 || s.H <= 0 || s.I <= 0) return 0;
    return align256(mx_tc_tiled_gu_bytes(s)) + align256(mx_tc_tiled_dn_bytes(s)) +
           align256(mx_tc_gu_pad_bytes(s)) + align256(mx_tc_dn_pad_bytes(s));
}
struct MxPrepared {
    const uint8_t* tiled;        // GEMM 1's atoms, then GEMM 2's at tiled_dn
    const uint8_t* tiled_dn;
    const uint8_t* gu_codes;     // padded copies, or NULL (use the caller's codes)
    const uint8_t* dn_codes;
};
static MxPrepared mx_tc_prepared_parts(const moe_shape& s, const void* base) {
    const uint8_t* b = static_cast<const uint8_t*>(base);
    MxPrepared m;
    m.tiled = b;
    m.tiled_dn = b + align256(mx_tc_tiled_gu_bytes(s));
    const uint8_t* pads = m.tiled_dn + align256(mx_tc_tiled_dn_bytes(s));
    m.gu_codes = mx_tc_gu_pad_bytes(s) ? pads : nullptr;
    m.dn_codes = mx_tc_dn_pad_bytes(s) ? pads + align256(mx_tc_gu_pad_bytes(s)) : nullptr;
    return m;
}

// Rows of K/2 code bytes copied into rows of Kp/2 bytes, the rest zero (16-byte
// vectors: K % 32 == 0, Kp % 128 == 0).
__global__ void __launch_bounds__(256) mx_tc_pad_codes_kernel(const uint4* __restrict__ src,
                                                              uint4* __restrict__ dst,
                                                              int64_t rows, int K, int Kp) {
    const int vin = K / 32, vout = Kp / 32;      // 16-byte vectors per row
    const int64_t n = rows * vout;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = i / vout;
        const int v = static_cast<int>(i - r * vout);
        dst[i] = v < vin ? src[r * vin + v] : make_uint4(0u, 0u, 0u, 0u);
    }
}

// The weight scales of both GEMMs in the order the tensor-core kernel copies
// them into tensor memory: per (expert, tile, K-group) an atom whose byte
// 4 w + kb is the scale of tile row (w >> 2) + 32 (w & 3), K-block 4 kg + kb
// (GEMM 1 tile rows: 64 gate rows, then the 64 up rows of the same columns);
// rows past the expert's and K-blocks past K/32 hold 127 (2^0, against codes
// the tensor maps read as zero).  One thread per 4-byte word.
__global__ void __launch_bounds__(256) mx_tc_tile_scales_kernel(
    const uint8_t* __restrict__ gu_s, const uint8_t* __restrict__ dn_s,
    uint32_t* __restrict__ out, int E, int H, int I, int64_t n_gu_words, int64_t n_words) {
    for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < n_words;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const bool gu = idx < n_gu_words;
        const int64_t j = gu ? idx : idx - n_gu_words;
        const int K = gu ? H : I;
        const int nkb = K / 32;
        const int n_kg = (K + mxtc::KG - 1) / mxtc::KG;
        const int mtiles = gu ? I / mxtc::HALF_ROWS : (H + 127) / 128;
        const int w = static_cast<int>(j % 128);
        const int64_t t = j / 128;
        const int kg = static_cast<int>(t % n_kg);
        const int mt = static_cast<int>((t / n_kg) % mtiles);
        const int e = static_cast<int>(t / (static_cast<int64_t>(n_kg) * mtiles));
        const int m = (w >> 2) + 32 * (w & 3);
        int64_t row;          // within the expert
        bool valid;
        if (gu) {
            row = m < mxtc::HALF_ROWS ? static_cast<int64_t>(mt) * mxtc::HALF_ROWS + m
                                      : I + static_cast<int64_t>(mt) * mxtc::HALF_ROWS + (m - mxtc::HALF_ROWS);
            valid = true;
        } else {
            row = static_cast<int64_t>(mt) * 128 + m;
            valid = row < H;
        }
        const uint8_t* src = (gu ? gu_s + (static_cast<int64_t>(e) * 2 * I + row) * nkb
                                 : dn_s + (static_cast<int64_t>(e) * H + row) * nkb);
        uint32_t word = 0;
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) {
            const int blk = 4 * kg + kb;
            const uint32_t v = (valid && blk < nkb) ? src[blk] : 127u;
            word |= v << (8 * kb);
        }
        out[idx] = word;
    }
}

static int grid_of(int64_t n, int num_sms) {
    const int64_t want = (n + 255) / 256;
    return static_cast<int>(want < 8 * num_sms ? (want > 0 ? want : 1) : 8 * num_sms);
}

// Fills the prepared weights (layout above mx_tc_prepared_bytes).
cudaError_t launch_mx_tc_prepare(const moe_shape& s, const uint8_t* gu_q, const uint8_t* gu_s,
                                 const uint8_t* dn_q, const uint8_t* dn_s, void* out, int num_sms,
                                 cudaStream_t st) {
    if (mx_tc_prepared_bytes(s) <= 0) return cudaErrorInvalidValue;
    const MxPrepared m = mx_tc_prepared_parts(s, out);
    // the scale atoms of GEMM 2 follow GEMM 1's after its 256-byte padding:
    // two launches, one per GEMM, each with its own word range
    const int64_t n_gu = mx_tc_tiled_gu_bytes(s) / 4, n_dn = mx_tc_tiled_dn_bytes(s) / 4;
    mx_tc_tile_scales_kernel<<<grid_of(n_gu, num_sms), 256, 0, st>>>(
        gu_s, dn_s, reinterpret_cast<uint32_t*>(const_cast<uint8_t*>(m.tiled)), s.E, s.H, s.I,
        n_gu, n_gu);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    mx_tc_tile_scales_kernel<<<grid_of(n_dn, num_sms), 256, 0, st>>>(
        gu_s, dn_s, reinterpret_cast<uint32_t*>(const_cast<uint8_t*>(m.tiled_dn)), s.E, s.H, s.I,
        0, n_dn);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (m.gu_codes) {
        const int64_t rows = static_cast<int64_t>(s.E) * 2 * s.I;
        const int Kp = static_cast<int>(round128(s.H));
        mx_tc_pad_codes_kernel<<<grid_of(rows * (Kp / 32), num_sms), 256, 0, st>>>(
            reinterpret_cast<const uint4*>(gu_q), reinterpret_cast<uint4*>(const_cast<uint8_t*>(m.gu_codes)),
            rows, s.H, Kp);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (m.dn_codes) {
        const int64_t rows = static_cast<int64_t>(s.E) * s.H;
        const int Kp = static_cast<int>(round128(s.I));
        mx_tc_pad_codes_kernel<<<grid_of(rows * (Kp / 32), num_sms), 256, 0, st>>>(
            reinterpret_cast<const uint4*>(dn_q), reinterpret_cast<uint4*>(const_cast<uint8_t*>(m.dn_codes)),
            rows, s.I, Kp);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

// The tensor-core path takes H and I multiples of 64 with the prepared
// weights, of 128 with the raw ones (whole 4-byte scale words per row).
bool mx_tc_supported(const moe_shape& s, const void* gu_q, const void* dn_q, bool prepared) {
    const bool shape_ok = prepared ? (s.H % 64 == 0 && s.I % 64 == 0)
                                : (s.H % 128 == 0 && s.I % 128 == 0);
    return shape_ok && s.T >= 1 && s.T <= 64 &&
           (reinterpret_cast<uintptr_t>(gu_q) & 31u) == 0 &&
           (reinterpret_cast<uintptr_t>(dn_q) & 31u) == 0;
}

template <int KIND, int CH, int KGS, int CPS, bool TILED>
static cudaError_t launch_tc(const CUtensorMap& mw, const CUtensorMap& ma, const MxTcParams& p,
                             int num_sms, cudaStream_t st) {
    using G = TcGeo<CH, KGS, CPS>;
    auto kern = decode_mx_tc_kernel<KIND, CH, KGS, CPS, TILED>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         G::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, dim3(CPS * num_sms), dim3(mxtc::THREADS), G::SMEM_BYTES, st, mw, ma, p);
}

template <int CH, int KGS, int CPS, bool TILED>
static cudaError_t run_tc(const moe_shape& s, const void* x, const int32_t* offsets,
                          const int32_t* perm, const float* topk_w, const uint8_t* gu_q,
                          const uint8_t* gu_s, const uint8_t* dn_q, const uint8_t* dn_s,
                          const void* prepared, uint8_t* xq, uint8_t* xsf, uint8_t* hq,
                          uint8_t* hsf, float* part, int32_t* ctl, void* y_slots,
                          int32_t* err_flag, int num_sms, cudaStream_t st) {
    const int S = static_cast<int>(s.T * s.k);
    const int SP = static_cast<int>(mx_tc_plane_rows(S));
    const MxPrepared m = TILED ? mx_tc_prepared_parts(s, prepared)
                               : MxPrepared{nullptr, nullptr, nullptr, nullptr};
    // codes: the padded copies where a row is not whole K-groups
    const uint8_t* gu_codes = m.gu_codes ? m.gu_codes : gu_q;
    const uint8_t* dn_codes = m.dn_codes ? m.dn_codes : dn_q;
    const int64_t Kg = m.gu_codes ? round128(s.H) : s.H, Kd = m.dn_codes ? round128(s.I) : s.I;
    CUtensorMap map_gu, map_dn, map_x, map_h;
    // GEMM 1 rows: gate row i of expert e at e*2I + i, up at e*2I + I + i
    // GEMM 2 rows: row n of expert e at e*H + n, blocks of 64
    if (!make_map_e2m1(&map_gu, gu_codes, s.E, 2 * static_cast<int64_t>(s.I), Kg, s.I, 2, s.I) ||
        !make_map_e2m1(&map_dn, dn_codes, s.E, s.H, Kd, mxtc::HALF_ROWS, s.H / mxtc::HALF_ROWS,
                       mxtc::HALF_ROWS) ||
        !make_map_e4m3(&map_x, xq, SP, s.H, CH) || !make_map_e4m3(&map_h, hq, SP, s.I, CH))
        return cudaErrorInvalidValue;
    const int nb_x = mx_tc_blocks(s.H), nb_h = mx_tc_blocks(s.I);
    const int sf_rows = mx_tc_sf_rows(SP);

    constexpr int WPB = mxtc::PREP_THREADS / 32;
    cudaError_t e = launch_pdl(mx_tc_prep_x_kernel, dim3((nb_x + WPB - 1) / WPB, S),
                               dim3(mxtc::PREP_THREADS), 0, st,
                               static_cast<const __nv_bfloat16*>(x), perm, s.k, s.H, SP, sf_rows,
                               xq, xsf);
    if (e != cudaSuccess) return e;

    MxTcParams p{};
    p.offsets = offsets;
    p.part = part;
    p.ctl = ctl;
    p.err_flag = err_flag;
    p.S = S;
    p.SP = SP;
    p.E = s.E;
    p.I = s.I;
    p.timeout_ns = 4000000000ull;
    // GEMM 1: gate_up, K = H, 64 gate + 64 up rows per tile
    p.w_scales = gu_s;
    p.w_tiled = m.tiled;
    p.act_sf = xsf;
    p.sf_rows = sf_rows;
    p.K = s.H;
    p.wrows = 2 * static_cast<int64_t>(s.I);
    p.n_out = 2 * s.I;
    p.mtiles = s.I / mxtc::HALF_ROWS;
    e = launch_tc<0, CH, KGS, CPS, TILED>(map_gu, map_x, p, num_sms, st);
    if (e != cudaSuccess) return e;
    e = launch_pdl(mx_tc_swiglu_kernel, dim3((nb_h + WPB - 1) / WPB, S),
                   dim3(mxtc::PREP_THREADS), 0, st, part, ctl, S, s.I, SP, sf_rows, hq, hsf);
    if (e != cudaSuccess) return e;
    // GEMM 2: down, K = I, 128 rows per tile (the last one partial when H % 128 != 0)
    p.w_scales = dn_s;
    p.w_tiled = m.tiled_dn;
    p.act_sf = hsf;
    p.K = s.I;
    p.wrows = s.H;
    p.n_out = s.H;
    p.mtiles = (s.H + 127) / 128;
    e = launch_tc<1, CH, KGS, CPS, TILED>(map_dn, map_h, p, num_sms, st);
    if (e != cudaSuccess) return e;
    return launch_pdl(mx_tc_down_out_kernel, dim3((s.H + 255) / 256, S), dim3(256), 0, st, part,
                      ctl, perm, topk_w, s.routed_scale, S, s.H,
                      static_cast<__nv_bfloat16*>(y_slots));
}

template <bool TILED>
static cudaError_t run_tc_t(const moe_shape& s, const void* x, const int32_t* offsets,
                            const int32_t* perm, const float* topk_w, const uint8_t* gu_q,
                            const uint8_t* gu_s, const uint8_t* dn_q, const uint8_t* dn_s,
                            const void* prepared, uint8_t* xq, uint8_t* xsf, uint8_t* hq,
                            uint8_t* hsf, float* part, int32_t* ctl, void* y_slots,
                            int32_t* err_flag, int num_sms, cudaStream_t st) {
    if (s.T <= 8)
        return run_tc<8, MxTcCfg<8>::KGS, MxTcCfg<8>::CPS, TILED>(
            s, x, offsets, perm, topk_w, gu_q, gu_s, dn_q, dn_s, prepared, xq, xsf, hq, hsf, part,
            ctl, y_slots, err_flag, num_sms, st);
    return run_tc<16, MxTcCfg<16>::KGS, MxTcCfg<16>::CPS, TILED>(
        s, x, offsets, perm, topk_w, gu_q, gu_s, dn_q, dn_s, prepared, xq, xsf, hq, hsf, part,
        ctl, y_slots, err_flag, num_sms, st);
}

// moe_forward_mxfp4 on the block-scaled tensor cores (mx_tc_supported), with
// the raw weights (prepared == NULL) or the prepared ones: chunks of 8 rows
// per expert for batches of up to 8 tokens, else 16.  An expert with more
// rows than a chunk streams its weights once per chunk (at T = 64 over 16
// experts a few do; chunks of 32 rows, which avoid that but fit only two CTAs
// per SM with a single accumulator, measured 8 % slower).  Several CTAs per
// SM: each tcgen05 instruction costs its issuing thread a roughly fixed time,
// so more issuing threads per SM move more bytes (MxTcCfg: CTAs per SM and
// K-groups per stage by chunk size).
cudaError_t launch_ffn_decode_mxfp4_tc(const moe_shape& s, const void* x, const int32_t* offsets,
                                       const int32_t* perm, const float* topk_w,
                                       const uint8_t* gu_q, const uint8_t* gu_s,
                                       const uint8_t* dn_q, const uint8_t* dn_s,
                                       const void* prepared, uint8_t* xq, uint8_t* xsf,
                                       uint8_t* hq, uint8_t* hsf, float* part, int32_t* ctl,
                                       void* y_slots, int32_t* err_flag, int num_sms,
                                       cudaStream_t st) {
    if (!mx_tc_supported(s, gu_q, dn_q, prepared != nullptr) || s.dtype != MOE_BF16 ||
        s.n_shared != 0)
        return cudaErrorInvalidValue;
    if (prepared)
        return run_tc_t<true>(s, x, offsets, perm, topk_w, gu_q, gu_s, dn_q, dn_s, prepared, xq,
                              xsf, hq, hsf, part, ctl, y_slots, err_flag, num_sms, st);
    return run_tc_t<false>(s, x, offsets, perm, topk_w, gu_q, gu_s, dn_q, dn_s, prepared, xq,
                           xsf, hq, hsf, part, ctl, y_slots, err_flag, num_sms, st);
}

}  // namespace moe
