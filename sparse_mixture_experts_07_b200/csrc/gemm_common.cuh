// Definitions shared by the grouped-GEMM kernels (one-CTA and CTA-pair
// variants): launch parameters, tile decoding, TMA tensor maps.
#pragma once

#include "common.cuh"

namespace moe {

enum : int { kSwiGLU = 0, kScaled = 1 };

struct GemmParams {
    const int32_t* offsets;   // [E+1]
    const int32_t* perm;      // [T*k]
    const float* topk_w;      // [T*k]
    int64_t T;
    int E, S, k;
    int n_tiles_routed, n_tiles_shared;
    int K_routed, K_shared;          // contraction length
    int N_routed, N_shared;          // valid output columns
    int b_rows_routed, b_rows_shared;  // B rows per expert (2I / H)
    int half_routed, half_shared;      // kSwiGLU: offset of the up rows (I / Is)
    void* out_routed;
    void* out_shared;
    int64_t ld_routed, ld_shared;      // output row strides (elements)
    int64_t out_row0_shared;           // kScaled: first y_slots row of shared outputs
    float routed_scale;
    int group_m;
    int32_t* err_flag;
    uint64_t timeout_ns;
    // kSwiGLU, training forward: also store the pre-activations [g | u] of
    // every row (bf16, row stride 2N) for the backward pass; NULL: do not
    void* gu_routed;
    void* gu_shared;
};

// Stores 32 gate and 32 up values of one row as bf16 into gu (row stride 2N,
// gate at column n, up at N + n), 16-byte vectors, columns < N only.
__device__ __forceinline__ void store_gu32(__nv_bfloat16* gu_row, int n, int N,
                                           const float (&gv)[32], const float (&uv)[32]) {
#pragma unroll
    for (int v = 0; v < 4; ++v) {
        if (n + 8 * v >= N) break;
        uint32_t g4[4], u4[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            g4[j] = pack_bf16x2(gv[8 * v + 2 * j], gv[8 * v + 2 * j + 1]);
            u4[j] = pack_bf16x2(uv[8 * v + 2 * j], uv[8 * v + 2 * j + 1]);
        }
        *reinterpret_cast<uint4*>(gu_row + n + 8 * v) = make_uint4(g4[0], g4[1], g4[2], g4[3]);
        *reinterpret_cast<uint4*>(gu_row + N + n + 8 * v) = make_uint4(u4[0], u4[1], u4[2], u4[3]);
    }
}

struct TileCoord {
    int g;          // group
    int m0;         // first row within the group
    int n0;         // first output column
    int rows;       // rows of the group
    bool routed;
};

template <int MAXG>
__device__ __forceinline__ TileCoord decode_tile(const GroupTableT<MAXG>& gt, const GemmParams& p,
                                                 int tile, int n_cols_per_tile, int BM) {
    TileCoord c;
    c.g = find_group(gt, tile);
    c.routed = c.g < p.E;
    c.rows = gt.rows[c.g];
    const int local = tile - gt.tile_start[c.g];
    const int nt = c.routed ? p.n_tiles_routed : p.n_tiles_shared;
    const int mt = (c.rows + BM - 1) / BM;
    const int band = local / (p.group_m * nt);
    const int within = local - band * p.group_m * nt;
    const int m_base = band * p.group_m;
    const int gm = min(p.group_m, mt - m_base);
    c.n0 = (within / gm) * n_cols_per_tile;
    c.m0 = (m_base + within % gm) * BM;
    return c;
}

// ---------------------------------------------------------------------------
// Host side: tensor maps.

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// 2D bf16 row-major [rows, cols], box = 64 columns x box_rows rows, 128-byte swizzle.
inline bool make_map(CUtensorMap* map, const void* base, int64_t rows, int64_t cols,
                     int box_rows) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc || rows <= 0 || cols <= 0) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
    cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace moe
