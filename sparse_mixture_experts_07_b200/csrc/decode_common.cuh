// Helpers shared by the decode (weight-streaming) kernels: the list of active
// expert groups and their work units, the warp-level bf16 / f16 MMA, bounded
// predicated loads, the split of a contraction over a CTA's warps, and the
// reduction of the warps' partial fragments.
#pragma once

#include "common.cuh"

namespace moe {

namespace dec {
constexpr int WARPS = 4;
constexpr int THREADS = WARPS * 32;
constexpr int MAX_ROWS = 8;      // rows per group handled here
constexpr int UNROLL = 8;        // 32-element k-steps in flight per warp
}  // namespace dec

// Active groups (routed experts with slots, then shared experts) and the
// prefix of their work units.
struct ActiveGroups {
    int n;
    int total_units;
    int gid[kMaxGroups];
    int unit_start[kMaxGroups + 1];
    int32_t offs[kMaxExperts + 1];   // the routed experts' offsets (stage_offsets)
};

// Groups 0..E-1 are routed experts (rows from offsets), E..E+S-1 shared
// experts (T rows each); a group's work units cover its ncols output
// columns 16 at a time.
// Built by one thread from a.offs, which stage_offsets filled.
__device__ __forceinline__ void build_active(ActiveGroups& a, int E, int S, int64_t T,
                                             int ncols_routed, int ncols_shared) {
    const int32_t* offsets = a.offs;
    int n = 0, acc = 0;
    for (int g = 0; g < E + S; ++g) {
        const bool routed = g < E;
        const int rows = routed ? offsets[g + 1] - offsets[g] : static_cast<int>(T);
        if (rows <= 0) continue;
        const int ncols = routed ? ncols_routed : ncols_shared;
        a.gid[n] = g;
        a.unit_start[n] = acc;
        acc += (ncols + 15) / 16;
        ++n;
    }
    a.unit_start[n] = acc;
    a.n = n;
    a.total_units = acc;
}

__device__ __forceinline__ int find_active(const ActiveGroups& a, int unit) {
    int lo = 0, hi = a.n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a.unit_start[mid] <= unit) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// Expert groups with rows, each with ceil(rows / chunk_rows) chunks of
// units_per_chunk work units (the MXFP4 decode kernels).  Built by one thread
// from a.offs, which stage_offsets filled.
struct MxUnits {
    int n;
    int total_units;
    int gid[kMaxExperts];
    int unit_start[kMaxExperts + 1];
    int32_t offs[kMaxExperts + 1];
};

__device__ __forceinline__ void build_mx_units(MxUnits& a, int E, int chunk_rows,
                                               int units_per_chunk) {
    int n = 0, acc = 0;
    for (int g = 0; g < E; ++g) {
        const int rows = a.offs[g + 1] - a.offs[g];
        if (rows <= 0) continue;
        a.gid[n] = g;
        a.unit_start[n] = acc;
        acc += ((rows + chunk_rows - 1) / chunk_rows) * units_per_chunk;
        ++n;
    }
    a.unit_start[n] = acc;
    a.n = n;
    a.total_units = acc;
}

__device__ __forceinline__ int find_mx_unit(const MxUnits& a, int unit) {
    int lo = 0, hi = a.n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a.unit_start[mid] <= unit) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// Not volatile: a pure function of its operands, so the compiler may
// interleave independent MMA chains.
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// c += W[rows w0 (g) and w1 (g+8)] . X[row xr]^T over one 32-element k-step,
// given this lane's 16-byte pieces wa (row g), wb (row g+8), xv (token row g).
__device__ __forceinline__ void mma_step(float (&c)[4], const uint4& wa, const uint4& wb,
                                         const uint4& xv) {
    mma_bf16_16816(c, wa.x, wb.x, wa.y, wb.y, xv.x, xv.y);
    mma_bf16_16816(c, wa.z, wb.z, wa.w, wb.w, xv.z, xv.w);
}

// Predicated 16-byte loads (zero when !ok), written as volatile PTX so that
// the compiler keeps them in program order ahead of the MMAs that consume
// them: all loads of an unrolled step are in flight together.
__device__ __forceinline__ uint4 ldg16(const __nv_bfloat16* p, bool ok) {
    uint4 v;
    asm volatile(
        "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %5, 0;\n\t"
        "mov.b32 %0, 0;\n\tmov.b32 %1, 0;\n\tmov.b32 %2, 0;\n\tmov.b32 %3, 0;\n\t"
        "@q ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];\n\t}"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(p), "r"(static_cast<int>(ok)));
    return v;
}

// Same, for weights that are read once: do not allocate them in L1.
__device__ __forceinline__ uint4 ldg16_stream(const __nv_bfloat16* p, bool ok) {
    uint4 v;
    asm volatile(
        "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %5, 0;\n\t"
        "mov.b32 %0, 0;\n\tmov.b32 %1, 0;\n\tmov.b32 %2, 0;\n\tmov.b32 %3, 0;\n\t"
        "@q ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n\t}"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(p), "r"(static_cast<int>(ok)));
    return v;
}

// Element range [k0, k1) of warp w when K is split over the CTA's warps in
// chunks of 32 * UNROLL elements (one unrolled loop iteration each).
__device__ __forceinline__ void k_split(int K, int w, int& k0, int& k1) {
    constexpr int CH = 32 * dec::UNROLL;
    const int nchunks = (K + CH - 1) / CH;
    k0 = ((nchunks * w) / dec::WARPS) * CH;
    k1 = ((nchunks * (w + 1)) / dec::WARPS) * CH;
}

// Sums the WARPS partial fragments of a CTA: every warp writes its NF floats
// per lane, then warp 0 reads all of them back.  Returns true in warp 0.
template <int NF>
__device__ __forceinline__ bool reduce_over_warps(float (&v)[NF], float* red) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int j = 0; j < NF; ++j) red[(warp * NF + j) * 32 + lane] = v[j];
    __syncthreads();
    if (warp == 0) {
#pragma unroll
        for (int j = 0; j < NF; ++j) {
            float acc = 0.f;
#pragma unroll
            for (int w = 0; w < dec::WARPS; ++w) acc += red[(w * NF + j) * 32 + lane];
            v[j] = acc;
        }
    }
    __syncthreads();
    return warp == 0;
}

}  // namespace moe
