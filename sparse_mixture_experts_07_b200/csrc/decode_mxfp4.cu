// Expert FFNs of decode batches (T <= 8) with MXFP4 expert weights.
//
// "Mixture of Experts in Transformers", section "from dense to sparse": at
// small batch the layer's time is the bytes of the active experts' weights
// read from memory, and gpt-oss stores its experts natively in mxfp4, for
// which a dedicated kernel is faster still.  MXFP4 (OCP Microscaling Formats
// v1.0): blocks of 32 consecutive weights along the contraction share one
// E8M0 scale 2^(s-127); each weight is a 4-bit E2M1 code.  A weight costs
// 0.5 + 1/32 bytes instead of bf16's 2.
//
// Storage: q [rows, K/2] bytes, element 2j of a row in the low nibble of byte
// j, element 2j+1 in the high nibble; s [rows, K/32] bytes.
//
// Same structure as the bf16 decode kernels (a CTA per (group, 16 output
// rows), 4 warps splitting the contraction, mma.sync m16n8k16 with weight rows
// as M and the group's <= 8 token rows as N), with three changes:
//   - the products run in f16 x f16 -> f32: an E2M1 pair converts to an f16
//     pair in one instruction (cvt.rn.f16x2.e2m1x2), exactly;
//   - so the activations enter as f16: each row is multiplied by 2^-p first,
//     p = floor(log2 max|row|) - 14, which puts the row's largest magnitude in
//     [2^14, 2^15) (no overflow) and is undone in fp32 in the epilogue;
//   - the contraction is permuted so that the 16 k-values of one MMA come from
//     one block of each weight row: lane (g, q) reads bytes 4q..4q+3 of a
//     block (weights 8q..8q+7), the first two bytes feed one MMA and the last
//     two the next.  The two MMAs of a block accumulate from zero, and the
//     block's scale multiplies the result into the fp32 accumulators (two
//     scales per lane: weight rows g and g+8).
#include "decode_common.cuh"

#include <cuda_fp16.h>

namespace moe {

namespace mx {
constexpr int UNROLL_GU = 8;     // blocks in flight per lane, gate_up (4 weight rows)
constexpr int UNROLL_DN = 16;    // blocks in flight per lane, down (2 weight rows)
constexpr int PREP_THREADS = 256;
}  // namespace mx

struct MxParams {
    const __half* x16;          // [T, H]    x * 2^-xexp[t]
    const int32_t* xexp;        // [T]
    const int32_t* offsets;     // [E+1]
    const int32_t* perm;        // [T*k]
    const float* topk_w;        // [T*k]
    const uint8_t* gu_q;        // [E, 2I, H/2]
    const uint8_t* gu_s;        // [E, 2I, H/32]
    const uint8_t* dn_q;        // [E, H, I/2]
    const uint8_t* dn_s;        // [E, H, I/32]
    __nv_bfloat16* h;           // [T*k, I]  SiLU(gate) * up, sorted slot order
    const __half* h16;          // [T*k, I]  h * 2^-hexp[p]
    const int32_t* hexp;        // [T*k]
    __nv_bfloat16* y_slots;     // [T*k, H]
    int64_t T;
    int H, I, E, k;
    float routed_scale;
};

// rows_to_f16: dst[r] = f16(src[r] * 2^-p_r), p_r = floor(log2 max|src[r]|) - 14
// (0 for an all-zero row), clamped to [-100, 100].  One CTA per row.
__global__ void __launch_bounds__(mx::PREP_THREADS) rows_to_f16_kernel(
    const __nv_bfloat16* __restrict__ src, __half* __restrict__ dst, int32_t* __restrict__ exps,
    int K) {
    __shared__ float wmax[mx::PREP_THREADS / 32];
    const int64_t r = blockIdx.x;
    const __nv_bfloat16* row = src + r * K;
    float m = 0.f;
    for (int i = threadIdx.x; i < K; i += mx::PREP_THREADS)
        m = fmaxf(m, fabsf(__bfloat162float(row[i])));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
    __syncthreads();
    m = 0.f;
#pragma unroll
    for (int w = 0; w < mx::PREP_THREADS / 32; ++w) m = fmaxf(m, wmax[w]);
    // floor(log2 m) from the float's exponent field (m = 0 or subnormal: p = 0)
    const int e = static_cast<int>((__float_as_uint(m) >> 23) & 0xff);
    int p = e == 0 ? 0 : e - 127 - 14;
    p = p < -100 ? -100 : (p > 100 ? 100 : p);
    const float inv = __uint_as_float(static_cast<uint32_t>(127 - p) << 23);   // 2^-p, exact
    for (int i = threadIdx.x; i < K; i += mx::PREP_THREADS)
        dst[r * K + i] = __float2half_rn(__bfloat162float(row[i]) * inv);
    if (threadIdx.x == 0) exps[r] = p;
}

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                              uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1,
                                              const float (&c)[4]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%11,%12,%13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]),
          "f"(c[2]), "f"(c[3]));
}

// The four bytes of w (8 E2M1 codes) as four f16 pairs, low nibble first.
__device__ __forceinline__ void e2m1x8_to_f16(uint32_t w, uint32_t (&h)[4]) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "r"(w));
}

// E8M0 scale code -> float: 2^(s-127); 0 -> 2^-127 (subnormal), 255 -> NaN.
__device__ __forceinline__ float e8m0_to_float(uint32_t s) {
    return s == 0 ? __uint_as_float(0x00400000u)
                  : (s == 255 ? __uint_as_float(0x7fc00000u) : __uint_as_float(s << 23));
}

__device__ __forceinline__ uint32_t ldg_u32(const uint8_t* p, bool ok) {
    uint32_t v;
    asm volatile(
        "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %2, 0;\n\tmov.b32 %0, 0;\n\t"
        "@q ld.global.nc.u32 %0, [%1];\n\t}"
        : "=r"(v)
        : "l"(p), "r"(static_cast<int>(ok)));
    return v;
}

__device__ __forceinline__ uint32_t ldg_u8(const uint8_t* p, bool ok) {
    uint32_t v;
    asm volatile(
        "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %2, 0;\n\tmov.b32 %0, 0;\n\t"
        "@q ld.global.nc.u8 %0, [%1];\n\t}"
        : "=r"(v)
        : "l"(p), "r"(static_cast<int>(ok)));
    return v;
}

__device__ __forceinline__ uint4 ldg_v4(const void* p, bool ok) {
    uint4 v;
    asm volatile(
        "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %5, 0;\n\t"
        "mov.b32 %0, 0;\n\tmov.b32 %1, 0;\n\tmov.b32 %2, 0;\n\tmov.b32 %3, 0;\n\t"
        "@q ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];\n\t}"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(p), "r"(static_cast<int>(ok)));
    return v;
}

// acc += scale(row g) / scale(row g+8) * (W_block . X_block) for one 32-weight
// block: w0 / w1 are this lane's 4 bytes of rows g / g+8, xv its 8 f16 of the
// token row, s0 / s1 the two rows' scale codes.
__device__ __forceinline__ void mx_block(float (&acc)[4], uint32_t w0, uint32_t w1,
                                         const uint4& xv, uint32_t s0, uint32_t s1) {
    uint32_t a[4], b[4];
    e2m1x8_to_f16(w0, a);
    e2m1x8_to_f16(w1, b);
    const float zero[4] = {0.f, 0.f, 0.f, 0.f};
    float d[4];
    mma_f16_16816(d, a[0], b[0], a[1], b[1], xv.x, xv.y, zero);
    mma_f16_16816(d, a[2], b[2], a[3], b[3], xv.z, xv.w, d);
    const float f0 = e8m0_to_float(s0), f1 = e8m0_to_float(s1);
    acc[0] = fmaf(f0, d[0], acc[0]);
    acc[1] = fmaf(f0, d[1], acc[1]);
    acc[2] = fmaf(f1, d[2], acc[2]);
    acc[3] = fmaf(f1, d[3], acc[3]);
}

// Blocks [b0, b1) of warp w when nblk blocks are split over the CTA's warps in
// chunks of `unroll` blocks.
__device__ __forceinline__ void block_split(int nblk, int unroll, int w, int& b0, int& b1) {
    const int nchunks = (nblk + unroll - 1) / unroll;
    b0 = ((nchunks * w) / dec::WARPS) * unroll;
    b1 = ((nchunks * (w + 1)) / dec::WARPS) * unroll;
    if (b1 > nblk) b1 = nblk;
}

__global__ void __launch_bounds__(dec::THREADS, 2) decode_mx_gate_up_kernel(const MxParams p) {
    __shared__ ActiveGroups act;
    __shared__ float red[dec::WARPS * 8 * 32];
    if (threadIdx.x == 0) build_active(act, p.offsets, p.E, 0, p.T, p.I, p.I);
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int nblk = p.H / 32;
    int bs0, bs1;
    block_split(nblk, mx::UNROLL_GU, warp, bs0, bs1);
    const int64_t qrow = p.H / 2, srow = p.H / 32;
    for (int unit = blockIdx.x; unit < act.total_units; unit += gridDim.x) {
        const int ai = find_active(act, unit);
        const int grp = act.gid[ai];
        const int i0 = (unit - act.unit_start[ai]) * 16;
        const int rows = p.offsets[grp + 1] - p.offsets[grp];
        const int64_t row0 = p.offsets[grp];
        const bool tok_ok = g < rows;
        const int64_t tok = tok_ok ? p.perm[row0 + g] / p.k : 0;
        const __half* xrow = p.x16 + tok * p.H;
        const bool r0_ok = i0 + g < p.I, r1_ok = i0 + g + 8 < p.I;
        const int64_t wr = static_cast<int64_t>(grp) * 2 * p.I + i0 + g;   // gate row g
        const uint8_t* qg0 = p.gu_q + wr * qrow + 4 * q;
        const uint8_t* qg1 = qg0 + 8 * qrow;
        const uint8_t* qu0 = qg0 + static_cast<int64_t>(p.I) * qrow;
        const uint8_t* qu1 = qg1 + static_cast<int64_t>(p.I) * qrow;
        const uint8_t* sg0 = p.gu_s + wr * srow;
        const uint8_t* sg1 = sg0 + 8 * srow;
        const uint8_t* su0 = sg0 + static_cast<int64_t>(p.I) * srow;
        const uint8_t* su1 = sg1 + static_cast<int64_t>(p.I) * srow;
        float cg[4] = {0.f, 0.f, 0.f, 0.f}, cu[4] = {0.f, 0.f, 0.f, 0.f};
        for (int b = bs0; b < bs1; b += mx::UNROLL_GU) {
            uint32_t wg0[mx::UNROLL_GU], wg1[mx::UNROLL_GU], wu0[mx::UNROLL_GU], wu1[mx::UNROLL_GU];
            uint32_t tg0[mx::UNROLL_GU], tg1[mx::UNROLL_GU], tu0[mx::UNROLL_GU], tu1[mx::UNROLL_GU];
            uint4 xv[mx::UNROLL_GU];
#pragma unroll
            for (int u = 0; u < mx::UNROLL_GU; ++u) {
                const int blk = b + u;
                const bool in = blk < bs1;
                const int64_t qo = static_cast<int64_t>(blk) * 16;
                wg0[u] = ldg_u32(qg0 + qo, in && r0_ok);
                wg1[u] = ldg_u32(qg1 + qo, in && r1_ok);
                wu0[u] = ldg_u32(qu0 + qo, in && r0_ok);
                wu1[u] = ldg_u32(qu1 + qo, in && r1_ok);
                tg0[u] = ldg_u8(sg0 + blk, in && r0_ok);
                tg1[u] = ldg_u8(sg1 + blk, in && r1_ok);
                tu0[u] = ldg_u8(su0 + blk, in && r0_ok);
                tu1[u] = ldg_u8(su1 + blk, in && r1_ok);
                xv[u] = ldg_v4(xrow + blk * 32 + 8 * q, in && tok_ok);
            }
#pragma unroll
            for (int u = 0; u < mx::UNROLL_GU; ++u) {
                mx_block(cg, wg0[u], wg1[u], xv[u], tg0[u], tg1[u]);
                mx_block(cu, wu0[u], wu1[u], xv[u], tu0[u], tu1[u]);
            }
        }
        float c[8] = {cg[0], cg[1], cg[2], cg[3], cu[0], cu[1], cu[2], cu[3]};
        if (!reduce_over_warps<8>(c, red)) continue;
        // c[0], c[1]: weight row g, tokens 2q, 2q+1; c[2], c[3]: row g+8 (up at +4)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int r = (j < 2) ? g : g + 8;
            const int t = 2 * q + (j & 1);
            if (t < rows && i0 + r < p.I) {
                const int64_t tk = p.perm[row0 + t] / p.k;
                const float up_scale = __uint_as_float(static_cast<uint32_t>(127 + p.xexp[tk]) << 23);
                const float gv = c[j] * up_scale;
                const float h = gv / (1.f + __expf(-gv)) * (c[4 + j] * up_scale);
                p.h[(row0 + t) * p.I + i0 + r] = __float2bfloat16_rn(h);
            }
        }
    }
}

__global__ void __launch_bounds__(dec::THREADS, 2) decode_mx_down_kernel(const MxParams p) {
    __shared__ ActiveGroups act;
    __shared__ float red[dec::WARPS * 4 * 32];
    if (threadIdx.x == 0) build_active(act, p.offsets, p.E, 0, p.T, p.H, p.H);
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int nblk = p.I / 32;
    int bs0, bs1;
    block_split(nblk, mx::UNROLL_DN, warp, bs0, bs1);
    const int64_t qrow = p.I / 2, srow = p.I / 32;
    for (int unit = blockIdx.x; unit < act.total_units; unit += gridDim.x) {
        const int ai = find_active(act, unit);
        const int grp = act.gid[ai];
        const int n0 = (unit - act.unit_start[ai]) * 16;
        const int rows = p.offsets[grp + 1] - p.offsets[grp];
        const int64_t row0 = p.offsets[grp];
        const bool tok_ok = g < rows;
        const __half* hrow = p.h16 + (row0 + (tok_ok ? g : 0)) * p.I;
        const bool r0_ok = n0 + g < p.H, r1_ok = n0 + g + 8 < p.H;
        const int64_t wr = static_cast<int64_t>(grp) * p.H + n0 + g;
        const uint8_t* q0 = p.dn_q + wr * qrow + 4 * q;
        const uint8_t* q1 = q0 + 8 * qrow;
        const uint8_t* s0 = p.dn_s + wr * srow;
        const uint8_t* s1 = s0 + 8 * srow;
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        for (int b = bs0; b < bs1; b += mx::UNROLL_DN) {
            uint32_t w0[mx::UNROLL_DN], w1[mx::UNROLL_DN], t0[mx::UNROLL_DN], t1[mx::UNROLL_DN];
            uint4 hv[mx::UNROLL_DN];
#pragma unroll
            for (int u = 0; u < mx::UNROLL_DN; ++u) {
                const int blk = b + u;
                const bool in = blk < bs1;
                const int64_t qo = static_cast<int64_t>(blk) * 16;
                w0[u] = ldg_u32(q0 + qo, in && r0_ok);
                w1[u] = ldg_u32(q1 + qo, in && r1_ok);
                t0[u] = ldg_u8(s0 + blk, in && r0_ok);
                t1[u] = ldg_u8(s1 + blk, in && r1_ok);
                hv[u] = ldg_v4(hrow + blk * 32 + 8 * q, in && tok_ok);
            }
#pragma unroll
            for (int u = 0; u < mx::UNROLL_DN; ++u) mx_block(c, w0[u], w1[u], hv[u], t0[u], t1[u]);
        }
        if (!reduce_over_warps<4>(c, red)) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int r = (j < 2) ? g : g + 8;
            const int t = 2 * q + (j & 1);
            if (t < rows && n0 + r < p.H) {
                const int64_t orow = row0 + t;
                const float unscale =
                    __uint_as_float(static_cast<uint32_t>(127 + p.hexp[orow]) << 23);
                const float scale = p.routed_scale * p.topk_w[p.perm[orow]] * unscale;
                p.y_slots[orow * p.H + n0 + r] = __float2bfloat16_rn(scale * c[j]);
            }
        }
    }
}

// moe_forward_mxfp4: T <= 8, bf16 activations, routed experts only.
cudaError_t launch_ffn_decode_mxfp4(const moe_shape& s, const void* x, const int32_t* offsets,
                                    const int32_t* perm, const float* topk_w,
                                    const uint8_t* gu_q, const uint8_t* gu_s, const uint8_t* dn_q,
                                    const uint8_t* dn_s, void* h, void* x16, int32_t* xexp,
                                    void* h16, int32_t* hexp, void* y_slots, int num_sms,
                                    cudaStream_t st) {
    if (s.T > dec::MAX_ROWS || s.T < 1 || s.dtype != MOE_BF16 || s.n_shared != 0 ||
        s.H % 32 != 0 || s.I % 32 != 0)
        return cudaErrorInvalidValue;
    MxParams p{};
    p.x16 = static_cast<const __half*>(x16);
    p.xexp = xexp;
    p.offsets = offsets;
    p.perm = perm;
    p.topk_w = topk_w;
    p.gu_q = gu_q;
    p.gu_s = gu_s;
    p.dn_q = dn_q;
    p.dn_s = dn_s;
    p.h = static_cast<__nv_bfloat16*>(h);
    p.h16 = static_cast<const __half*>(h16);
    p.hexp = hexp;
    p.y_slots = static_cast<__nv_bfloat16*>(y_slots);
    p.T = s.T;
    p.H = s.H;
    p.I = s.I;
    p.E = s.E;
    p.k = s.k;
    p.routed_scale = s.routed_scale;
    const int grid = num_sms * 4;
    rows_to_f16_kernel<<<static_cast<unsigned>(s.T), mx::PREP_THREADS, 0, st>>>(
        static_cast<const __nv_bfloat16*>(x), static_cast<__half*>(x16), xexp, s.H);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    decode_mx_gate_up_kernel<<<grid, dec::THREADS, 0, st>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    rows_to_f16_kernel<<<static_cast<unsigned>(s.T * s.k), mx::PREP_THREADS, 0, st>>>(
        static_cast<const __nv_bfloat16*>(h), static_cast<__half*>(h16), hexp, s.I);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    decode_mx_down_kernel<<<grid, dec::THREADS, 0, st>>>(p);
    return cudaGetLastError();
}

}  // namespace moe
