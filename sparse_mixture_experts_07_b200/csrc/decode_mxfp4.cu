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
// Work unit: (expert group, 16 output rows), as in the bf16 decode kernels;
// the MMAs are mma.sync m16n8k16 with weight rows as M and the group's <= 8
// token rows as N.  Per CTA:
//   - warp 0 streams the unit's weight bytes through a ring of shared-memory
//     stages: lane 0 issues, per weight matrix, MOE_MX_BOXES adjacent 16-row x
//     128-byte TMA boxes (128-byte swizzle), so each row is read in runs of
//     128 * MOE_MX_BOXES bytes;
//   - warps 1..MOE_MX_CONSUMERS split each stage's blocks; each lane loads the
//     block scales of its weight rows and its activation fragments one stage
//     ahead (scale rows are not 16-byte aligned, so they cannot use TMA),
//     converts E2M1 pairs to f16 pairs (cvt.rn.f16x2.e2m1x2, exact) and runs
//     the MMAs in f16 x f16 -> f32; the warps' partial sums meet in shared
//     memory at the end of the unit.
// Activations enter as f16: each row is multiplied by 2^-p first, p =
// floor(log2 max|row|) - 14, which puts its largest magnitude in [2^14, 2^15);
// the epilogue undoes it in fp32.  The contraction is permuted so that the 16
// k-values of one MMA come from one block of each weight row: lane (g, q)
// takes bytes 4q..4q+3 of a block (weights 8q..8q+7), the first two bytes
// feed one MMA and the last two the next.  The two MMAs of a block start
// from zero and the block's scale multiplies their sum into the fp32
// accumulators.  Waits are bounded (MOE_ERR_TIMEOUT).
#include "decode_common.cuh"
#include "gemm_common.cuh"

#include <cuda_fp16.h>

namespace moe {

namespace mx {
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
    int32_t* err_flag;
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
// token row, f0 / f1 the two rows' block scales.
__device__ __forceinline__ void mx_block(float (&acc)[4], uint32_t w0, uint32_t w1,
                                         const uint4& xv, float f0, float f1) {
    uint32_t a[4], b[4];
    e2m1x8_to_f16(w0, a);
    e2m1x8_to_f16(w1, b);
    const float zero[4] = {0.f, 0.f, 0.f, 0.f};
    float d[4];
    mma_f16_16816(d, a[0], b[0], a[1], b[1], xv.x, xv.y, zero);
    mma_f16_16816(d, a[2], b[2], a[3], b[3], xv.z, xv.w, d);
    acc[0] = fmaf(f0, d[0], acc[0]);
    acc[1] = fmaf(f0, d[1], acc[1]);
    acc[2] = fmaf(f1, d[2], acc[2]);
    acc[3] = fmaf(f1, d[3], acc[3]);
}

#ifndef MOE_MX_CONSUMERS
#define MOE_MX_CONSUMERS 4
#endif
namespace mxt {
constexpr int CONSUMERS = MOE_MX_CONSUMERS;     // warps 1..CONSUMERS
constexpr int THREADS = 32 * (1 + CONSUMERS);
constexpr int BOX_ROWS = 16;
constexpr int BOX_BYTES = BOX_ROWS * 128;       // 16 rows x 8 blocks of 16 bytes
#ifndef MOE_MX_RING_KB
#define MOE_MX_RING_KB 64
#endif
constexpr int SMEM_BUDGET = MOE_MX_RING_KB * 1024;   // ring bytes per CTA
}  // namespace mxt

#ifndef MOE_MX_BOXES
#define MOE_MX_BOXES 2
#endif
#ifndef MOE_MX_MIN_BLOCKS
#define MOE_MX_MIN_BLOCKS 3
#endif

// Stage geometry.  KIND 0: gate_up (K = H, output rows I; a stage holds NB
// adjacent boxes of the 16 gate rows and NB of the matching 16 up rows).
// KIND 1: down (K = I, output rows H; NB adjacent boxes of 16 rows).  A stage
// covers BPS = 8 NB blocks of each weight row, so every row is read in runs of
// 128 NB contiguous bytes.  Scale bytes of a stage: [R rows][BPS blocks].
template <int KIND, int NB>
struct MxGeo {
    static constexpr int MAT = KIND == 0 ? 2 : 1;                // weight matrices per stage
    static constexpr int BPS = 8 * NB;                           // blocks per stage
    static constexpr int BPW = BPS / mxt::CONSUMERS;             // blocks per consumer warp
    static constexpr int R = 16 * MAT;                           // weight rows per stage
    static constexpr int Q_BYTES = MAT * NB * mxt::BOX_BYTES;    // a 1024-byte multiple
    static constexpr int SR = 2 * MAT;                           // scale rows per lane
    static constexpr int STAGES_FIT = mxt::SMEM_BUDGET / Q_BYTES;
    static constexpr int STAGES = STAGES_FIT < 4 ? 4 : (STAGES_FIT > 24 ? 24 : STAGES_FIT);
    static constexpr int NF = KIND == 0 ? 8 : 4;                 // accumulators per lane
    static constexpr int SMEM_BYTES = STAGES * Q_BYTES + 1024 + 2 * STAGES * 8 + 64;
};

template <int KIND, int NB>
__global__ void __launch_bounds__(mxt::THREADS, MOE_MX_MIN_BLOCKS) decode_mx_kernel(
    const __grid_constant__ CUtensorMap map_q, const MxParams p, uint64_t timeout_ns) {
    using G = MxGeo<KIND, NB>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ ActiveGroups act;
    __shared__ float red[mxt::CONSUMERS * G::NF * 32];
    __shared__ int fail_sh;
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + G::STAGES * G::Q_BYTES);
    uint64_t* empty = full + G::STAGES;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint64_t deadline = global_ns() + timeout_ns;

    const int K = KIND == 0 ? p.H : p.I;                     // contraction
    const int N = KIND == 0 ? p.I : p.H;                     // output rows per expert
    const int64_t wrows = KIND == 0 ? 2 * static_cast<int64_t>(p.I) : p.H;   // weight rows per expert
    const int nblk = K / 32;
    const int nst = (nblk + G::BPS - 1) / G::BPS;            // stages per unit
    const uint8_t* scales = KIND == 0 ? p.gu_s : p.dn_s;
    const int64_t total_rows = static_cast<int64_t>(p.E) * wrows;

    stage_offsets(act.offs, p.offsets, p.E);
    __syncthreads();
    if (threadIdx.x == 0) {
        build_active(act, p.E, 0, p.T, N, N);
        for (int s = 0; s < G::STAGES; ++s) {
            mbar_init(&full[s], 1);                // one arrive.expect_tx per stage
            mbar_init(&empty[s], mxt::CONSUMERS);
        }
        fail_sh = 0;
        fence_barrier_init();
        tma_prefetch_desc(&map_q);
    }
    __syncthreads();
    const int n_units = act.total_units;
    const int my_units = n_units > static_cast<int>(blockIdx.x)
                             ? (n_units - 1 - static_cast<int>(blockIdx.x)) / gridDim.x + 1
                             : 0;

    // expert group and first output row of unit u
    auto unit_row0 = [&](int u, int& grp, int& r0) {
        const int ai = find_active(act, u);
        grp = act.gid[ai];
        r0 = (u - act.unit_start[ai]) * 16;
    };

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        // lane 0 alone: the weight boxes of every stage, the unit looked up once
        if (lane != 0) return;
        bool ok = true;
        int f = 0;
        for (int ui = 0; ui < my_units && ok; ++ui) {
            const int u = static_cast<int>(blockIdx.x) + ui * static_cast<int>(gridDim.x);
            int grp, r0;
            unit_row0(u, grp, r0);
            const int row = static_cast<int>(static_cast<int64_t>(grp) * wrows + r0);
            for (int st = 0; st < nst; ++st, ++f) {
                const int slot = f % G::STAGES;
                const uint32_t ph = static_cast<uint32_t>(f / G::STAGES) & 1u;
                if (!mbar_wait(&empty[slot], ph ^ 1u, deadline)) { ok = false; break; }
                uint8_t* stage = smem + slot * G::Q_BYTES;
                mbar_arrive_expect_tx(&full[slot], G::Q_BYTES);
#pragma unroll
                for (int m = 0; m < G::MAT; ++m)
#pragma unroll
                    for (int b = 0; b < NB; ++b)
                        tma_load_2d(stage + (m * NB + b) * mxt::BOX_BYTES, &map_q, &full[slot],
                                    (st * NB + b) * 128, row + m * p.I);
            }
        }
        if (!ok) raise_error(p.err_flag, MOE_ERR_TIMEOUT);
        return;
    }
    // ---------------------------------------------------------------- consumers
    const int cw = warp - 1, g = lane >> 2, q = lane & 3;
    bool ok = true;
    int f = 0;
    for (int ui = 0; ui < my_units; ++ui) {
        const int u = static_cast<int>(blockIdx.x) + ui * static_cast<int>(gridDim.x);
        int grp, r0;
        unit_row0(u, grp, r0);
        const int rows = act.offs[grp + 1] - act.offs[grp];
        const int64_t row0 = act.offs[grp];
        const bool tok_ok = g < rows;
        const __half* brow;                       // this lane's token row (column g)
        if (KIND == 0) {
            const int64_t tok = tok_ok ? p.perm[row0 + g] / p.k : 0;
            brow = p.x16 + tok * p.H;
        } else {
            brow = p.h16 + (row0 + (tok_ok ? g : 0)) * p.I;
        }
        // epilogue factors of this lane's two token columns (2q, 2q+1), fetched
        // now so that their latency hides under the unit's stages
        float un[2] = {1.f, 1.f}, wsc[2] = {0.f, 0.f};
        if (cw == 0) {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const int t = 2 * q + c;
                if (t < rows) {
                    if (KIND == 0) {
                        const int64_t tk = p.perm[row0 + t] / p.k;
                        un[c] = __uint_as_float(static_cast<uint32_t>(127 + p.xexp[tk]) << 23);
                    } else {
                        un[c] = __uint_as_float(static_cast<uint32_t>(127 + p.hexp[row0 + t]) << 23);
                        wsc[c] = p.routed_scale * p.topk_w[p.perm[row0 + t]];
                    }
                }
            }
        }
        float acc[G::NF];
#pragma unroll
        for (int j = 0; j < G::NF; ++j) acc[j] = 0.f;
        // this warp's activation fragments, loaded one stage ahead of their use
        auto load_b = [&](int st, uint4 (&v)[G::BPW]) {
#pragma unroll
            for (int i = 0; i < G::BPW; ++i) {
                const int blk = st * G::BPS + cw * G::BPW + i;
                v[i] = ldg_v4(brow + blk * 32 + 8 * q, tok_ok && st < nst && blk < nblk);
            }
        };
        uint4 bv[G::BPW], bn[G::BPW];
        load_b(0, bv);
        // block scales of this lane's weight rows (g, g+8; KIND 0 also the up
        // rows), loaded one stage ahead like the activation fragments
        constexpr int SR = G::SR;
        const uint8_t* srow[SR];
        bool sok[SR];
        {
            const int64_t wr0 = static_cast<int64_t>(grp) * wrows + r0 + g;
#pragma unroll
            for (int r = 0; r < SR; ++r) {
                const int64_t row = wr0 + (r & 1) * 8 + (r >= 2 ? p.I : 0);
                sok[r] = row < total_rows;
                srow[r] = scales + (sok[r] ? row : 0) * nblk;
            }
        }
        auto load_s = [&](int st, uint32_t (&v)[G::BPW][SR]) {
#pragma unroll
            for (int i = 0; i < G::BPW; ++i) {
                const int blk = st * G::BPS + cw * G::BPW + i;
#pragma unroll
                for (int r = 0; r < SR; ++r)
                    v[i][r] = ldg_u8(srow[r] + blk, sok[r] && st < nst && blk < nblk);
            }
        };
        uint32_t sv[G::BPW][SR], sn[G::BPW][SR];
        load_s(0, sv);
        for (int st = 0; st < nst; ++st, ++f) {
            const int slot = f % G::STAGES;
            const uint32_t ph = static_cast<uint32_t>(f / G::STAGES) & 1u;
            load_b(st + 1, bn);
            load_s(st + 1, sn);
            if (ok && !mbar_wait(&full[slot], ph, deadline)) ok = false;
            const uint8_t* stage = smem + slot * G::Q_BYTES;
#pragma unroll
            for (int i = 0; i < G::BPW; ++i) {
                const int jj = cw * G::BPW + i;                  // block within the stage
                const uint8_t* bx = stage + (jj >> 3) * mxt::BOX_BYTES;
                const uint32_t swz = static_cast<uint32_t>(((jj & 7) ^ g) << 4) + 4 * q;
                const uint32_t w0 = *reinterpret_cast<const uint32_t*>(bx + g * 128 + swz);
                const uint32_t w1 = *reinterpret_cast<const uint32_t*>(bx + (g + 8) * 128 + swz);
                if (KIND == 0) {
                    const uint8_t* ux = bx + NB * mxt::BOX_BYTES;
                    const uint32_t v0 = *reinterpret_cast<const uint32_t*>(ux + g * 128 + swz);
                    const uint32_t v1 = *reinterpret_cast<const uint32_t*>(ux + (g + 8) * 128 + swz);
                    float tg[4] = {acc[0], acc[1], acc[2], acc[3]};
                    float tu[4] = {acc[4], acc[5], acc[6], acc[7]};
                    mx_block(tg, w0, w1, bv[i], e8m0_to_float(sv[i][0]), e8m0_to_float(sv[i][1]));
                    mx_block(tu, v0, v1, bv[i], e8m0_to_float(sv[i][2]), e8m0_to_float(sv[i][3]));
#pragma unroll
                    for (int j = 0; j < 4; ++j) { acc[j] = tg[j]; acc[4 + j] = tu[j]; }
                } else {
                    float t4[4] = {acc[0], acc[1], acc[2], acc[3]};
                    mx_block(t4, w0, w1, bv[i], e8m0_to_float(sv[i][0]), e8m0_to_float(sv[i][1]));
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[j] = t4[j];
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);
#pragma unroll
            for (int i = 0; i < G::BPW; ++i) {
                bv[i] = bn[i];
#pragma unroll
                for (int r = 0; r < SR; ++r) sv[i][r] = sn[i][r];
            }
        }
        // partial sums of the four consumer warps meet in shared memory
#pragma unroll
        for (int j = 0; j < G::NF; ++j) red[(cw * G::NF + j) * 32 + lane] = acc[j];
        if (!ok) fail_sh = 1;
        asm volatile("bar.sync 1, %0;" ::"r"(32 * mxt::CONSUMERS) : "memory");
        if (cw == 0) {
#pragma unroll
            for (int j = 0; j < G::NF; ++j) {
                float v = 0.f;
#pragma unroll
                for (int w = 0; w < mxt::CONSUMERS; ++w) v += red[(w * G::NF + j) * 32 + lane];
                acc[j] = v;
            }
            // acc[0], acc[1]: weight row g, tokens 2q, 2q+1; acc[2], acc[3]: row g+8
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int r = (j < 2) ? g : g + 8;
                const int t = 2 * q + (j & 1);
                if (t < rows && r0 + r < N && ok) {
                    if (KIND == 0) {
                        const float gv = acc[j] * un[j & 1];
                        const float h = gv / (1.f + __expf(-gv)) * (acc[4 + j] * un[j & 1]);
                        p.h[(row0 + t) * p.I + r0 + r] = __float2bfloat16_rn(h);
                    } else {
                        p.y_slots[(row0 + t) * p.H + r0 + r] =
                            __float2bfloat16_rn(wsc[j & 1] * un[j & 1] * acc[j]);
                    }
                }
            }
        }
        asm volatile("bar.sync 1, %0;" ::"r"(32 * mxt::CONSUMERS) : "memory");
        if (fail_sh) break;
    }
    if (cw == 0 && lane == 0 && !ok) raise_error(p.err_flag, MOE_ERR_TIMEOUT);
}

// uint8 2D [rows, cols] map, box 128 columns x 16 rows, 128-byte swizzle.
static bool make_map_u8(CUtensorMap* map, const void* base, int64_t rows, int64_t cols) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc || rows <= 0 || cols <= 0) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols)};
    cuuint32_t box[2] = {128u, static_cast<cuuint32_t>(mxt::BOX_ROWS)};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// moe_forward_mxfp4: T <= 8, bf16 activations, routed experts only.
cudaError_t launch_ffn_decode_mxfp4(const moe_shape& s, const void* x, const int32_t* offsets,
                                    const int32_t* perm, const float* topk_w,
                                    const uint8_t* gu_q, const uint8_t* gu_s, const uint8_t* dn_q,
                                    const uint8_t* dn_s, void* h, void* x16, int32_t* xexp,
                                    void* h16, int32_t* hexp, void* y_slots, int32_t* err_flag,
                                    int num_sms, cudaStream_t st) {
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
    p.err_flag = err_flag;
    p.T = s.T;
    p.H = s.H;
    p.I = s.I;
    p.E = s.E;
    p.k = s.k;
    p.routed_scale = s.routed_scale;
    CUtensorMap map_gu, map_dn;
    if (!make_map_u8(&map_gu, gu_q, static_cast<int64_t>(s.E) * 2 * s.I, s.H / 2) ||
        !make_map_u8(&map_dn, dn_q, static_cast<int64_t>(s.E) * s.H, s.I / 2))
        return cudaErrorInvalidValue;
    using G0 = MxGeo<0, MOE_MX_BOXES>;
    using G1 = MxGeo<1, MOE_MX_BOXES>;
    cudaError_t e = cudaFuncSetAttribute(decode_mx_kernel<0, MOE_MX_BOXES>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         G0::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(decode_mx_kernel<1, MOE_MX_BOXES>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, G1::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    // as many CTAs as fit next to each other (shared memory), on every SM
    const int per_sm0 = (200 * 1024) / G0::SMEM_BYTES, per_sm1 = (200 * 1024) / G1::SMEM_BYTES;
    const int grid0 = num_sms * (per_sm0 > 0 ? per_sm0 : 1);
    const int grid1 = num_sms * (per_sm1 > 0 ? per_sm1 : 1);
    const uint64_t timeout = 4000000000ull;
    rows_to_f16_kernel<<<static_cast<unsigned>(s.T), mx::PREP_THREADS, 0, st>>>(
        static_cast<const __nv_bfloat16*>(x), static_cast<__half*>(x16), xexp, s.H);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    decode_mx_kernel<0, MOE_MX_BOXES><<<grid0, mxt::THREADS, G0::SMEM_BYTES, st>>>(map_gu, p,
                                                                                   timeout);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    rows_to_f16_kernel<<<static_cast<unsigned>(s.T * s.k), mx::PREP_THREADS, 0, st>>>(
        static_cast<const __nv_bfloat16*>(h), static_cast<__half*>(h16), hexp, s.I);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    decode_mx_kernel<1, MOE_MX_BOXES><<<grid1, mxt::THREADS, G1::SMEM_BYTES, st>>>(map_dn, p,
                                                                                   timeout);
    return cudaGetLastError();
}

}  // namespace moe
