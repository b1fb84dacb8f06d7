// Expert FFNs of decode batches (T <= 64) with MXFP4 expert weights.
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
// Work unit: (expert group, chunk of 8*NT of its rows, 16 weight rows), NT = 1
// for batches of up to 8 tokens and 2 above.  The
// MMAs are mma.sync m16n8k16 with weight rows as M and the chunk's token rows
// as NT tiles of N = 8.  Per CTA, a ring of shared-memory stages, each holding
// 512 weights of every row of the unit (gate and up rows for GEMM 1):
//   - warp 0 fills the ring.  Lane 0 issues the code bytes as TMA boxes of 16
//     rows x 128 bytes (128-byte swizzle); all 32 lanes copy the rows' scale
//     bytes with 4-byte cp.async (a scale row is only byte aligned, so each
//     lane copies the five aligned words that cover the stage's 16 scales of
//     a row) and report them on the stage's barrier with
//     cp.async.mbarrier.arrive, so no consumer ever waits on a global load of
//     a scale;
//   - warps 1..4 each take 4 of the stage's 16 blocks.  Per stage a warp first
//     turns the scale bytes of its blocks into floats once (lane r converts
//     row r), then every lane converts its E2M1 codes to f16 pairs
//     (cvt.rn.f16x2.e2m1x2, exact), runs the MMAs in f16 x f16 -> f32 and adds
//     each block's two-MMA partial sum into its accumulators times the
//     block's scale; the warps' partial sums meet in shared memory at the end
//     of the unit.
// Activations enter as f16 rows padded with zeros to a multiple of 512
// columns: each row is multiplied by 2^-p first, p = floor(log2 max|row|) -
// 14, which puts its largest magnitude in [2^14, 2^15); the epilogue undoes
// it in fp32.  The contraction is permuted so that the 16 k-values of one MMA
// come from one block of each weight row: lane (g, q) takes bytes 4q..4q+3 of
// a block (weights 8q..8q+7), the first two bytes feed one MMA and the last
// two the next.  Waits are bounded (MOE_ERR_TIMEOUT).
#include "decode_common.cuh"
#include "gemm_common.cuh"

#include <cuda_fp16.h>

namespace moe {

namespace mx {
constexpr int PREP_THREADS = 256;
constexpr int CONSUMERS = 4;                     // warps 1..CONSUMERS
constexpr int THREADS = 32 * (1 + CONSUMERS);
constexpr int NB = 2;                            // TMA boxes per weight matrix per stage
constexpr int BOX_ROWS = 16;
constexpr int BOX_BYTES = BOX_ROWS * 128;        // 16 rows x 128 bytes (256 codes each)
constexpr int BPS = 8 * NB;                      // 32-weight blocks of a row per stage
constexpr int KSTAGE = BPS * 32;                 // weights of a row per stage
constexpr int BPW = BPS / CONSUMERS;             // blocks per consumer warp per stage
constexpr int SWORDS = 5;                        // scale words copied per row per stage
constexpr int MAX_T = 64;
constexpr int CTA_SMEM = 68 * 1024;              // dynamic shared memory per CTA (3 per SM)
}  // namespace mx

struct MxParams {
    const __half* x16;          // [T, ldx]    x * 2^-xexp[t], zero padded
    const int32_t* xexp;        // [T]
    const int32_t* offsets;     // [E+1]
    const int32_t* perm;        // [T*k]
    const float* topk_w;        // [T*k]
    const uint8_t* gu_s;        // [E, 2I, H/32]
    const uint8_t* dn_s;        // [E, H, I/32]
    __nv_bfloat16* h;           // [T*k, I]  SiLU(gate) * up, sorted slot order
    const __half* h16;          // [T*k, ldh]  h * 2^-hexp[p], zero padded
    const int32_t* hexp;        // [T*k]
    __nv_bfloat16* y_slots;     // [T*k, H]
    int32_t* err_flag;
    int64_t T;
    int H, I, E, k;
    int ldx, ldh;
    float routed_scale;
};

// rows_to_f16: dst[r, 0:K] = f16(src[r] * 2^-p_r), p_r = floor(log2 max|src[r]|)
// - 14 (0 for an all-zero row), clamped to [-100, 100]; dst[r, K:ld] = 0.  One
// CTA per row.
__global__ void __launch_bounds__(mx::PREP_THREADS) rows_to_f16_kernel(
    const __nv_bfloat16* __restrict__ src, __half* __restrict__ dst, int32_t* __restrict__ exps,
    int K, int ld) {
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
    for (int i = threadIdx.x; i < ld; i += mx::PREP_THREADS)
        dst[r * ld + i] = i < K ? __float2half_rn(__bfloat162float(row[i]) * inv)
                                : __float2half_rn(0.f);
    if (threadIdx.x == 0) exps[r] = p;
}

// Not volatile: a pure function of its operands, so the compiler may
// interleave the MMAs of independent blocks.
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                              uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1,
                                              const float (&c)[4]) {
    asm(
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

// 4-byte asynchronous copy global -> shared; src_bytes 0 writes zeros and
// reads nothing.
__device__ __forceinline__ void cp_async4(void* dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}
// Arrive on `bar` once all cp.async of this thread issued so far have landed
// (the arrival is one of the barrier's expected arrivals).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.wait_all;" ::: "memory");
}

__device__ __forceinline__ uint4 ldg_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// d (fresh) = W_block . X_block for one 32-weight block: w0 / w1 are this
// lane's 4 bytes of weight rows g / g+8, xv its 8 f16 of the token row.
__device__ __forceinline__ void mx_block_mma(float (&d)[4], const uint32_t (&a)[4],
                                             const uint32_t (&b)[4], const uint4& xv) {
    const float zero[4] = {0.f, 0.f, 0.f, 0.f};
    mma_f16_16816(d, a[0], b[0], a[1], b[1], xv.x, xv.y, zero);
    mma_f16_16816(d, a[2], b[2], a[3], b[3], xv.z, xv.w, d);
}

// Stage geometry.  KIND 0: gate_up (K = H, output rows I; a stage holds NB
// boxes of the unit's 16 gate rows and NB of the matching 16 up rows).
// KIND 1: down (K = I, output rows H; NB boxes of 16 rows).
template <int KIND, int NT>
struct MxGeo {
    static constexpr int MAT = KIND == 0 ? 2 : 1;                  // weight matrices per stage
    static constexpr int R = 16 * MAT;                             // weight rows per stage
    static constexpr int Q_BYTES = MAT * mx::NB * mx::BOX_BYTES;   // a 1024-byte multiple
    static constexpr int S_BYTES = R * mx::SWORDS * 4;             // scale words per stage
    static constexpr int NF = MAT * NT * 4;                        // accumulators per lane
    static constexpr int CONV_FLOATS = mx::CONSUMERS * R * mx::BPW;
    static constexpr int RED_FLOATS = 2 * mx::CONSUMERS * NF * 32;   // double-buffered
    static constexpr int FIXED = 1024 + 4 * (CONV_FLOATS + RED_FLOATS);
    static constexpr int STAGES_FIT = (mx::CTA_SMEM - FIXED) / (Q_BYTES + S_BYTES + 16);
    static constexpr int STAGES = STAGES_FIT < 3 ? 3 : (STAGES_FIT > 16 ? 16 : STAGES_FIT);
    static constexpr int SMEM_BYTES = FIXED + STAGES * (Q_BYTES + S_BYTES + 16);
};

// CTAs per SM the register budget is sized for: three with one n-tile, two
// with more (their accumulators and prefetched fragments need more than 128
// registers a thread).
template <int NT>
struct MxOccupancy {
    static constexpr int CTAS = NT == 1 ? 3 : 2;
};

template <int KIND, int NT>
__global__ void __launch_bounds__(mx::THREADS, MxOccupancy<NT>::CTAS) decode_mx_kernel(
    const __grid_constant__ CUtensorMap map_q, const MxParams p, uint64_t timeout_ns) {
    using G = MxGeo<KIND, NT>;
    using namespace mx;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ MxUnits act;
    __shared__ int fail_sh;
    uint8_t* q_ring = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* s_ring = q_ring + G::STAGES * G::Q_BYTES;
    uint64_t* full = reinterpret_cast<uint64_t*>(s_ring + G::STAGES * G::S_BYTES);
    uint64_t* empty = full + G::STAGES;
    float* conv = reinterpret_cast<float*>(empty + G::STAGES);   // [CONSUMERS][R][BPW]
    float* red = conv + G::CONV_FLOATS;                          // [2][CONSUMERS][NF][32]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint64_t deadline = global_ns() + timeout_ns;

    const int K = KIND == 0 ? p.H : p.I;                     // contraction
    const int N = KIND == 0 ? p.I : p.H;                     // output rows per expert
    const int64_t wrows = KIND == 0 ? 2 * static_cast<int64_t>(p.I) : p.H;
    const int nblk = K / 32;
    const int nst = (nblk + BPS - 1) / BPS;                  // stages per unit
    const uint8_t* scales = KIND == 0 ? p.gu_s : p.dn_s;
    const int64_t scale_bytes = static_cast<int64_t>(p.E) * wrows * nblk;
    const int units_per_chunk = N / 16;
    constexpr int CHUNK = 8 * NT;

    stage_offsets(act.offs, p.offsets, p.E);
    __syncthreads();
    if (threadIdx.x == 0) {
        build_mx_units(act, p.E, CHUNK, units_per_chunk);
        for (int s = 0; s < G::STAGES; ++s) {
            mbar_init(&full[s], 1 + 32);     // TMA expect_tx + one cp.async arrival per lane
            mbar_init(&empty[s], CONSUMERS);
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

    // expert group, chunk and first weight row of unit u
    auto unit_of = [&](int u, int& grp, int& chunk, int& r0) {
        const int ai = find_mx_unit(act, u);
        grp = act.gid[ai];
        const int local = u - act.unit_start[ai];
        chunk = local / units_per_chunk;
        r0 = (local - chunk * units_per_chunk) * 16;
    };

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        bool ok = true;
        int f = 0;
        for (int ui = 0; ui < my_units && ok; ++ui) {
            const int u = static_cast<int>(blockIdx.x) + ui * static_cast<int>(gridDim.x);
            int grp, chunk, r0;
            unit_of(u, grp, chunk, r0);
            const int64_t wrow0 = static_cast<int64_t>(grp) * wrows + r0;
            for (int st = 0; st < nst; ++st, ++f) {
                const int slot = f % G::STAGES;
                const uint32_t ph = static_cast<uint32_t>(f / G::STAGES) & 1u;
                ok = __all_sync(0xffffffffu, mbar_wait(&empty[slot], ph ^ 1u, deadline));
                if (!ok) break;
                if (lane == 0) {
                    uint8_t* stage = q_ring + slot * G::Q_BYTES;
                    mbar_arrive_expect_tx(&full[slot], G::Q_BYTES);
#pragma unroll
                    for (int m = 0; m < G::MAT; ++m)
#pragma unroll
                        for (int b = 0; b < NB; ++b)
                            tma_load_2d(stage + (m * NB + b) * BOX_BYTES, &map_q, &full[slot],
                                        (st * NB + b) * 128,
                                        static_cast<int32_t>(wrow0 + m * p.I));
                }
                // scale bytes [st*16, st*16 + 16) of every row of the stage: the
                // five aligned words from floor4(row start) + st*16
                uint8_t* sdst = s_ring + slot * G::S_BYTES;
                for (int w = lane; w < G::R * SWORDS; w += 32) {
                    const int rr = w / SWORDS, j = w - rr * SWORDS;
                    const int64_t grow = wrow0 + (rr & 15) + (rr >= 16 ? p.I : 0);
                    const int64_t rowb = grow * nblk;
                    const int64_t a = rowb - (rowb & 3) + st * BPS + 4 * j;
                    // bytes past the end of the scale array are zero-filled, not read
                    const int64_t left = scale_bytes - a;
                    const uint32_t n = left >= 4 ? 4u : (left > 0 ? static_cast<uint32_t>(left) : 0u);
                    cp_async4(sdst + 4 * w, scales + (n ? a : 0), n);
                }
                cp_async_arrive_noinc(&full[slot]);
            }
        }
        cp_async_wait_all();
        if (!ok && lane == 0) raise_error(p.err_flag, MOE_ERR_TIMEOUT);
        return;
    }
    // ---------------------------------------------------------------- consumers
    const int cw = warp - 1, g = lane >> 2, q = lane & 3;
    float* my_conv = conv + cw * G::R * BPW;
    bool ok = true;
    int f = 0;
    for (int ui = 0; ui < my_units; ++ui) {
        const int u = static_cast<int>(blockIdx.x) + ui * static_cast<int>(gridDim.x);
        int grp, chunk, r0;
        unit_of(u, grp, chunk, r0);
        const int rows = act.offs[grp + 1] - act.offs[grp];
        const int64_t row0 = act.offs[grp];
        const int crow0 = chunk * CHUNK;
        // this lane's token row (column g) of each n-tile; rows past the
        // group read row 0 of the activations and are never stored
        const __half* brow[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int t = crow0 + nt * 8 + g;
            if (KIND == 0) {
                const int64_t tok = t < rows ? p.perm[row0 + t] / p.k : 0;
                brow[nt] = p.x16 + tok * p.ldx + 8 * q;
            } else {
                brow[nt] = p.h16 + (t < rows ? row0 + t : 0) * p.ldh + 8 * q;
            }
        }
        // the scale row this lane converts (lane < R) and its byte offset in
        // the copied words
        uint32_t conv_shift = 0;
        if (lane < G::R) {
            const int64_t grow = static_cast<int64_t>(grp) * wrows + r0 + (lane & 15) +
                                 (lane >= 16 ? p.I : 0);
            conv_shift = static_cast<uint32_t>((grow * nblk) & 3) * 8u;
        }
        // epilogue factors of this lane's two token columns (2q, 2q+1) of each
        // n-tile, fetched now so that their latency hides under the stages
        float un[NT][2], wsc[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                un[nt][c] = 1.f;
                wsc[nt][c] = 0.f;
                const int t = crow0 + nt * 8 + 2 * q + c;
                if (cw == 0 && t < rows) {
                    if (KIND == 0) {
                        const int64_t tk = p.perm[row0 + t] / p.k;
                        un[nt][c] = __uint_as_float(static_cast<uint32_t>(127 + p.xexp[tk]) << 23);
                    } else {
                        un[nt][c] =
                            __uint_as_float(static_cast<uint32_t>(127 + p.hexp[row0 + t]) << 23);
                        wsc[nt][c] = p.routed_scale * p.topk_w[p.perm[row0 + t]];
                    }
                }
            }
        float acc[G::NF];
#pragma unroll
        for (int j = 0; j < G::NF; ++j) acc[j] = 0.f;
        // this warp's activation fragments (BPW blocks x NT tiles), loaded one
        // stage ahead of their use
        uint4 bv[BPW][NT];
#pragma unroll
        for (int i = 0; i < BPW; ++i)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) bv[i][nt] = ldg_v4(brow[nt] + (cw * BPW + i) * 32);
        for (int st = 0; st < nst; ++st, ++f) {
            const int slot = f % G::STAGES;
            const uint32_t ph = static_cast<uint32_t>(f / G::STAGES) & 1u;
            uint4 bn[BPW][NT];
            if (st + 1 < nst) {
#pragma unroll
                for (int i = 0; i < BPW; ++i)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        bn[i][nt] = ldg_v4(brow[nt] + ((st + 1) * BPS + cw * BPW + i) * 32);
            }
            if (ok && !mbar_wait(&full[slot], ph, deadline)) ok = false;
            // this warp's blocks' scales as floats, once per stage (lane = row)
            if (lane < G::R) {
                const uint32_t* sw =
                    reinterpret_cast<const uint32_t*>(s_ring + slot * G::S_BYTES) + lane * SWORDS;
                const uint32_t v = __funnelshift_r(sw[cw], sw[cw + 1], conv_shift);
                float4 fs;
                float* fp = reinterpret_cast<float*>(&fs);
#pragma unroll
                for (int i = 0; i < BPW; ++i) {
                    const int blk = st * BPS + cw * BPW + i;
                    fp[i] = blk < nblk ? e8m0_to_float((v >> (8 * i)) & 0xffu) : 0.f;
                }
                *reinterpret_cast<float4*>(my_conv + lane * BPW) = fs;
            }
            __syncwarp();
            const float4 s_g0 = *reinterpret_cast<const float4*>(my_conv + g * BPW);
            const float4 s_g1 = *reinterpret_cast<const float4*>(my_conv + (g + 8) * BPW);
            float4 s_u0 = s_g0, s_u1 = s_g1;
            if (KIND == 0) {
                s_u0 = *reinterpret_cast<const float4*>(my_conv + (16 + g) * BPW);
                s_u1 = *reinterpret_cast<const float4*>(my_conv + (24 + g) * BPW);
            }
            const uint8_t* stage = q_ring + slot * G::Q_BYTES;
#pragma unroll
            for (int i = 0; i < BPW; ++i) {
                const int jj = cw * BPW + i;                  // block within the stage
                const uint8_t* bx = stage + (jj >> 3) * BOX_BYTES;
                const uint32_t swz = static_cast<uint32_t>(((jj & 7) ^ g) << 4) + 4 * q;
                const float f0 = reinterpret_cast<const float*>(&s_g0)[i];
                const float f1 = reinterpret_cast<const float*>(&s_g1)[i];
                uint32_t a[4], b[4];
                e2m1x8_to_f16(*reinterpret_cast<const uint32_t*>(bx + g * 128 + swz), a);
                e2m1x8_to_f16(*reinterpret_cast<const uint32_t*>(bx + (g + 8) * 128 + swz), b);
                uint32_t ua[4], ub[4];
                float f2 = 0.f, f3 = 0.f;
                if (KIND == 0) {
                    const uint8_t* ux = bx + NB * BOX_BYTES;
                    e2m1x8_to_f16(*reinterpret_cast<const uint32_t*>(ux + g * 128 + swz), ua);
                    e2m1x8_to_f16(*reinterpret_cast<const uint32_t*>(ux + (g + 8) * 128 + swz),
                                  ub);
                    f2 = reinterpret_cast<const float*>(&s_u0)[i];
                    f3 = reinterpret_cast<const float*>(&s_u1)[i];
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const uint4 xv = bv[i][nt];
                    float d[4];
                    mx_block_mma(d, a, b, xv);
                    float* ag = acc + nt * 4;
                    ag[0] = fmaf(f0, d[0], ag[0]);
                    ag[1] = fmaf(f0, d[1], ag[1]);
                    ag[2] = fmaf(f1, d[2], ag[2]);
                    ag[3] = fmaf(f1, d[3], ag[3]);
                    if (KIND == 0) {
                        float e[4];
                        mx_block_mma(e, ua, ub, xv);
                        float* au = acc + (NT + nt) * 4;
                        au[0] = fmaf(f2, e[0], au[0]);
                        au[1] = fmaf(f2, e[1], au[1]);
                        au[2] = fmaf(f3, e[2], au[2]);
                        au[3] = fmaf(f3, e[3], au[3]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);
            if (st + 1 < nst) {
#pragma unroll
                for (int i = 0; i < BPW; ++i)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) bv[i][nt] = bn[i][nt];
            }
        }
        // partial sums of the consumer warps meet in shared memory, in one of
        // two buffers by unit parity: warp 1 reduces unit ui's buffer after the
        // barrier while the other warps go on to unit ui + 1, whose barrier they
        // cannot pass before warp 1 has finished with this buffer
        float* rb = red + (ui & 1) * (CONSUMERS * G::NF * 32);
#pragma unroll
        for (int j = 0; j < G::NF; ++j) rb[(cw * G::NF + j) * 32 + lane] = acc[j];
        if (!ok) fail_sh = 1;
        asm volatile("bar.sync 1, %0;" ::"r"(32 * CONSUMERS) : "memory");
        const bool failed = fail_sh != 0;
        if (cw == 0) {
#pragma unroll
            for (int j = 0; j < G::NF; ++j) {
                float v = 0.f;
#pragma unroll
                for (int w = 0; w < CONSUMERS; ++w) v += rb[(w * G::NF + j) * 32 + lane];
                acc[j] = v;
            }
            // acc[nt*4 + 0..1]: weight row g, tokens 2q, 2q+1 of n-tile nt;
            // acc[nt*4 + 2..3]: row g+8 (KIND 0: up at + NT*4)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int r = (j < 2) ? g : g + 8;
                    const int t = crow0 + nt * 8 + 2 * q + (j & 1);
                    if (t < rows && ok) {
                        const float s = un[nt][j & 1];
                        if (KIND == 0) {
                            const float gv = acc[nt * 4 + j] * s;
                            const float h = gv / (1.f + __expf(-gv)) * (acc[(NT + nt) * 4 + j] * s);
                            p.h[(row0 + t) * p.I + r0 + r] = __float2bfloat16_rn(h);
                        } else {
                            p.y_slots[(row0 + t) * p.H + r0 + r] =
                                __float2bfloat16_rn(wsc[nt][j & 1] * s * acc[nt * 4 + j]);
                        }
                    }
                }
        }
        if (failed) break;
    }
    if (cw == 0 && lane == 0 && !ok) raise_error(p.err_flag, MOE_ERR_TIMEOUT);
}

// uint8 2D [rows, cols] map, box 128 columns x 16 rows, 128-byte swizzle.
static bool make_map_u8(CUtensorMap* map, const void* base, int64_t rows, int64_t cols) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc || rows <= 0 || cols <= 0) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols)};
    cuuint32_t box[2] = {128u, static_cast<cuuint32_t>(mx::BOX_ROWS)};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Row stride (elements) of the f16 activation copies: K rounded up to a whole
// number of stages, so that every stage's loads stay inside the row.
int mx_padded_cols(int K) { return (K + mx::KSTAGE - 1) / mx::KSTAGE * mx::KSTAGE; }

template <int KIND, int NT>
static cudaError_t launch_mx(const CUtensorMap& map, const MxParams& p, int num_sms,
                             cudaStream_t st) {
    using G = MxGeo<KIND, NT>;
    cudaError_t e = cudaFuncSetAttribute(decode_mx_kernel<KIND, NT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         G::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    // as many CTAs as fit next to each other on an SM (registers, shared memory)
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_mx_kernel<KIND, NT>,
                                                      mx::THREADS, G::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    per_sm = per_sm < 1 ? 1 : (per_sm > MxOccupancy<NT>::CTAS ? MxOccupancy<NT>::CTAS : per_sm);
    decode_mx_kernel<KIND, NT><<<num_sms * per_sm, mx::THREADS, G::SMEM_BYTES, st>>>(
        map, p, 4000000000ull);
    return cudaGetLastError();
}

// moe_forward_mxfp4: 1 <= T <= 64, bf16 activations, routed experts only.
cudaError_t launch_ffn_decode_mxfp4(const moe_shape& s, const void* x, const int32_t* offsets,
                                    const int32_t* perm, const float* topk_w,
                                    const uint8_t* gu_q, const uint8_t* gu_s, const uint8_t* dn_q,
                                    const uint8_t* dn_s, void* h, void* x16, int32_t* xexp,
                                    void* h16, int32_t* hexp, void* y_slots, int32_t* err_flag,
                                    int num_sms, cudaStream_t st) {
    if (s.T > mx::MAX_T || s.T < 1 || s.dtype != MOE_BF16 || s.n_shared != 0 ||
        s.H % 32 != 0 || s.I % 32 != 0)
        return cudaErrorInvalidValue;
    MxParams p{};
    p.x16 = static_cast<const __half*>(x16);
    p.xexp = xexp;
    p.offsets = offsets;
    p.perm = perm;
    p.topk_w = topk_w;
    p.gu_s = gu_s;
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
    p.ldx = mx_padded_cols(s.H);
    p.ldh = mx_padded_cols(s.I);
    p.routed_scale = s.routed_scale;
    CUtensorMap map_gu, map_dn;
    if (!make_map_u8(&map_gu, gu_q, static_cast<int64_t>(s.E) * 2 * s.I, s.H / 2) ||
        !make_map_u8(&map_dn, dn_q, static_cast<int64_t>(s.E) * s.H, s.I / 2))
        return cudaErrorInvalidValue;
    rows_to_f16_kernel<<<static_cast<unsigned>(s.T), mx::PREP_THREADS, 0, st>>>(
        static_cast<const __nv_bfloat16*>(x), static_cast<__half*>(x16), xexp, s.H, p.ldx);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // one n-tile of 8 token rows covers every group of a batch of <= 8 tokens;
    // above, chunks of 16 rows (two tiles): a group of more rows streams its
    // weights once per chunk, which at T <= 64 is rare (2 T / E rows on average)
    const bool small = s.T <= 8;
    e = small ? launch_mx<0, 1>(map_gu, p, num_sms, st) : launch_mx<0, 2>(map_gu, p, num_sms, st);
    if (e != cudaSuccess) return e;
    rows_to_f16_kernel<<<static_cast<unsigned>(s.T * s.k), mx::PREP_THREADS, 0, st>>>(
        static_cast<const __nv_bfloat16*>(h), static_cast<__half*>(h16), hexp, s.I, p.ldh);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return small ? launch_mx<1, 1>(map_dn, p, num_sms, st) : launch_mx<1, 2>(map_dn, p, num_sms, st);
}

}  // namespace moe
