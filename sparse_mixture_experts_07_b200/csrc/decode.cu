// Expert FFNs for decode batches (at most 8 rows per expert group).
//
// "Mixture of Experts in Transformers", section "from dense to sparse": at
// batch size 1 the generation speed is set by the bytes of the active
// parameters read per token (the gpt-oss-20b estimate 800 GB/s / (3.6e9 x 2 B)).
// With a handful of rows per expert the layer is a weight stream: every active
// expert's gate_up and down rows are read exactly once, and the work per byte
// is tiny.  The tile-based grouped GEMM reads its weight panels 128 bytes per
// row per request, which scatters DRAM accesses over hundreds of rows; here
// each warp streams its own rows front to back instead.
//
// Two kernels, each a grid-stride loop of CTAs over work units; the 4 warps of
// a CTA split the unit's contraction and sum their fragments in shared memory:
//   decode_gate_up: unit = (group, 16 output columns); the CTA streams the
//     16 gate rows and the 16 matching up rows of the packed gate_up (P1 §2
//     item 3) and writes h = SiLU(gate x) * (up x) for the group's rows;
//   decode_down: unit = (group, 16 hidden columns); the CTA streams 16 rows
//     of down and writes scale * (down h) into the group's slot rows.
// The products run on mma.sync m16n8k16 (bf16 in, fp32 accumulate): weight
// rows are the 16 M rows, the group's <= 8 token rows are the 8 N columns.
// The contraction order is permuted consistently on both operands so that
// every load is a contiguous 16 bytes: lane (g = lane/4, q = lane%4) loads
// elements [base + 8q, base + 8q + 8) of weight rows g and g+8 and of token
// row g, and feeds elements 0..3 to one MMA and 4..7 to the next.
#include "decode_common.cuh"

namespace moe {

struct DecodeParams {
    const __nv_bfloat16* x;          // [T, H]
    const int32_t* offsets;          // [E+1]
    const int32_t* perm;             // [T*k]
    const float* topk_w;             // [T*k]
    const __nv_bfloat16* gate_up;    // [E, 2I, H]
    const __nv_bfloat16* down;       // [E, H, I]
    const __nv_bfloat16* sh_gate_up; // [S, 2Is, H]
    const __nv_bfloat16* sh_down;    // [S, H, Is]
    __nv_bfloat16* h_routed;         // [T*k, I]
    __nv_bfloat16* h_shared;         // [S*T, Is]
    __nv_bfloat16* y_slots;          // [T*k + S*T, H]
    int64_t T;
    int H, I, E, k, S, Is;
    float routed_scale;
};

// One CTA per work unit (grid-stride); its 4 warps split the contraction.
// Both kernels wait for the previous kernel (pdl_wait) and let the next one
// launch as they drain; decode_down runs as a programmatic dependent.
__global__ void __launch_bounds__(dec::THREADS, 2) decode_gate_up_kernel(const DecodeParams p) {
    __shared__ ActiveGroups act;
    __shared__ float red[dec::WARPS * 8 * 32];
    pdl_wait();
    stage_offsets(act.offs, p.offsets, p.E);
    __syncthreads();
    if (threadIdx.x == 0) build_active(act, p.E, p.S, p.T, p.I, p.Is);
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    int s0, s1;
    k_split(p.H, warp, s0, s1);
    for (int unit = blockIdx.x; unit < act.total_units; unit += gridDim.x) {
        const int ai = find_active(act, unit);
        const int grp = act.gid[ai];
        const bool routed = grp < p.E;
        const int N = routed ? p.I : p.Is;
        const int i0 = (unit - act.unit_start[ai]) * 16;
        const int rows = routed ? act.offs[grp + 1] - act.offs[grp] : static_cast<int>(p.T);
        const int64_t row0 = routed ? act.offs[grp] : static_cast<int64_t>(grp - p.E) * p.T;
        const __nv_bfloat16* W =
            routed ? p.gate_up + static_cast<int64_t>(grp) * 2 * p.I * p.H
                   : p.sh_gate_up + static_cast<int64_t>(grp - p.E) * 2 * p.Is * p.H;
        // this lane's token row (column g of the MMA) and weight rows
        const bool tok_ok = g < rows;
        const int64_t tok = tok_ok ? (routed ? p.perm[row0 + g] / p.k : g) : 0;
        const __nv_bfloat16* xrow = p.x + tok * p.H;
        const bool r0_ok = i0 + g < N, r1_ok = i0 + g + 8 < N;
        const __nv_bfloat16* gate0 = W + static_cast<int64_t>(i0 + g) * p.H;
        const __nv_bfloat16* gate1 = gate0 + static_cast<int64_t>(8) * p.H;
        const __nv_bfloat16* up0 = gate0 + static_cast<int64_t>(N) * p.H;
        const __nv_bfloat16* up1 = gate1 + static_cast<int64_t>(N) * p.H;
        float cg[4] = {0.f, 0.f, 0.f, 0.f}, cu[4] = {0.f, 0.f, 0.f, 0.f};
        for (int k0 = s0; k0 < s1; k0 += 32 * dec::UNROLL) {
            uint4 ga[dec::UNROLL], gb[dec::UNROLL], ua[dec::UNROLL], ub[dec::UNROLL],
                xv[dec::UNROLL];
#pragma unroll
            for (int u = 0; u < dec::UNROLL; ++u) {
                const int col = k0 + u * 32 + 8 * q;
                const bool in = col < p.H;
                ga[u] = ldg16_stream(gate0 + col, in && r0_ok);
                gb[u] = ldg16_stream(gate1 + col, in && r1_ok);
                ua[u] = ldg16_stream(up0 + col, in && r0_ok);
                ub[u] = ldg16_stream(up1 + col, in && r1_ok);
                xv[u] = ldg16(xrow + col, in && tok_ok);
            }
#pragma unroll
            for (int u = 0; u < dec::UNROLL; ++u) {
                mma_step(cg, ga[u], gb[u], xv[u]);
                mma_step(cu, ua[u], ub[u], xv[u]);
            }
        }
        float c[8] = {cg[0], cg[1], cg[2], cg[3], cu[0], cu[1], cu[2], cu[3]};
        if (!reduce_over_warps<8>(c, red)) continue;
        // c[0],c[1]: weight row g, tokens 2q, 2q+1; c[2],c[3]: row g+8 (gate; up at +4)
        __nv_bfloat16* hout = routed ? p.h_routed : p.h_shared;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int r = (j < 2) ? g : g + 8;
            const int t = 2 * q + (j & 1);
            if (t < rows && i0 + r < N) {
                const float gv = c[j];
                const float h = gv / (1.f + __expf(-gv)) * c[4 + j];
                hout[(row0 + t) * N + i0 + r] = __float2bfloat16_rn(h);
            }
        }
    }
    // the next kernel is let in only as this one drains: its CTAs would
    // otherwise sit on the SMs through this kernel's second round of CTAs
    pdl_launch_dependents();
}

// Four CTAs per SM (at most 128 registers): with one token the kernel has
// 2 x H/16 units, which three CTAs per SM would run in two rounds.
__global__ void __launch_bounds__(dec::THREADS, 4) decode_down_kernel(const DecodeParams p) {
    __shared__ ActiveGroups act;
    __shared__ float red[dec::WARPS * 4 * 32];
    pdl_wait();
    stage_offsets(act.offs, p.offsets, p.E);
    __syncthreads();
    if (threadIdx.x == 0) build_active(act, p.E, p.S, p.T, p.H, p.H);
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
    const int64_t routed_rows = p.T * p.k;
    for (int unit = blockIdx.x; unit < act.total_units; unit += gridDim.x) {
        const int ai = find_active(act, unit);
        const int grp = act.gid[ai];
        const bool routed = grp < p.E;
        const int K = routed ? p.I : p.Is;
        int s0, s1;
        k_split(K, warp, s0, s1);
        const int n0 = (unit - act.unit_start[ai]) * 16;
        const int rows = routed ? act.offs[grp + 1] - act.offs[grp] : static_cast<int>(p.T);
        const int64_t row0 = routed ? act.offs[grp] : static_cast<int64_t>(grp - p.E) * p.T;
        const __nv_bfloat16* W = routed ? p.down + static_cast<int64_t>(grp) * p.H * p.I
                                        : p.sh_down + static_cast<int64_t>(grp - p.E) * p.H * p.Is;
        const __nv_bfloat16* hin = routed ? p.h_routed : p.h_shared;
        const bool tok_ok = g < rows;
        const __nv_bfloat16* hrow = hin + (row0 + (tok_ok ? g : 0)) * K;
        const bool r0_ok = n0 + g < p.H, r1_ok = n0 + g + 8 < p.H;
        const __nv_bfloat16* w0 = W + static_cast<int64_t>(n0 + g) * K;
        const __nv_bfloat16* w1 = w0 + static_cast<int64_t>(8) * K;
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        for (int k0 = s0; k0 < s1; k0 += 32 * dec::UNROLL) {
            uint4 wa[dec::UNROLL], wb[dec::UNROLL], hv[dec::UNROLL];
#pragma unroll
            for (int u = 0; u < dec::UNROLL; ++u) {
                const int col = k0 + u * 32 + 8 * q;
                const bool in = col < K;
                wa[u] = ldg16_stream(w0 + col, in && r0_ok);
                wb[u] = ldg16_stream(w1 + col, in && r1_ok);
                hv[u] = ldg16(hrow + col, in && tok_ok);
            }
#pragma unroll
            for (int u = 0; u < dec::UNROLL; ++u) mma_step(c, wa[u], wb[u], hv[u]);
        }
        if (!reduce_over_warps<4>(c, red)) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int r = (j < 2) ? g : g + 8;
            const int t = 2 * q + (j & 1);
            if (t < rows && n0 + r < p.H) {
                int64_t orow;
                float scale = 1.f;
                if (routed) {
                    orow = row0 + t;
                    scale = p.routed_scale * p.topk_w[p.perm[orow]];
                } else {
                    orow = routed_rows + row0 + t;
                }
                p.y_slots[orow * p.H + n0 + r] = __float2bfloat16_rn(scale * c[j]);
            }
        }
    }
    pdl_launch_dependents();   // as in decode_gate_up
}

// Decode path of moe_forward: T <= 8 so every group has at most 8 rows.
cudaError_t launch_ffn_decode(const moe_shape& s, const void* x, const int32_t* offsets,
                              const int32_t* perm, const float* topk_w, const void* gate_up,
                              const void* down, const void* sh_gate_up, const void* sh_down,
                              void* h_routed, void* h_shared, void* y_slots, int num_sms,
                              cudaStream_t st) {
    if (s.T > dec::MAX_ROWS || s.dtype != MOE_BF16) return cudaErrorInvalidValue;
    DecodeParams p{};
    p.x = static_cast<const __nv_bfloat16*>(x);
    p.offsets = offsets;
    p.perm = perm;
    p.topk_w = topk_w;
    p.gate_up = static_cast<const __nv_bfloat16*>(gate_up);
    p.down = static_cast<const __nv_bfloat16*>(down);
    p.sh_gate_up = static_cast<const __nv_bfloat16*>(sh_gate_up);
    p.sh_down = static_cast<const __nv_bfloat16*>(sh_down);
    p.h_routed = static_cast<__nv_bfloat16*>(h_routed);
    p.h_shared = static_cast<__nv_bfloat16*>(h_shared);
    p.y_slots = static_cast<__nv_bfloat16*>(y_slots);
    p.T = s.T;
    p.H = s.H;
    p.I = s.I;
    p.E = s.E;
    p.k = s.k;
    p.S = s.n_shared;
    p.Is = s.n_shared > 0 ? s.I_shared : s.I;
    p.routed_scale = s.routed_scale;
    // 4 CTAs per SM: all resident for decode_down; decode_gate_up (about
    // 216 registers a thread) holds 2 per SM and takes the rest as they finish.
    // decode_gate_up is launched the ordinary way: as a programmatic dependent
    // its CTAs became resident while the router was still running, and its
    // own run at T = 8 (PhiMoE shape) took 15 % longer (measured; cause not
    // identified).  decode_down and the combine follow as dependents.
    const int grid = num_sms * 4;
    decode_gate_up_kernel<<<grid, dec::THREADS, 0, st>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_pdl(decode_down_kernel, dim3(grid), dim3(dec::THREADS), 0, st, p);
}

}  // namespace moe
