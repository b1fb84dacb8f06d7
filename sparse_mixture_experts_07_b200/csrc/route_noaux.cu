// DeepSeek-V3 routing ("noaux_tc", named by the Instella-MoE walk-through,
// "config at a glance"; defined by the DeepSeek-V3 technical report, section
// 2.1) on the router's bias-free float32 logits, one warp per token:
//   s_e = sigmoid(l_e); c_e = s_e + b_e (the bias enters the selection only);
//   the E experts form n_group contiguous groups, a group scores the float32
//   sum of its two largest c_e, the topk_group best groups are kept (ties to
//   the lower group); the k largest c_e of the kept groups are selected in
//   descending order (ties to the lower expert); w_j = s_j / sum_i s_i.
// Lane l holds experts l, l + 32, ...; the group scores are formed by lane g
// for group g from the warp's copy of c in shared memory, and every arg-max is
// a warp shuffle reduction on (value, index).
#include "common.cuh"

namespace moe {

constexpr int kNxWarps = 8;

__device__ __forceinline__ void warp_argmax(float& v, int& i) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, v, off);
        const int oi = __shfl_xor_sync(0xffffffffu, i, off);
        if (ov > v || (ov == v && oi < i)) {
            v = ov;
            i = oi;
        }
    }
}

template <int EPL>   // experts per lane: ceil(E / 32)
__global__ void __launch_bounds__(kNxWarps * 32) route_noaux_kernel(
    const float* __restrict__ logits, const float* __restrict__ bias, int32_t* __restrict__ idx,
    float* __restrict__ w, int64_t T, int E, int k, int n_group, int topk_group) {
    __shared__ float c_sh[kNxWarps][EPL * 32];
    __shared__ float s_sh[kNxWarps][EPL * 32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * kNxWarps + warp;
    if (t >= T) return;
    const int gsize = E / n_group;
    const float ninf = -__int_as_float(0x7f800000);
    float c[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        c[i] = ninf;
        if (e < E) {
            const float s = 1.f / (1.f + expf(-logits[t * E + e]));
            c[i] = s + (bias ? bias[e] : 0.f);
            c_sh[warp][e] = c[i];
            s_sh[warp][e] = s;
        }
    }
    __syncwarp();
    // group g's score: the sum of its two largest c (lane g)
    float gs = ninf;
    if (lane < n_group) {
        float b1 = ninf, b2 = ninf;
        for (int e = lane * gsize; e < (lane + 1) * gsize; ++e) {
            const float v = c_sh[warp][e];
            if (v > b1) {
                b2 = b1;
                b1 = v;
            } else if (v > b2) {
                b2 = v;
            }
        }
        gs = gsize >= 2 ? b1 + b2 : b1;
    }
    // keep the topk_group best groups
    bool keep = false;
    for (int r = 0; r < topk_group; ++r) {
        float v = (lane < n_group && !keep) ? gs : ninf;
        int g = lane < n_group ? lane : 1 << 30;
        warp_argmax(v, g);
        if (lane == g) keep = true;
    }
    const uint32_t kept = __ballot_sync(0xffffffffu, keep);
    // the k best experts of the kept groups
    uint32_t taken = 0;
    float den = 0.f;
    int sel_j = 0;
    for (int j = 0; j < k; ++j) {
        float v = ninf;
        int bi = 1 << 30;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            const int e = lane + 32 * i;
            if (e < E && !((taken >> i) & 1u) && ((kept >> (e / gsize)) & 1u) && c[i] > v) {
                v = c[i];
                bi = e;
            }
        }
        warp_argmax(v, bi);
        if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
        den += s_sh[warp][bi];
        if (lane == j) sel_j = bi;
    }
    if (lane < k) {
        idx[t * k + lane] = sel_j;
        w[t * k + lane] = s_sh[warp][sel_j] / den;
    }
}

cudaError_t launch_route_noaux(const moe_shape& s, int n_group, int topk_group,
                               const float* logits, const float* bias, int32_t* idx, float* w,
                               cudaStream_t st) {
    const unsigned grid = static_cast<unsigned>((s.T + kNxWarps - 1) / kNxWarps);
    const int threads = kNxWarps * 32;
    if (s.E <= 32)
        route_noaux_kernel<1><<<grid, threads, 0, st>>>(logits, bias, idx, w, s.T, s.E, s.k,
                                                        n_group, topk_group);
    else if (s.E <= 64)
        route_noaux_kernel<2><<<grid, threads, 0, st>>>(logits, bias, idx, w, s.T, s.E, s.k,
                                                        n_group, topk_group);
    else if (s.E <= 128)
        route_noaux_kernel<4><<<grid, threads, 0, st>>>(logits, bias, idx, w, s.T, s.E, s.k,
                                                        n_group, topk_group);
    else
        route_noaux_kernel<8><<<grid, threads, 0, st>>>(logits, bias, idx, w, s.T, s.E, s.k,
                                                        n_group, topk_group);
    return cudaGetLastError();
}

}  // namespace moe
