// Expert parallelism: the per-rank pieces of the block when the routed experts
// are split across ranks.
//
// "Mixture of Experts in Transformers", section "expert parallelism": with
// GroupedGemmParallel each rank keeps E/N of the experts (a slice of dim 0 of
// the packed expert weights); RouterParallel maps the router's global expert
// indices to the rank's local ones and masks the experts of the other ranks,
// and the ranks' partial outputs are summed by an all-reduce.
//
// combine_experts_kernel is that masked combine: for each token, the float32
// sum of its slot rows whose expert lies in [e_begin, e_end) (j ascending),
// plus the shared experts' rows when this rank computed them.  The partial
// stays float32 so that the all-reduce adds unrounded partials and the block
// output is rounded once, by cast_f32_kernel, after the exchange.
#include "common.cuh"

namespace moe {

constexpr int kEpThreads = 256;

// One CTA per token (grid-stride); bf16 rows as 16-byte vectors of 8.
__global__ void __launch_bounds__(kEpThreads) combine_experts_bf16_kernel(
    const uint4* __restrict__ y_slots, const int32_t* __restrict__ inv,
    const int32_t* __restrict__ topk_idx, float4* __restrict__ y32, int64_t n_tokens,
    int vec_per_row, int k, int S, int e_begin, int e_end) {
    __shared__ int64_t rows_sh[kMaxK + kMaxShared];
    __shared__ int n_sh;
    const int64_t routed_rows = n_tokens * k;
    for (int64_t t = blockIdx.x; t < n_tokens; t += gridDim.x) {
        if (threadIdx.x == 0) {
            int n = 0;
            for (int j = 0; j < k; ++j) {
                const int e = topk_idx[t * k + j];
                if (e >= e_begin && e < e_end) rows_sh[n++] = inv[t * k + j];
            }
            for (int s = 0; s < S; ++s) rows_sh[n++] = routed_rows + s * n_tokens + t;
            n_sh = n;
        }
        __syncthreads();
        const int n = n_sh;
        for (int v = threadIdx.x; v < vec_per_row; v += kEpThreads) {
            float acc[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = 0.f;
            for (int j = 0; j < n; ++j) {
                const uint4 u = y_slots[rows_sh[j] * vec_per_row + v];
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    acc[2 * q] += bf16_to_f32(static_cast<uint16_t>(w[q] & 0xffffu));
                    acc[2 * q + 1] += bf16_to_f32(static_cast<uint16_t>(w[q] >> 16));
                }
            }
            float4* dst = y32 + (t * vec_per_row + v) * 2;
            dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
            dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
        }
        __syncthreads();
    }
}

// float32 slot rows, any H: one CTA per token, one column per thread step.
__global__ void __launch_bounds__(kEpThreads) combine_experts_f32_kernel(
    const float* __restrict__ y_slots, const int32_t* __restrict__ inv,
    const int32_t* __restrict__ topk_idx, float* __restrict__ y32, int64_t n_tokens, int H,
    int k, int S, int e_begin, int e_end) {
    __shared__ int64_t rows_sh[kMaxK + kMaxShared];
    __shared__ int n_sh;
    const int64_t routed_rows = n_tokens * k;
    for (int64_t t = blockIdx.x; t < n_tokens; t += gridDim.x) {
        if (threadIdx.x == 0) {
            int n = 0;
            for (int j = 0; j < k; ++j) {
                const int e = topk_idx[t * k + j];
                if (e >= e_begin && e < e_end) rows_sh[n++] = inv[t * k + j];
            }
            for (int s = 0; s < S; ++s) rows_sh[n++] = routed_rows + s * n_tokens + t;
            n_sh = n;
        }
        __syncthreads();
        const int n = n_sh;
        for (int c = threadIdx.x; c < H; c += kEpThreads) {
            float acc = 0.f;
            for (int j = 0; j < n; ++j) acc += y_slots[rows_sh[j] * H + c];
            y32[t * H + c] = acc;
        }
        __syncthreads();
    }
}

// y = y32 rounded once to the block's dtype (round to nearest even).
__global__ void __launch_bounds__(kEpThreads) cast_f32_bf16_kernel(const float4* __restrict__ src,
                                                                   uint2* __restrict__ dst,
                                                                   int64_t n4) {
    for (int64_t i = blockIdx.x * static_cast<int64_t>(kEpThreads) + threadIdx.x; i < n4;
         i += static_cast<int64_t>(gridDim.x) * kEpThreads) {
        const float4 v = src[i];
        dst[i] = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
    }
}

__global__ void __launch_bounds__(kEpThreads) cast_f32_bf16_tail_kernel(
    const float* __restrict__ src, __nv_bfloat16* __restrict__ dst, int64_t n) {
    for (int64_t i = blockIdx.x * static_cast<int64_t>(kEpThreads) + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * kEpThreads)
        dst[i] = __float2bfloat16_rn(src[i]);
}

static int grid_for(int64_t n_items, int num_sms) {
    const int64_t cap = static_cast<int64_t>(num_sms) * 8;
    return static_cast<int>(n_items < cap ? (n_items > 0 ? n_items : 1) : cap);
}

cudaError_t launch_combine_experts(const moe_shape& s, int e_begin, int e_end, int with_shared,
                                   const void* y_slots, const int32_t* inv,
                                   const int32_t* topk_idx, float* y32, int num_sms,
                                   cudaStream_t st) {
    const int S = with_shared ? s.n_shared : 0;
    const int grid = grid_for(s.T, num_sms);
    if (s.dtype == MOE_BF16) {
        combine_experts_bf16_kernel<<<grid, kEpThreads, 0, st>>>(
            static_cast<const uint4*>(y_slots), inv, topk_idx, reinterpret_cast<float4*>(y32),
            s.T, s.H / 8, s.k, S, e_begin, e_end);
    } else {
        combine_experts_f32_kernel<<<grid, kEpThreads, 0, st>>>(
            static_cast<const float*>(y_slots), inv, topk_idx, y32, s.T, s.H, s.k, S, e_begin,
            e_end);
    }
    return cudaGetLastError();
}

cudaError_t launch_cast_f32(const moe_shape& s, const float* y32, void* y, int num_sms,
                            cudaStream_t st) {
    const int64_t n = s.T * static_cast<int64_t>(s.H);
    if (s.dtype == MOE_F32)
        return cudaMemcpyAsync(y, y32, static_cast<size_t>(n) * 4, cudaMemcpyDeviceToDevice, st);
    if (n % 4 == 0) {
        cast_f32_bf16_kernel<<<grid_for((n / 4 + kEpThreads - 1) / kEpThreads, num_sms), kEpThreads,
                               0, st>>>(reinterpret_cast<const float4*>(y32),
                                        static_cast<uint2*>(y), n / 4);
    } else {
        cast_f32_bf16_tail_kernel<<<grid_for((n + kEpThreads - 1) / kEpThreads, num_sms),
                                    kEpThreads, 0, st>>>(y32, static_cast<__nv_bfloat16*>(y), n);
    }
    return cudaGetLastError();
}

}  // namespace moe
