// Combine: scatter the slot outputs back to token order and sum them.
//
// "Mixture of Experts in Transformers", expert backends: after the projections
// and the routing weights, the runtime gathers and reorders the results into
// token order.  y[t] = sum_j y_slots[inv[t*k+j]] + sum_s y_slots[T*k + s*T + t]
// (shared experts: Instella-MoE walk-through, FarSkipMoE "routed + shared";
// GraniteMoeSWA decoder layer, moe output + shared_mlp).  The sum is float32 in
// a fixed order (j ascending, then s ascending) and is rounded once.
//
// float32: one CTA of 256 threads per token row, each thread owning 16-byte
// vectors (or single elements when H % 4 != 0) of the row, so every y_slots
// row is read once, coalesced; bf16: the persistent kernel further down.
// Memory-bound: (k + S) * H * elem bytes read and H * elem bytes written per
// token.
#include "common.cuh"

namespace moe {

template <typename T, int VEC>
__global__ void __launch_bounds__(256) combine_kernel(const T* __restrict__ y_slots,
                                                      const int32_t* __restrict__ inv,
                                                      T* __restrict__ y, int64_t n_tokens, int H,
                                                      int k, int S) {
    const int64_t routed_rows = n_tokens * k;
    for (int64_t t = blockIdx.x; t < n_tokens; t += gridDim.x) {
        int64_t rows[kMaxK + kMaxShared];
        for (int j = 0; j < k; ++j) rows[j] = inv[t * k + j];
        for (int s = 0; s < S; ++s) rows[k + s] = routed_rows + s * n_tokens + t;
        for (int c = threadIdx.x * VEC; c < H; c += 256 * VEC) {
            float acc[VEC];
#pragma unroll
            for (int v = 0; v < VEC; ++v) acc[v] = 0.f;
            for (int j = 0; j < k + S; ++j) {
                const T* src = y_slots + rows[j] * H + c;
                if constexpr (VEC == 4) {
                    const float4 u = *reinterpret_cast<const float4*>(src);
                    acc[0] += u.x; acc[1] += u.y; acc[2] += u.z; acc[3] += u.w;
                } else {
#pragma unroll
                    for (int v = 0; v < VEC; ++v) acc[v] += ElemIO<T>::load(src, v);
                }
            }
            T* dst = y + t * H + c;
            if constexpr (VEC == 4) {
                *reinterpret_cast<float4*>(dst) = make_float4(acc[0], acc[1], acc[2], acc[3]);
            } else {
#pragma unroll
                for (int v = 0; v < VEC; ++v) ElemIO<T>::store(dst, v, acc[v]);
            }
        }
    }
}

// bf16, H % 8 == 0: a persistent grid; each CTA walks its tokens t, t + grid,
// ... and loads the slot indices of its next token while it sums the current
// one, so the index round trip overlaps the row loads.  Same sum, same order.
__global__ void __launch_bounds__(256) combine_bf16_pipelined_kernel(
    const uint4* __restrict__ y_slots, const int32_t* __restrict__ inv, uint4* __restrict__ y,
    int64_t n_tokens, int vec_per_row, int k, int S) {
    const int64_t routed_rows = n_tokens * k;
    const int nrows = k + S;
    int64_t t = blockIdx.x;
    pdl_launch_dependents();     // launched as a programmatic dependent
    pdl_wait();
    // the threads < k fetch one slot index each for the next token
    int32_t next_idx = (t < n_tokens && static_cast<int>(threadIdx.x) < k)
                           ? inv[t * k + threadIdx.x] : 0;
    __shared__ int64_t rows_sh[2][kMaxK + kMaxShared];
    int buf = 0;
    for (; t < n_tokens; t += gridDim.x) {
        if (static_cast<int>(threadIdx.x) < k) rows_sh[buf][threadIdx.x] = next_idx;
        if (static_cast<int>(threadIdx.x) < S)
            rows_sh[buf][k + threadIdx.x] = routed_rows + threadIdx.x * n_tokens + t;
        __syncthreads();
        const int64_t tn = t + gridDim.x;
        if (tn < n_tokens && static_cast<int>(threadIdx.x) < k) next_idx = inv[tn * k + threadIdx.x];
        for (int v = threadIdx.x; v < vec_per_row; v += 256) {
            float acc[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = 0.f;
            // up to four rows' loads in flight at once, summed in row order
            for (int j = 0; j < nrows; j += 4) {
                const int n = nrows - j < 4 ? nrows - j : 4;
                uint4 u[4];
#pragma unroll
                for (int r = 0; r < 4; ++r)
                    if (r < n) u[r] = y_slots[rows_sh[buf][j + r] * vec_per_row + v];
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    if (r >= n) break;
                    const uint32_t w[4] = {u[r].x, u[r].y, u[r].z, u[r].w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        acc[2 * q] += bf16_to_f32(static_cast<uint16_t>(w[q] & 0xffffu));
                        acc[2 * q + 1] += bf16_to_f32(static_cast<uint16_t>(w[q] >> 16));
                    }
                }
            }
            uint4 o;
            o.x = pack_bf16x2(acc[0], acc[1]);
            o.y = pack_bf16x2(acc[2], acc[3]);
            o.z = pack_bf16x2(acc[4], acc[5]);
            o.w = pack_bf16x2(acc[6], acc[7]);
            y[t * vec_per_row + v] = o;
        }
        buf ^= 1;
    }
}

cudaError_t launch_combine(const moe_shape& s, const void* y_slots, const int32_t* inv, void* y,
                           cudaStream_t st) {
    if (s.dtype == MOE_BF16) {
        // as many CTAs as are resident at once, so that every CTA starts
        // right away (looked up once per device)
        static int resident[64] = {0};
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
        if (resident[dev] <= 0) {
            int sms = 148, per_sm = 0;
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                    &per_sm, combine_bf16_pipelined_kernel, 256, 0) != cudaSuccess ||
                per_sm <= 0)
                per_sm = 4;
            resident[dev] = sms * per_sm;
        }
        const int64_t cap = resident[dev];
        const unsigned grid = static_cast<unsigned>(s.T < cap ? s.T : cap);
        return launch_pdl(combine_bf16_pipelined_kernel, dim3(grid), dim3(256), 0, st,
                          static_cast<const uint4*>(y_slots), inv, static_cast<uint4*>(y), s.T,
                          s.H / 8, s.k, s.n_shared);
    }
    const unsigned grid = static_cast<unsigned>(s.T < 1048576 ? s.T : 1048576);
    if (s.H % 4 == 0) {
        combine_kernel<float, 4><<<grid, 256, 0, st>>>(static_cast<const float*>(y_slots), inv,
                                                       static_cast<float*>(y), s.T, s.H, s.k,
                                                       s.n_shared);
    } else {
        combine_kernel<float, 1><<<grid, 256, 0, st>>>(static_cast<const float*>(y_slots), inv,
                                                       static_cast<float*>(y), s.T, s.H, s.k,
                                                       s.n_shared);
    }
    return cudaGetLastError();
}

// x_perm[p] = x[perm[p] / k]: the rows of x in sorted slot order (bf16, H % 8 == 0).
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4* __restrict__ x,
                                                          const int32_t* __restrict__ perm,
                                                          uint4* __restrict__ x_perm, int64_t n_rows,
                                                          int vec_per_row, int k) {
    const int64_t total = n_rows * vec_per_row;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * 256;
    // four pieces per thread and pass, their loads in flight together
    for (int64_t i0 = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; i0 < total;
         i0 += 4 * stride) {
        uint4 val[4];
        bool ok[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int64_t i = i0 + u * stride;
            ok[u] = false;
            if (i < total) {
                const int64_t p = i / vec_per_row;
                const int v = static_cast<int>(i - p * vec_per_row);
                const int64_t q = perm[p];
                ok[u] = q >= 0 && q < n_rows;
                if (ok[u]) val[u] = x[(q / k) * vec_per_row + v];
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (ok[u]) x_perm[i0 + u * stride] = val[u];
    }
}

// inv[perm[p]] = p: the sorted position of every slot.
__global__ void __launch_bounds__(256) invert_perm_kernel(const int32_t* __restrict__ perm,
                                                          int32_t* __restrict__ inv, int64_t n) {
    for (int64_t p = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; p < n;
         p += static_cast<int64_t>(gridDim.x) * 256) {
        const int32_t q = perm[p];
        // a plan with skipped slots (bad expert index) leaves holes: stay in bounds
        if (q >= 0 && q < n) inv[q] = static_cast<int32_t>(p);
    }
}

// Token-major gather: thread i reads the 16-byte piece i of x once and writes
// it to the k sorted rows of that token, x_perm[inv[t*k + j]] (bf16, H % 8 == 0).
// x is read from memory once even when it does not fit in L2.
__global__ void __launch_bounds__(256) gather_by_token_kernel(const uint4* __restrict__ x,
                                                              const int32_t* __restrict__ inv,
                                                              uint4* __restrict__ x_perm,
                                                              int64_t n_tokens, int vec_per_row,
                                                              int k) {
    const int64_t total = n_tokens * vec_per_row;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * 256;
    // four pieces per thread and pass, their loads in flight together
    for (int64_t i0 = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; i0 < total;
         i0 += 4 * stride) {
        uint4 val[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (i0 + u * stride < total) val[u] = x[i0 + u * stride];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int64_t i = i0 + u * stride;
            if (i >= total) break;
            const int64_t t = i / vec_per_row;
            const int v = static_cast<int>(i - t * vec_per_row);
            for (int j = 0; j < k; ++j) {
                const int64_t p = inv[t * k + j];
                if (p >= 0 && p < n_tokens * k) x_perm[p * vec_per_row + v] = val[u];
            }
        }
    }
}

cudaError_t launch_gather_by_token(const moe_shape& s, const void* x, const int32_t* perm,
                                   int32_t* inv_scratch, void* x_perm, int num_sms,
                                   cudaStream_t st) {
    const int64_t n = s.T * s.k;
    int64_t grid = (n + 255) / 256;
    if (grid > static_cast<int64_t>(num_sms) * 8) grid = static_cast<int64_t>(num_sms) * 8;
    if (grid < 1) return cudaSuccess;
    invert_perm_kernel<<<static_cast<unsigned>(grid), 256, 0, st>>>(perm, inv_scratch, n);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int vpr = s.H / 8;
    const int64_t total = s.T * vpr;
    grid = (total + 255) / 256;
    if (grid > static_cast<int64_t>(num_sms) * 16) grid = static_cast<int64_t>(num_sms) * 16;
    gather_by_token_kernel<<<static_cast<unsigned>(grid), 256, 0, st>>>(
        static_cast<const uint4*>(x), inv_scratch, static_cast<uint4*>(x_perm), s.T, vpr, s.k);
    return cudaGetLastError();
}

cudaError_t launch_gather_rows(const moe_shape& s, const void* x, const int32_t* perm,
                               void* x_perm, int num_sms, cudaStream_t st) {
    const int64_t n_rows = s.T * s.k;
    const int vpr = s.H / 8;
    const int64_t total = n_rows * vpr;
    int64_t grid = (total + 255) / 256;
    if (grid > static_cast<int64_t>(num_sms) * 16) grid = static_cast<int64_t>(num_sms) * 16;
    if (grid < 1) return cudaSuccess;
    gather_rows_kernel<<<static_cast<unsigned>(grid), 256, 0, st>>>(
        static_cast<const uint4*>(x), perm, static_cast<uint4*>(x_perm), n_rows, vpr, s.k);
    return cudaGetLastError();
}

}  // namespace moe
