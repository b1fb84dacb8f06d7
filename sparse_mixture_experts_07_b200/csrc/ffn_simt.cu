// Grouped expert FFN on the CUDA cores, float32 throughout.
//
// Used for float32 activations and weights, where the tensor cores' tf32 or
// bf16 inputs would not meet float32 accuracy.  Same structure as the
// tensor-core path: GEMM 1 computes h = SiLU(A Wg^T) * (A Wu^T) per expert
// group ("PhiMoE in Transformers", section 2 item 3: packed gate_up_proj,
// chunked into gate then up, act(gate) * up); GEMM 2 computes
// y_slots = scale * h Wd^T ("Mixture of Experts in Transformers", expert
// backends: the routing weights are applied to the projected results).
//
// Tiles are 32 rows x 32 columns; 256 threads each own 4 rows of one column.
// A routed group reads its A rows through perm (x[perm[p] / k]), so no
// permuted copy of x is materialised; a shared group reads x directly.
#include "common.cuh"

namespace moe {

constexpr int kSimtBM = 32, kSimtBN = 32, kSimtBK = 32;

struct SimtArgs {
    const void* x;          // [T, H]
    const int32_t* offsets; // [E+1]
    const int32_t* perm;    // [T*k]
    const float* topk_w;    // [T*k]
    const void* gate_up;    // [E, 2I, H]
    const void* down;       // [E, H, I]
    const void* sh_gate_up; // [S, 2Is, H]
    const void* sh_down;    // [S, H, Is]
    void* h_routed;         // [T*k, I]
    void* h_shared;         // [S*T, Is]
    void* y_slots;          // [T*k + S*T, H]
    int64_t T;
    int H, I, E, k, S, Is;
    float routed_scale;
};

__device__ __forceinline__ float silu_f32(float z) { return z / (1.f + expf(-z)); }

template <typename T>
__global__ void __launch_bounds__(256) simt_gate_up_kernel(SimtArgs a) {
    __shared__ GroupTable gt;
    __shared__ float As[kSimtBM][kSimtBK + 1];
    __shared__ float Bg[kSimtBN][kSimtBK + 1];
    __shared__ float Bu[kSimtBN][kSimtBK + 1];
    __shared__ int64_t arow[kSimtBM];
    stage_offsets(gt.tile_start, a.offsets, a.E);
    __syncthreads();
    if (threadIdx.x == 0) build_group_table(gt, a.E, a.S, a.T, kSimtBM, 1, 1);
    __syncthreads();
    const int tile = blockIdx.x;
    if (tile >= gt.total_tiles) return;
    const int g = find_group(gt, tile);
    const int m0 = (tile - gt.tile_start[g]) * kSimtBM;
    const int rows = gt.rows[g];
    const bool routed = g < a.E;
    const int N = routed ? a.I : a.Is;
    const int n0 = blockIdx.y * kSimtBN;
    if (n0 >= N) return;
    const T* x = static_cast<const T*>(a.x);
    const T* W;
    if (routed) W = static_cast<const T*>(a.gate_up) + static_cast<int64_t>(g) * 2 * a.I * a.H;
    else W = static_cast<const T*>(a.sh_gate_up) + static_cast<int64_t>(g - a.E) * 2 * a.Is * a.H;
    if (threadIdx.x < kSimtBM) {
        const int m = m0 + threadIdx.x;
        int64_t r = -1;
        if (m < rows) r = routed ? a.perm[gt.row0[g] + m] / a.k : m;
        arow[threadIdx.x] = r;
    }
    const int c = threadIdx.x & 31, r4 = threadIdx.x >> 5;
    float accg[4] = {0.f, 0.f, 0.f, 0.f}, accu[4] = {0.f, 0.f, 0.f, 0.f};
    for (int k0 = 0; k0 < a.H; k0 += kSimtBK) {
        __syncthreads();
        for (int i = threadIdx.x; i < kSimtBM * kSimtBK; i += 256) {
            const int rr = i / kSimtBK, kk = i % kSimtBK;
            const int64_t xr = arow[rr];
            As[rr][kk] = (xr >= 0 && k0 + kk < a.H) ? ElemIO<T>::load(x, xr * a.H + k0 + kk) : 0.f;
            const int n = n0 + rr;
            float vg = 0.f, vu = 0.f;
            if (n < N && k0 + kk < a.H) {
                vg = ElemIO<T>::load(W, static_cast<int64_t>(n) * a.H + k0 + kk);
                vu = ElemIO<T>::load(W, static_cast<int64_t>(N + n) * a.H + k0 + kk);
            }
            Bg[rr][kk] = vg;
            Bu[rr][kk] = vu;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < kSimtBK; ++kk) {
            const float bg = Bg[c][kk], bu = Bu[c][kk];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float av = As[r4 * 4 + i][kk];
                accg[i] = fmaf(av, bg, accg[i]);
                accu[i] = fmaf(av, bu, accu[i]);
            }
        }
    }
    const int n = n0 + c;
    if (n >= N) return;
    T* hout = static_cast<T*>(routed ? a.h_routed : a.h_shared);
    const int64_t hrow0 = routed ? gt.row0[g] : static_cast<int64_t>(g - a.E) * a.T;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + r4 * 4 + i;
        if (m < rows) ElemIO<T>::store(hout, (hrow0 + m) * N + n, silu_f32(accg[i]) * accu[i]);
    }
}

template <typename T>
__global__ void __launch_bounds__(256) simt_down_kernel(SimtArgs a) {
    __shared__ GroupTable gt;
    __shared__ float As[kSimtBM][kSimtBK + 1];
    __shared__ float Bd[kSimtBN][kSimtBK + 1];
    stage_offsets(gt.tile_start, a.offsets, a.E);
    __syncthreads();
    if (threadIdx.x == 0) build_group_table(gt, a.E, a.S, a.T, kSimtBM, 1, 1);
    __syncthreads();
    const int tile = blockIdx.x;
    if (tile >= gt.total_tiles) return;
    const int g = find_group(gt, tile);
    const int m0 = (tile - gt.tile_start[g]) * kSimtBM;
    const int rows = gt.rows[g];
    const bool routed = g < a.E;
    const int K = routed ? a.I : a.Is;
    const int n0 = blockIdx.y * kSimtBN;
    const T* hin = static_cast<const T*>(routed ? a.h_routed : a.h_shared);
    const int64_t hrow0 = routed ? gt.row0[g] : static_cast<int64_t>(g - a.E) * a.T;
    const T* W;
    if (routed) W = static_cast<const T*>(a.down) + static_cast<int64_t>(g) * a.H * a.I;
    else W = static_cast<const T*>(a.sh_down) + static_cast<int64_t>(g - a.E) * a.H * a.Is;
    const int c = threadIdx.x & 31, r4 = threadIdx.x >> 5;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int k0 = 0; k0 < K; k0 += kSimtBK) {
        __syncthreads();
        for (int i = threadIdx.x; i < kSimtBM * kSimtBK; i += 256) {
            const int rr = i / kSimtBK, kk = i % kSimtBK;
            const int m = m0 + rr;
            As[rr][kk] = (m < rows && k0 + kk < K) ? ElemIO<T>::load(hin, (hrow0 + m) * K + k0 + kk)
                                                   : 0.f;
            const int n = n0 + rr;
            Bd[rr][kk] = (n < a.H && k0 + kk < K)
                             ? ElemIO<T>::load(W, static_cast<int64_t>(n) * K + k0 + kk)
                             : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < kSimtBK; ++kk) {
            const float b = Bd[c][kk];
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[i] = fmaf(As[r4 * 4 + i][kk], b, acc[i]);
        }
    }
    const int n = n0 + c;
    if (n >= a.H) return;
    T* y = static_cast<T*>(a.y_slots);
    const int64_t routed_rows = a.T * a.k;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + r4 * 4 + i;
        if (m >= rows) continue;
        int64_t orow;
        float scale;
        if (routed) {
            const int64_t p = gt.row0[g] + m;
            orow = p;
            scale = a.routed_scale * a.topk_w[a.perm[p]];
        } else {
            orow = routed_rows + static_cast<int64_t>(g - a.E) * a.T + m;
            scale = 1.f;
        }
        ElemIO<T>::store(y, orow * a.H + n, scale * acc[i]);
    }
}

cudaError_t launch_ffn_simt(const moe_shape& s, const void* x, const int32_t* offsets,
                            const int32_t* perm, const float* topk_w, const void* gate_up,
                            const void* down, const void* sh_gate_up, const void* sh_down,
                            void* h_routed, void* h_shared, void* y_slots, cudaStream_t st) {
    SimtArgs a{x, offsets, perm, topk_w, gate_up, down, sh_gate_up, sh_down,
               h_routed, h_shared, y_slots, s.T, s.H, s.I, s.E, s.k, s.n_shared, s.I_shared,
               s.routed_scale};
    const int64_t mt = (s.T * s.k + kSimtBM - 1) / kSimtBM + s.E +
                       static_cast<int64_t>(s.n_shared) * ((s.T + kSimtBM - 1) / kSimtBM);
    const int nmax = s.I > s.I_shared ? s.I : s.I_shared;
    dim3 g1(static_cast<unsigned>(mt), (nmax + kSimtBN - 1) / kSimtBN);
    dim3 g2(static_cast<unsigned>(mt), (s.H + kSimtBN - 1) / kSimtBN);
    if (s.dtype != MOE_F32) return cudaErrorInvalidValue;
    simt_gate_up_kernel<float><<<g1, 256, 0, st>>>(a);
    simt_down_kernel<float><<<g2, 256, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace moe
