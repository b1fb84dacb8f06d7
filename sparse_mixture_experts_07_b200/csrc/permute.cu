// Dropless dispatch plan: per-expert counts, offsets and the stable
// permutation of the T*k slots by expert.
//
// "Mixture of Experts in Transformers", expert backends (grouped_mm): tokens
// are sorted and grouped by expert id before one grouped GEMM; "PhiMoE in
// Transformers", section 2 item 4: no token is dropped and there is no
// capacity factor, so every slot gets a place.
//
// Three launches over blocks of 2048 consecutive slots:
//   1. histogram: each block counts its slots per expert (shared-memory
//      atomics; integer counts, so the result is order-independent);
//   2. scan: one CTA turns the per-block counts into per-expert totals, the
//      exclusive offsets, and each block's starting position per expert;
//   3. scatter: each block ranks its slots stably (warp match + per-warp
//      counts, rounds in slot order) and writes perm and inv.
// The order (expert ascending, slot ascending) is fixed, so the plan is
// bit-identical run to run.  Workspace: nblocks * E int32.  A plan of a
// single block (T*k <= 2048) runs all three steps in one CTA and one launch.
#include "common.cuh"

namespace moe {

constexpr int kPermThreads = 256;
constexpr int kPermRounds = 8;
constexpr int kPermSlotsPerBlock = kPermThreads * kPermRounds;

__global__ void __launch_bounds__(kPermThreads) permute_hist_kernel(
    const int32_t* __restrict__ idx, int64_t n, int E, int32_t* __restrict__ blk_counts,
    int32_t* __restrict__ err_flag) {
    __shared__ int32_t hist[kMaxExperts];
    for (int e = threadIdx.x; e < E; e += kPermThreads) hist[e] = 0;
    __syncthreads();
    const int64_t base = static_cast<int64_t>(blockIdx.x) * kPermSlotsPerBlock;
    bool bad = false;
    for (int r = 0; r < kPermRounds; ++r) {
        const int64_t q = base + r * kPermThreads + threadIdx.x;
        if (q < n) {
            const int e = idx[q];
            if (e >= 0 && e < E) atomicAdd(&hist[e], 1);
            else bad = true;
        }
    }
    if (bad) raise_error(err_flag, MOE_ERR_BAD_INDEX);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += kPermThreads)
        blk_counts[static_cast<int64_t>(blockIdx.x) * E + e] = hist[e];
}

// One CTA.  blk_counts [nblk][E] becomes blk_base [nblk][E] in place.
__global__ void __launch_bounds__(kPermThreads) permute_scan_kernel(
    int32_t* __restrict__ blk, int nblk, int E, int32_t* __restrict__ counts,
    int32_t* __restrict__ offsets) {
    __shared__ int32_t warp_sum[kPermThreads / 32];
    const int e = threadIdx.x;
    int32_t run = 0;
    if (e < E) {
        for (int b = 0; b < nblk; ++b) {
            const int32_t c = blk[static_cast<int64_t>(b) * E + e];
            blk[static_cast<int64_t>(b) * E + e] = run;
            run += c;
        }
        counts[e] = run;
    }
    // exclusive scan of the per-expert totals (E <= 256 = blockDim)
    const int lane = e & 31, warp = e >> 5;
    int32_t v = (e < E) ? run : 0;
    int32_t incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        int32_t o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) warp_sum[warp] = incl;
    __syncthreads();
    int32_t before = 0;
    for (int w = 0; w < warp; ++w) before += warp_sum[w];
    const int32_t excl = before + incl - v;
    if (e < E) {
        offsets[e] = excl;
        if (e == E - 1) offsets[E] = excl + v;
        for (int b = 0; b < nblk; ++b) blk[static_cast<int64_t>(b) * E + e] += excl;
    }
}

__global__ void __launch_bounds__(kPermThreads) permute_scatter_kernel(
    const int32_t* __restrict__ idx, int64_t n, int E, const int32_t* __restrict__ blk_base,
    int32_t* __restrict__ perm, int32_t* __restrict__ inv) {
    __shared__ int32_t running[kMaxExperts];
    __shared__ int32_t wcnt[kPermThreads / 32][kMaxExperts];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int e = tid; e < E; e += kPermThreads)
        running[e] = blk_base[static_cast<int64_t>(blockIdx.x) * E + e];
    const int64_t base = static_cast<int64_t>(blockIdx.x) * kPermSlotsPerBlock;
    for (int r = 0; r < kPermRounds; ++r) {
        for (int i = tid; i < (kPermThreads / 32) * E; i += kPermThreads)
            wcnt[i / E][i % E] = 0;
        __syncthreads();
        const int64_t q = base + r * kPermThreads + tid;
        int e = -1;
        if (q < n) {
            e = idx[q];
            if (e < 0 || e >= E) e = -1;
        }
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int lane_rank = __popc(peers & ((1u << lane) - 1u));
        if (e >= 0 && lane_rank == 0) wcnt[warp][e] = __popc(peers);
        __syncthreads();
        if (e >= 0) {
            int32_t p = running[e] + lane_rank;
            for (int w = 0; w < warp; ++w) p += wcnt[w][e];
            perm[p] = static_cast<int32_t>(q);
            inv[q] = p;
        }
        __syncthreads();
        for (int ee = tid; ee < E; ee += kPermThreads) {
            int32_t s = 0;
            for (int w = 0; w < kPermThreads / 32; ++w) s += wcnt[w][ee];
            running[ee] += s;
        }
        __syncthreads();
    }
}

// Plans of at most one block of slots (T*k <= 2048, e.g. decode batches): the
// three steps above in one CTA and one launch, no workspace.
__global__ void __launch_bounds__(kPermThreads) permute_single_kernel(
    const int32_t* __restrict__ idx, int64_t n, int E, int32_t* __restrict__ counts,
    int32_t* __restrict__ offsets, int32_t* __restrict__ perm, int32_t* __restrict__ inv,
    int32_t* __restrict__ err_flag) {
    __shared__ int32_t hist[kMaxExperts];
    __shared__ int32_t running[kMaxExperts];
    __shared__ int32_t wcnt[kPermThreads / 32][kMaxExperts];
    __shared__ int32_t warp_sum[kPermThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int e = tid; e < E; e += kPermThreads) hist[e] = 0;
    __syncthreads();
    bool bad = false;
    for (int r = 0; r < kPermRounds; ++r) {
        const int64_t q = r * kPermThreads + tid;
        if (q < n) {
            const int e = idx[q];
            if (e >= 0 && e < E) atomicAdd(&hist[e], 1);
            else bad = true;
        }
    }
    if (bad) raise_error(err_flag, MOE_ERR_BAD_INDEX);
    __syncthreads();
    // exclusive scan of the counts (E <= 256 = blockDim)
    const int32_t v = tid < E ? hist[tid] : 0;
    int32_t incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int32_t o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) warp_sum[warp] = incl;
    __syncthreads();
    int32_t before = 0;
    for (int w = 0; w < warp; ++w) before += warp_sum[w];
    if (tid < E) {
        const int32_t excl = before + incl - v;
        counts[tid] = v;
        offsets[tid] = excl;
        running[tid] = excl;
        if (tid == E - 1) offsets[E] = excl + v;
    }
    // stable scatter, rounds in slot order (as permute_scatter_kernel)
    for (int r = 0; r < kPermRounds; ++r) {
        for (int i = tid; i < (kPermThreads / 32) * E; i += kPermThreads) wcnt[i / E][i % E] = 0;
        __syncthreads();
        const int64_t q = r * kPermThreads + tid;
        int e = -1;
        if (q < n) {
            e = idx[q];
            if (e < 0 || e >= E) e = -1;
        }
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int lane_rank = __popc(peers & ((1u << lane) - 1u));
        if (e >= 0 && lane_rank == 0) wcnt[warp][e] = __popc(peers);
        __syncthreads();
        if (e >= 0) {
            int32_t p = running[e] + lane_rank;
            for (int w = 0; w < warp; ++w) p += wcnt[w][e];
            perm[p] = static_cast<int32_t>(q);
            inv[q] = p;
        }
        __syncthreads();
        for (int ee = tid; ee < E; ee += kPermThreads) {
            int32_t s = 0;
            for (int w = 0; w < kPermThreads / 32; ++w) s += wcnt[w][ee];
            running[ee] += s;
        }
        __syncthreads();
    }
}

size_t permute_workspace_bytes(const moe_shape& s) {
    const int64_t n = s.T * s.k;
    const int64_t nblk = (n + kPermSlotsPerBlock - 1) / kPermSlotsPerBlock;
    return static_cast<size_t>(nblk) * s.E * sizeof(int32_t);
}

cudaError_t launch_permute(const moe_shape& s, const int32_t* idx, int32_t* counts,
                           int32_t* offsets, int32_t* perm, int32_t* inv, int32_t* err_flag,
                           void* workspace, cudaStream_t st) {
    const int64_t n = s.T * s.k;
    const int nblk = static_cast<int>((n + kPermSlotsPerBlock - 1) / kPermSlotsPerBlock);
    if (nblk == 1) {
        permute_single_kernel<<<1, kPermThreads, 0, st>>>(idx, n, s.E, counts, offsets, perm, inv,
                                                          err_flag);
        return cudaGetLastError();
    }
    int32_t* blk = static_cast<int32_t*>(workspace);
    if (nblk > 0) {
        permute_hist_kernel<<<nblk, kPermThreads, 0, st>>>(idx, n, s.E, blk, err_flag);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    permute_scan_kernel<<<1, kPermThreads, 0, st>>>(blk, nblk, s.E, counts, offsets);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || nblk == 0) return e;
    permute_scatter_kernel<<<nblk, kPermThreads, 0, st>>>(idx, n, s.E, blk, perm, inv);
    return cudaGetLastError();
}

}  // namespace moe

// ---------------------------------------------------------------------------
// moe_permute_noalloc: the same dispatch plan for callers that cannot allocate
// device memory - for example a plugin whose host framework owns every device
// allocation and hands it only its input and output buffers, or a latency-
// critical path where a cudaMalloc (which may synchronise the device) is not
// allowed.  The per-block expert counts live in a file-scope __device__ array
// of kNoallocScratchInts int32 (1 MiB); every GPU that loads this library holds
// it until the process exits.
//
// Host code must not pass `g_permute_scratch` itself to a kernel: on the host
// that name is only a stand-in, not a device address.  The device address is
// looked up once per device with cudaGetSymbolAddress, on the first call made
// while that device is current, and cached; make that first call before any
// stream capture.  The array keeps the last call's contents; the histogram
// kernel overwrites every entry it later reads, so nothing needs clearing.
// All calls share the one array: calls whose kernels may overlap on the GPU
// (different streams without ordering between them) race on it.
#include <mutex>

namespace moe {
constexpr int64_t kNoallocScratchInts = 256 * 1024;
constexpr int kNoallocMaxDevices = 64;
}  // namespace moe

static __device__ __align__(256) int32_t g_permute_scratch[moe::kNoallocScratchInts];

namespace {

std::mutex g_scratch_mu;
void* g_scratch_ptr[moe::kNoallocMaxDevices] = {nullptr};

// Device address of g_permute_scratch on the current device (looked up once).
cudaError_t noalloc_scratch(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= moe::kNoallocMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_permute_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" moe_status moe_permute_noalloc(const moe_shape* shape, const int32_t* topk_idx,
                                          int32_t* counts, int32_t* offsets, int32_t* perm,
                                          int32_t* inv, int32_t* err_flag, void* stream) {
    if (!shape) return MOE_ERR_INVALID_ARG;
    const moe_shape& s = *shape;
    if (s.T < 0 || s.H <= 0 || s.I <= 0 || s.E <= 0 || s.k <= 0 || s.k > s.E ||
        s.n_shared < 0 || (s.n_shared > 0 && s.I_shared <= 0) ||
        (s.dtype != MOE_F32 && s.dtype != MOE_BF16))
        return MOE_ERR_INVALID_ARG;
    if (s.E > moe::kMaxExperts || s.k > moe::kMaxK || s.T * s.k >= (int64_t(1) << 31))
        return MOE_ERR_UNSUPPORTED;
    if (!counts || !offsets) return MOE_ERR_INVALID_ARG;
    if (s.T > 0 && (!topk_idx || !perm || !inv)) return MOE_ERR_INVALID_ARG;
    // the plan needs ceil(T*k / 2048) * E ints of scratch
    if (moe::permute_workspace_bytes(s) > sizeof(int32_t) * moe::kNoallocScratchInts)
        return MOE_ERR_UNSUPPORTED;
    void* scratch = nullptr;
    if (noalloc_scratch(&scratch) != cudaSuccess) return MOE_ERR_CUDA;
    cudaError_t e = moe::launch_permute(s, topk_idx, counts, offsets, perm, inv, err_flag, scratch,
                                        static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
