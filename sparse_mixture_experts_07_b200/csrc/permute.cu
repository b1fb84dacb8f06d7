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
// bit-identical run to run.  Workspace: nblocks * E int32.
//
// Up to 8 * 8 * 1024 slots, the plan runs instead as ONE launch on one
// thread-block cluster of up to 8 CTAs of 1024 threads (permute_cluster_kernel):
// each CTA counts its contiguous slice of slots, reads the other CTAs'
// counts from their shared memory (DSMEM) to find its starting position per
// expert, and ranks its slots with the same stable scheme.  No workspace.
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
        // 16 independent loads in flight, then their running prefix
        constexpr int B = 16;
        for (int b0 = 0; b0 < nblk; b0 += B) {
            int32_t c[B];
#pragma unroll
            for (int j = 0; j < B; ++j)
                c[j] = b0 + j < nblk ? blk[static_cast<int64_t>(b0 + j) * E + e] : 0;
#pragma unroll
            for (int j = 0; j < B; ++j) {
                if (b0 + j < nblk) blk[static_cast<int64_t>(b0 + j) * E + e] = run;
                run += c[j];
            }
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
    __shared__ int32_t running[2][kMaxExperts];
    // per-warp counts of the current round, stamped with the round in the high
    // half so that entries left from earlier rounds read as zero
    __shared__ int32_t wcnt[kPermThreads / 32][kMaxExperts];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int e = tid; e < E; e += kPermThreads)
        running[0][e] = blk_base[static_cast<int64_t>(blockIdx.x) * E + e];
    for (int i = tid; i < (kPermThreads / 32) * kMaxExperts; i += kPermThreads)
        (&wcnt[0][0])[i] = -1;
    const int64_t base = static_cast<int64_t>(blockIdx.x) * kPermSlotsPerBlock;
    int ev[kPermRounds];
#pragma unroll
    for (int r = 0; r < kPermRounds; ++r) {
        const int64_t q = base + r * kPermThreads + tid;
        int e = q < n ? idx[q] : -1;
        ev[r] = (e >= 0 && e < E) ? e : -1;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kPermRounds; ++r) {
        const int cur = r & 1;
        const int e = ev[r];
        const int64_t q = base + r * kPermThreads + tid;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int lane_rank = __popc(peers & ((1u << lane) - 1u));
        if (e >= 0 && lane_rank == 0) wcnt[warp][e] = (r << 16) | __popc(peers);
        __syncthreads();
        if (e >= 0) {
            int32_t p = running[cur][e] + lane_rank;
            for (int w = 0; w < warp; ++w) {
                const int32_t v = wcnt[w][e];
                if ((v >> 16) == r) p += v & 0xffff;
            }
            perm[p] = static_cast<int32_t>(q);
            inv[q] = p;
        }
        for (int ee = tid; ee < E; ee += kPermThreads) {
            int32_t sum = 0;
            for (int w = 0; w < kPermThreads / 32; ++w) {
                const int32_t v = wcnt[w][ee];
                if ((v >> 16) == r) sum += v & 0xffff;
            }
            running[cur ^ 1][ee] = running[cur][ee] + sum;
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// One-launch plan on a cluster (see the header comment).  CTA c of the
// cluster owns slots [c * chunk, (c + 1) * chunk); ROUNDS * 1024 >= chunk.
constexpr int kPcThreads = 1024;
constexpr int kPcWarps = kPcThreads / 32;
constexpr int kPcMaxCluster = 8;

template <int ROUNDS>
__global__ void __launch_bounds__(kPcThreads, 1) permute_cluster_kernel(
    const int32_t* __restrict__ idx, int64_t n, int E, int64_t chunk, int32_t* __restrict__ counts,
    int32_t* __restrict__ offsets, int32_t* __restrict__ perm, int32_t* __restrict__ inv,
    int32_t* __restrict__ err_flag) {
    __shared__ int32_t hist[kMaxExperts];
    __shared__ int32_t running[2][kMaxExperts];
    // per-warp counts of the current round, stamped with the round in the high
    // half so that entries left from earlier rounds read as zero
    __shared__ int32_t wcnt[kPcWarps][kMaxExperts];
    __shared__ int32_t warp_sum[kPcWarps];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int rank = static_cast<int>(cluster_ctarank());
    const int csize = static_cast<int>(gridDim.x);
    const int64_t lo = rank * chunk;
    const int64_t hi = lo + chunk < n ? lo + chunk : n;

    // launched as a programmatic dependent: shared memory is cleared while
    // the router finishes, its indices read after pdl_wait
    pdl_launch_dependents();
    for (int e = tid; e < E; e += kPcThreads) hist[e] = 0;
    for (int i = tid; i < kPcWarps * kMaxExperts; i += kPcThreads)
        (&wcnt[0][0])[i] = -1;                                  // stamp -1: no round
    pdl_wait();
    __syncthreads();
    // this thread's slots, one per round, kept in registers
    int ev[ROUNDS];
    bool bad = false;
#pragma unroll
    for (int r = 0; r < ROUNDS; ++r) {
        const int64_t q = lo + static_cast<int64_t>(r) * kPcThreads + tid;
        ev[r] = q < hi ? idx[q] : -1;
    }
#pragma unroll
    for (int r = 0; r < ROUNDS; ++r) {
        const int64_t q = lo + static_cast<int64_t>(r) * kPcThreads + tid;
        if (q < hi) {
            if (ev[r] >= 0 && ev[r] < E) atomicAdd(&hist[ev[r]], 1);
            else { bad = true; ev[r] = -1; }
        }
    }
    if (bad) raise_error(err_flag, MOE_ERR_BAD_INDEX);
    cluster_sync();                                             // every CTA's hist is final

    // per expert: total over the cluster and the count of the CTAs before this one
    int32_t total = 0, before_cta = 0;
    if (tid < E) {
        const uint32_t local = smem_u32(&hist[tid]);
        for (int c = 0; c < csize; ++c) {
            int32_t v;
            asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(mapa_shared(local, c))
                         : "memory");
            total += v;
            if (c < rank) before_cta += v;
        }
    }
    // exclusive scan of the totals over experts (E <= 256 < blockDim)
    int32_t incl = total;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int32_t o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) warp_sum[warp] = incl;
    __syncthreads();
    if (tid < E) {
        int32_t excl = incl - total;
        for (int w = 0; w < warp; ++w) excl += warp_sum[w];
        running[0][tid] = excl + before_cta;
        if (rank == 0) {
            counts[tid] = total;
            offsets[tid] = excl;
            if (tid == E - 1) offsets[E] = excl + total;
        }
    }
    __syncthreads();

    // stable scatter, rounds in slot order
#pragma unroll
    for (int r = 0; r < ROUNDS; ++r) {
        const int cur = r & 1;
        const int e = ev[r];
        const int64_t q = lo + static_cast<int64_t>(r) * kPcThreads + tid;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int lane_rank = __popc(peers & ((1u << lane) - 1u));
        if (e >= 0 && lane_rank == 0) wcnt[warp][e] = (r << 16) | __popc(peers);
        __syncthreads();
        if (e >= 0) {
            int32_t p = running[cur][e] + lane_rank;
            for (int w = 0; w < warp; ++w) {
                const int32_t v = wcnt[w][e];
                if ((v >> 16) == r) p += v & 0xffff;
            }
            perm[p] = static_cast<int32_t>(q);
            inv[q] = p;
        }
        for (int ee = tid; ee < E; ee += kPcThreads) {
            int32_t sum = 0;
            for (int w = 0; w < kPcWarps; ++w) {
                const int32_t v = wcnt[w][ee];
                if ((v >> 16) == r) sum += v & 0xffff;
            }
            running[cur ^ 1][ee] = running[cur][ee] + sum;
        }
        __syncthreads();
    }
    cluster_sync();          // no CTA leaves while another may still read its hist
}

// Largest plan the one-launch cluster path takes.
// (Beyond 8 rounds per CTA the three launches over many CTAs are faster.)
constexpr int64_t kPcMaxSlots = static_cast<int64_t>(kPcMaxCluster) * 8 * kPcThreads;

template <int ROUNDS>
static cudaError_t launch_permute_cluster_t(const moe_shape& s, int csize, int64_t chunk,
                                            const int32_t* idx, int32_t* counts, int32_t* offsets,
                                            int32_t* perm, int32_t* inv, int32_t* err_flag,
                                            cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(csize), 1, 1);
    cfg.blockDim = dim3(kPcThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(csize);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, permute_cluster_kernel<ROUNDS>, idx, s.T * s.k, s.E, chunk,
                              counts, offsets, perm, inv, err_flag);
}

static cudaError_t launch_permute_cluster(const moe_shape& s, const int32_t* idx, int32_t* counts,
                                          int32_t* offsets, int32_t* perm, int32_t* inv,
                                          int32_t* err_flag, cudaStream_t st) {
    const int64_t n = s.T * s.k;
    int64_t csize = (n + kPcThreads - 1) / kPcThreads;
    if (csize > kPcMaxCluster) csize = kPcMaxCluster;
    if (csize < 1) csize = 1;
    const int64_t chunk = (n + csize - 1) / csize;
    const int64_t rounds = (chunk + kPcThreads - 1) / kPcThreads;
    const int c = static_cast<int>(csize);
    if (rounds <= 1)
        return launch_permute_cluster_t<1>(s, c, chunk, idx, counts, offsets, perm, inv, err_flag, st);
    if (rounds <= 2)
        return launch_permute_cluster_t<2>(s, c, chunk, idx, counts, offsets, perm, inv, err_flag, st);
    if (rounds <= 4)
        return launch_permute_cluster_t<4>(s, c, chunk, idx, counts, offsets, perm, inv, err_flag, st);
    return launch_permute_cluster_t<8>(s, c, chunk, idx, counts, offsets, perm, inv, err_flag, st);
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
    if (n <= kPcMaxSlots)
        return launch_permute_cluster(s, idx, counts, offsets, perm, inv, err_flag, st);
    const int nblk = static_cast<int>((n + kPermSlotsPerBlock - 1) / kPermSlotsPerBlock);
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
// looked up with cudaGetSymbolAddress on the first call made while a device is
// current, and cached together with the id of the CUDA context it belongs to;
// a call that finds a different context current (the device was reset since)
// looks it up again.  Make the first call on a device before any stream
// capture.  The array keeps the last call's contents; the histogram kernel
// overwrites every entry it later reads, so nothing needs clearing.  All calls
// share the one array: calls whose kernels may overlap on the GPU (different
// streams without ordering between them) race on it.
#include <mutex>

namespace moe {
constexpr int64_t kNoallocScratchInts = 256 * 1024;
constexpr int kNoallocMaxDevices = 64;
}  // namespace moe

static __device__ __align__(256) int32_t g_permute_scratch[moe::kNoallocScratchInts];

namespace {

struct ScratchEntry {
    void* ptr;
    unsigned long long ctx_id;
};

std::mutex g_scratch_mu;
ScratchEntry g_scratch[moe::kNoallocMaxDevices] = {};

// Id of the current CUDA context (driver entry points cuCtxGetCurrent and
// cuCtxGetId); 0 when it cannot be determined, which disables the cache.
unsigned long long current_context_id() {
    typedef CUresult (*GetCurrentFn)(CUcontext*);
    typedef CUresult (*GetIdFn)(CUcontext, unsigned long long*);
    static GetCurrentFn get_current = nullptr;
    static GetIdFn get_id = nullptr;
    static bool looked_up = false;
    if (!looked_up) {
        void* a = nullptr;
        void* b = nullptr;
        cudaDriverEntryPointQueryResult qa, qb;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) ==
                cudaSuccess && qa == cudaDriverEntryPointSuccess &&
            cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) == cudaSuccess &&
            qb == cudaDriverEntryPointSuccess) {
            get_current = reinterpret_cast<GetCurrentFn>(a);
            get_id = reinterpret_cast<GetIdFn>(b);
        }
        looked_up = true;
    }
    if (!get_current || !get_id) return 0;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of g_permute_scratch in the current device's context.
cudaError_t noalloc_scratch(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= moe::kNoallocMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    // 0 before the runtime has made a context current: then look the address
    // up, which initialises the context, and read the id afterwards
    const unsigned long long ctx = current_context_id();
    ScratchEntry& entry = g_scratch[dev];
    if (!entry.ptr || ctx == 0 || entry.ctx_id != ctx) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_permute_scratch);
        if (e != cudaSuccess) return e;
        entry.ptr = p;
        entry.ctx_id = current_context_id();
    }
    *out = entry.ptr;
    return cudaSuccess;
}

}  // namespace

extern "C" moe_status moe_permute_noalloc(const moe_shape* shape, const int32_t* topk_idx,
                                          int32_t* counts, int32_t* offsets, int32_t* perm,
                                          int32_t* inv, int32_t* err_flag, void* stream) {
    // the same validation as moe_permute, then the scratch limit
    const moe_status st = moe::check_shape(shape);
    if (st != MOE_OK) return st;
    const moe_shape& s = *shape;
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
