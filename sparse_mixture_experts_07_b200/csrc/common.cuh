// Shared device helpers of the sm_100a MoE kernels: bf16 packing, the group
// table of the grouped GEMMs, and thin wrappers over the PTX of mbarriers,
// TMA, and the 5th-generation tensor cores (tcgen05) with tensor memory.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "../../include/moe.h"

namespace moe {

constexpr int kMaxExperts = 256;
constexpr int kMaxShared = 8;
constexpr int kMaxK = 16;
constexpr int kMaxGroups = kMaxExperts + kMaxShared;

// Host-side validation of a moe_shape, common to every entry point of the C
// ABI (defined in moe_api.cu): MOE_ERR_INVALID_ARG for inconsistent sizes,
// MOE_ERR_UNSUPPORTED for sizes outside what the kernels implement.
moe_status check_shape(const moe_shape* s);

// Workspace buffers of the backward pass (backward.cu); rows of the padded
// sorted order (P rows: each expert's rows padded to a multiple of 128).
struct BackwardBuffers {
    int32_t* poffsets;   // [E+1] padded expert offsets
    void* dO;            // [P, H] routed output gradients; later dX of the slots
    void* dgu;           // [P, 2I] gradients of the gate and up pre-activations
    void* dgu_sh;        // [S*T, 2Is] the same for the shared experts
    void* dX_sh;         // [S*T, H] the shared experts' input gradients
    float* dw_raw;       // [T*k, n-tiles] parts of the routing-weight gradients x weight
    float* dl;           // [T, E] logit gradients
    float* part;         // [chunks, E, H] router weight gradient partials
    float* partb;        // [chunks, E] router bias gradient partials
};

// Device-detected faults are OR-ed into the caller's err_flag as 1 << status.
__device__ __forceinline__ void raise_error(int32_t* err_flag, int status) {
    if (err_flag) atomicOr(err_flag, 1 << status);
}

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// Round-to-nearest-even pack of two floats into one bf16x2 word (lo first).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

template <typename T> struct ElemIO;
template <> struct ElemIO<float> {
    __device__ __forceinline__ static float load(const float* p, int64_t i) { return p[i]; }
    __device__ __forceinline__ static void store(float* p, int64_t i, float v) { p[i] = v; }
};
template <> struct ElemIO<__nv_bfloat16> {
    __device__ __forceinline__ static float load(const __nv_bfloat16* p, int64_t i) {
        return __bfloat162float(p[i]);
    }
    __device__ __forceinline__ static void store(__nv_bfloat16* p, int64_t i, float v) {
        p[i] = __float2bfloat16_rn(v);
    }
};

// ---------------------------------------------------------------------------
// Group table of a grouped GEMM launch.  Group g < E is routed expert g whose
// rows are [offsets[g], offsets[g+1]) of the sorted slot space; group E + s is
// shared expert s whose rows are the T tokens.  The table is rebuilt by every
// CTA from the device offsets, so the host never reads the expert counts.
template <int MAXG>
struct GroupTableT {
    int32_t n_groups;
    int32_t total_tiles;
    int32_t tile_start[MAXG + 1];   // prefix over groups of tiles
    int32_t rows[MAXG];             // M of each group
    int32_t row0[MAXG];             // first row of the group in its A space
};

// All threads of the CTA copy offsets[0..E] into shared memory (one parallel
// load instead of E dependent ones in the thread that builds a table); the
// caller synchronises before the copy is read.
__device__ __forceinline__ void stage_offsets(int32_t* dst, const int32_t* offsets, int E) {
    for (int g = static_cast<int>(threadIdx.x); g <= E; g += static_cast<int>(blockDim.x))
        dst[g] = offsets[g];
}
using GroupTable = GroupTableT<kMaxGroups>;

// ---------------------------------------------------------------------------
// PTX wrappers (sm_100a).
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Programmatic dependent launch (the decode chain: router, plan, decode
// expert kernels, combine).  A kernel launched by launch_pdl may begin while
// the kernel before it in the stream is still running.  It calls
// pdl_launch_dependents() on entry, so that the kernel after it may be
// scheduled early in turn, and pdl_wait() before it first touches memory
// that an earlier kernel writes or reads: pdl_wait returns once the previous
// kernel has completed and its writes are visible, and since that kernel
// waited the same way, every earlier one has too.  A kernel launched the
// ordinary way finds both instructions without effect.
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args&&... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// try_wait with a suspend-time hint: a thread whose phase is not complete is
// suspended (it issues nothing) until the phase completes or about hint_ns
// nanoseconds pass.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity,
                                                    uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Bounded wait: until the phase with `parity` completes, or until
// `deadline_ns` (globaltimer) passes; returns false on timeout.  Waiting
// threads are suspended between checks (at most about 20 us each), so warps
// that wait do not take issue slots from the warps that work.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t deadline_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    while (!mbar_try_wait_sleep(bar, parity, 20000u)) {
        if (global_ns() > deadline_ns) return false;
    }
    return true;
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 2D tiled TMA load of a box at coordinates (c0 = inner/column, c1 = row).
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
        : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// --- tensor memory -----------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
                 "r"(ncols));
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols));
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

// Arrive on an mbarrier once all previously issued tcgen05.mma of this thread
// have completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t* r = reinterpret_cast<uint32_t*>(v);
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// --- CTA pairs (cluster of 2) -------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t n_clusters_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
// Arrive on an mbarrier given by its shared::cluster address (any CTA of the cluster).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
                 : "memory");
}
// Cluster-wide barrier (all threads of all CTAs); the non-.aligned form, so
// threads of a warp may arrive from different branches.
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
// 2D tiled TMA load into this CTA's shared memory whose completion is counted
// on an mbarrier that may live in the peer CTA of the pair (cta_group::2).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map,
                                                 uint32_t bar_cluster_addr, int32_t c0, int32_t c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster_addr), "r"(c0), "r"(c1)
        : "memory");
}
// Same, with an L2 eviction-priority policy for the loaded lines.
__device__ __forceinline__ void tma_load_2d_pair_hint(void* dst, const CUtensorMap* map,
                                                      uint32_t bar_cluster_addr, int32_t c0,
                                                      int32_t c1, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster_addr), "r"(c0), "r"(c1),
        "l"(policy)
        : "memory");
}
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_normal() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
                 "r"(ncols));
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::);
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols));
}
// D (+)= A * B^T across the CTA pair: A rows [0, M/2) and B rows [0, N/2) come
// from the issuing CTA's shared memory, the other halves from the peer CTA at
// the same offsets; D rows [0, M/2) land in the issuing CTA's tensor memory,
// rows [M/2, M) in the peer's.
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}
// Arrive on the mbarrier at this shared-memory offset in every CTA of
// `cta_mask` once the pair MMAs issued so far have completed.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar, uint16_t cta_mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;" ::"r"(smem_u32(bar)),
        "h"(cta_mask)
        : "memory");
}

// Shared-memory matrix descriptor of a K-major operand tile stored with the
// 128-byte swizzle: rows of 64 bf16 (128 B), 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);   // start address
    d |= static_cast<uint64_t>(1) << 16;                    // leading byte offset (unused)
    d |= static_cast<uint64_t>(1024 >> 4) << 32;            // stride byte offset
    d |= static_cast<uint64_t>(1) << 46;                    // descriptor version (sm_100)
    d |= static_cast<uint64_t>(2) << 61;                    // swizzle: 128 B
    return d;
}

// Instruction descriptor, kind::f16: bf16 A and B (K-major), fp32 D, M x N.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}

}  // namespace moe

namespace moe {

// Builds the group table (one thread; at most kMaxGroups iterations).
// Routed group g covers rows [offsets[g], offsets[g+1]); shared group E+s
// covers the T token rows.  Tiles of a group: ceil(rows / BM) * n_tiles.
// Built by one thread.  stage_offsets has put the routed experts' offsets in
// gt.tile_start[0..E]; entry g is read (as offsets[g] and offsets[g+1]) before
// the loop overwrites it with the tile prefix.
template <int MAXG>
__device__ __forceinline__ void build_group_table(GroupTableT<MAXG>& gt, int E, int S, int64_t T,
                                                  int BM, int n_tiles_routed, int n_tiles_shared) {
    int32_t* offsets = gt.tile_start;
    int32_t acc = 0;
    gt.n_groups = E + S;
    for (int g = 0; g < E + S; ++g) {
        int32_t rows, row0, nt;
        if (g < E) {
            row0 = offsets[g];
            rows = offsets[g + 1] - row0;
            nt = n_tiles_routed;
        } else {
            row0 = static_cast<int32_t>((g - E) * T);
            rows = static_cast<int32_t>(T);
            nt = n_tiles_shared;
        }
        if (rows < 0) rows = 0;
        gt.rows[g] = rows;
        gt.row0[g] = row0;
        gt.tile_start[g] = acc;
        acc += ((rows + BM - 1) / BM) * nt;
    }
    gt.tile_start[E + S] = acc;
    gt.total_tiles = acc;
}

// Group of a linear tile index (binary search over the prefix).
template <int MAXG>
__device__ __forceinline__ int find_group(const GroupTableT<MAXG>& gt, int32_t tile) {
    int lo = 0, hi = gt.n_groups - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (gt.tile_start[mid] <= tile) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

}  // namespace moe
