// The C ABI of include/moe.h: host-side validation, workspace layout and
// dispatch to the kernels.  No memory is allocated here.
#include <cstring>

#include "common.cuh"

namespace moe {
cudaError_t launch_route(const moe_shape&, const void*, const float*, const float*, float*,
                         int32_t*, float*, cudaStream_t);
cudaError_t launch_route_tc(const moe_shape&, const void*, const float*, const float*, float*,
                            int32_t*, float*, int32_t*, cudaStream_t);
int router_split_rows(const moe_shape&);
cudaError_t launch_router_split(const moe_shape&, const float*, void*, int, cudaStream_t);
cudaError_t launch_route_tc_split(const moe_shape&, const void*, const void*, const float*, float*,
                                  int32_t*, float*, int32_t*, int, cudaStream_t);
cudaError_t launch_route_small(const moe_shape&, const void*, const float*, const float*, float*,
                               int32_t*, float*, cudaStream_t);
cudaError_t launch_route_cluster(const moe_shape&, const void*, const float*, const float*, float*,
                                 int32_t*, float*, int32_t*, int32_t*, int32_t*, int32_t*,
                                 cudaStream_t);
constexpr int64_t kRoutePlanTokens = 16;   // tokens of one cluster block (route.cu)
size_t permute_workspace_bytes(const moe_shape&);
cudaError_t launch_permute(const moe_shape&, const int32_t*, int32_t*, int32_t*, int32_t*,
                           int32_t*, int32_t*, void*, cudaStream_t);
cudaError_t launch_ffn_simt(const moe_shape&, const void*, const int32_t*, const int32_t*,
                            const float*, const void*, const void*, const void*, const void*,
                            void*, void*, void*, cudaStream_t);
cudaError_t launch_ffn_sm100(const moe_shape&, const void*, const void*, const int32_t*,
                             const int32_t*, const float*, const void*, const void*, const void*,
                             const void*, void*, void*, void*, int32_t*, int, int, cudaStream_t,
                             void*, void*);
cudaError_t launch_ffn_decode(const moe_shape&, const void*, const int32_t*, const int32_t*,
                              const float*, const void*, const void*, const void*, const void*,
                              void*, void*, void*, int, cudaStream_t);
cudaError_t launch_ffn_sm100_pair(const moe_shape&, const void*, const void*, const int32_t*,
                                  const int32_t*, const float*, const void*, const void*,
                                  const void*, const void*, void*, void*, void*, int32_t*, int, int,
                                  cudaStream_t, void*, void*);
cudaError_t launch_ffn_decode_mxfp4(const moe_shape&, const void*, const int32_t*,
                                    const int32_t*, const float*, const uint8_t*, const uint8_t*,
                                    const uint8_t*, const uint8_t*, void*, void*, int32_t*, void*,
                                    int32_t*, void*, int32_t*, int, cudaStream_t);
cudaError_t launch_combine(const moe_shape&, const void*, const int32_t*, void*, cudaStream_t);
int mx_padded_cols(int K);
bool mx_tc_supported(const moe_shape&, const void*, const void*, bool);
int64_t mx_tc_prepared_bytes(const moe_shape&);
cudaError_t launch_mx_tc_prepare(const moe_shape&, const uint8_t*, const uint8_t*, const uint8_t*,
                                 const uint8_t*, void*, int, cudaStream_t);
int64_t mx_tc_plane_rows(int64_t slots);
int mx_tc_sf_rows(int64_t SP);
int64_t mx_tc_part_floats(int64_t slots, int H, int I);
cudaError_t launch_ffn_decode_mxfp4_tc(const moe_shape&, const void*, const int32_t*,
                                       const int32_t*, const float*, const uint8_t*,
                                       const uint8_t*, const uint8_t*, const uint8_t*,
                                       const void*, uint8_t*, uint8_t*, uint8_t*, uint8_t*,
                                       float*, int32_t*, void*, int32_t*, int, cudaStream_t);
cudaError_t launch_combine_experts(const moe_shape&, int, int, int, const void*, const int32_t*,
                                   const int32_t*, float*, int, cudaStream_t);
cudaError_t launch_cast_f32(const moe_shape&, const float*, void*, int, cudaStream_t);
cudaError_t launch_route_noaux(const moe_shape&, int, int, const float*, const float*, int32_t*,
                               float*, cudaStream_t);
size_t backward_pad_rows(const moe_shape&);
int backward_dw_tiles(const moe_shape&);
int router_wgrad_chunks(const moe_shape&);
cudaError_t launch_backward(const moe_shape&, const void*, const float*, const int32_t*,
                            const float*, const int32_t*, const int32_t*, const int32_t*,
                            const int32_t*, const void*, const void*, const void*, const void*,
                            const void*, const void*, const void*, const void*, const void*,
                            const float*, float, const void*, void*, float*, float*, float*,
                            float*, float*, float*, float*, float*, const BackwardBuffers&,
                            int32_t*, int, cudaStream_t);
cudaError_t launch_gather_rows(const moe_shape&, const void*, const int32_t*, void*, int,
                               cudaStream_t);
cudaError_t launch_gather_by_token(const moe_shape&, const void*, const int32_t*, int32_t*, void*,
                                   int, cudaStream_t);

// Host-side validation shared by every entry point (declared in common.cuh).
moe_status check_shape(const moe_shape* s) {
    if (!s) return MOE_ERR_INVALID_ARG;
    if (s->T < 0 || s->H <= 0 || s->I <= 0 || s->E <= 0 || s->k <= 0 || s->k > s->E ||
        s->n_shared < 0 || (s->n_shared > 0 && s->I_shared <= 0) ||
        (s->dtype != MOE_F32 && s->dtype != MOE_BF16))
        return MOE_ERR_INVALID_ARG;
    if (s->E > moe::kMaxExperts || s->k > moe::kMaxK || s->n_shared > moe::kMaxShared)
        return MOE_ERR_UNSUPPORTED;
    const int64_t rows = s->T * (s->k + s->n_shared);
    if (s->T > (int64_t(1) << 31) || rows >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
    if (s->dtype == MOE_BF16) {
        if (s->H % 8 || s->I % 8 || (s->n_shared > 0 && s->I_shared % 8))
            return MOE_ERR_UNSUPPORTED;
    }
    return MOE_OK;
}

}  // namespace moe

namespace {

using moe::check_shape;

constexpr size_t kAlign = 256;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

size_t elem_bytes(const moe_shape& s) { return s.dtype == MOE_BF16 ? 2 : 4; }

int num_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    static int cached[64] = {0};
    if (dev >= 0 && dev < 64 && cached[dev] > 0) return cached[dev];
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        n = 148;
    if (dev >= 0 && dev < 64) cached[dev] = n;
    return n;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

struct Workspace {
    size_t permute_off, h_routed_off, h_shared_off, x_perm_off, inv_off;
    size_t mx_x16_off, mx_xexp_off, mx_h16_off, mx_hexp_off;   // MXFP4 decode (T <= 64)
    size_t mx_xq_off, mx_xsf_off, mx_hq_off, mx_hsf_off, mx_part_off, mx_ctl_off;
    size_t total;
};

Workspace layout(const moe_shape& s) {
    Workspace w{};
    const size_t eb = elem_bytes(s);
    const int64_t Tk = s.T * s.k;
    size_t off = 0;
    w.permute_off = off;
    off += align_up(moe::permute_workspace_bytes(s));
    w.h_routed_off = off;
    off += align_up(static_cast<size_t>(Tk) * s.I * eb);
    w.h_shared_off = off;
    off += align_up(static_cast<size_t>(s.n_shared) * s.T * (s.n_shared ? s.I_shared : 0) * eb);
    w.x_perm_off = off;
    if (s.dtype == MOE_BF16) off += align_up(static_cast<size_t>(Tk) * s.H * 2);
    w.inv_off = off;               // sorted position of each slot (token-major gather)
    off += align_up(static_cast<size_t>(Tk) * 4);
    if (s.dtype == MOE_BF16 && s.T <= 64) {
        // f16 copies of x and h for moe_forward_mxfp4, rows padded with zeros
        w.mx_x16_off = off;
        off += align_up(static_cast<size_t>(s.T) * moe::mx_padded_cols(s.H) * 2);
        w.mx_xexp_off = off;
        off += align_up(static_cast<size_t>(s.T) * 4);
        w.mx_h16_off = off;
        off += align_up(static_cast<size_t>(Tk) * moe::mx_padded_cols(s.I) * 2);
        w.mx_hexp_off = off;
        off += align_up(static_cast<size_t>(Tk) * 4);
        if (s.H % 64 == 0 && s.I % 64 == 0) {
            // block-scaled tensor-core path: E4M3 hi/lo planes of x and h with
            // their exponents (per 128-column K-group a block of
            // mx_tc_sf_rows 16-byte rows), the split partials, and the split
            // count
            const size_t SP = static_cast<size_t>(moe::mx_tc_plane_rows(Tk));
            const size_t sf_block = static_cast<size_t>(moe::mx_tc_sf_rows(SP)) * 16;
            w.mx_xq_off = off;
            off += align_up(2 * SP * s.H);
            w.mx_xsf_off = off;
            off += align_up((s.H + 127) / 128 * sf_block);
            w.mx_hq_off = off;
            off += align_up(2 * SP * s.I);
            w.mx_hsf_off = off;
            off += align_up((s.I + 127) / 128 * sf_block);
            w.mx_part_off = off;
            off += align_up(static_cast<size_t>(moe::mx_tc_part_floats(Tk, s.H, s.I)) * 4);
            w.mx_ctl_off = off;
            off += align_up(16);
        }
    }
    w.total = off;
    return w;
}

}  // namespace

extern "C" {

const char* moe_status_str(moe_status status) {
    switch (status) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
        case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
        case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
        case MOE_ERR_BAD_INDEX: return "MOE_ERR_BAD_INDEX";
        case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
    }
    return "MOE_ERR_UNKNOWN";
}

moe_status moe_workspace_size(const moe_shape* shape, size_t* bytes) {
    moe_status st = check_shape(shape);
    if (st != MOE_OK) return st;
    if (!bytes) return MOE_ERR_INVALID_ARG;
    *bytes = layout(*shape).total;
    return MOE_OK;
}

moe_status moe_route(const moe_shape* shape, const void* x, const float* w_router,
                     const float* router_bias, float* logits, int32_t* topk_idx, float* topk_w,
                     int32_t* err_flag, void* stream) {
    moe_status st = check_shape(shape);
    if (st != MOE_OK) return st;
    if (shape->T == 0) return MOE_OK;
    if (!x || !w_router || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    // few tokens: a cluster per 16 tokens splitting the hidden dimension (one
    // CTA per token where its shared memory does not fit); many tokens, bf16:
    // tensor cores; else CUDA cores
    if (shape->T <= 256 && shape->H <= 32768 && aligned16(w_router)) {
        const cudaError_t e = moe::launch_route_cluster(*shape, x, w_router, router_bias, logits,
                                                        topk_idx, topk_w, nullptr, nullptr,
                                                        nullptr, nullptr, cs);
        if (e != cudaErrorNotSupported) return cuda_status(e);
        return cuda_status(moe::launch_route_small(*shape, x, w_router, router_bias, logits,
                                                   topk_idx, topk_w, cs));
    }
    if (shape->dtype == MOE_BF16 && shape->E <= 64 && aligned16(x) && aligned16(w_router))
        return cuda_status(moe::launch_route_tc(*shape, x, w_router, router_bias, logits,
                                                topk_idx, topk_w, err_flag, cs));
    return cuda_status(moe::launch_route(*shape, x, w_router, router_bias, logits, topk_idx,
                                         topk_w, cs));
}

moe_status moe_router_split_size(const moe_shape* shape, size_t* bytes) {
    moe_status st = check_shape(shape);
    if (st != MOE_OK) return st;
    if (!bytes) return MOE_ERR_INVALID_ARG;
    *bytes = static_cast<size_t>(moe::router_split_rows(*shape)) * shape->H * 2;
    return MOE_OK;
}

moe_status moe_router_split(const moe_shape* shape, const float* w_router, void* w_split,
                            size_t w_split_bytes, void* stream) {
    moe_status st = check_shape(shape);
    if (st != MOE_OK) return st;
    const size_t need = static_cast<size_t>(moe::router_split_rows(*shape)) * shape->H * 2;
    if (need == 0) return MOE_ERR_UNSUPPORTED;
    if (!w_router || !w_split) return MOE_ERR_INVALID_ARG;
    if (w_split_bytes < need) return MOE_ERR_WORKSPACE;
    if (!aligned16(w_router) || !aligned16(w_split)) return MOE_ERR_UNSUPPORTED;
    return cuda_status(moe::launch_router_split(*shape, w_router, w_split, num_sms(),
                                                static_cast<cudaStream_t>(stream)));
}

moe_status moe_route_split(const moe_shape* shape, const void* x, const float* w_router,
                           const void* w_split, const float* router_bias, float* logits,
                           int32_t* topk_idx, float* topk_w, int32_t* err_flag, void* stream) {
    moe_status st = check_shape(shape);
    if (st != MOE_OK) return st;
    if (shape->T == 0) return MOE_OK;
    if (!x || !w_router || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
    // the split weight serves the tensor-core path; everything else is moe_route
    const bool tc = shape->T > 256 && moe::router_split_rows(*shape) > 0;
    if (!tc || !w_split)
        return moe_route(shape, x, w_router, router_bias, logits, topk_idx, topk_w, err_flag,
                         stream);
    if (!aligned16(x) || !aligned16(w_split)) return MOE_ERR_UNSUPPORTED;
    return cuda_status(moe::launch_route_tc_split(*shape, x, w_split, router_bias, logits,
                                                  topk_idx, topk_w, err_flag, num_sms(),
                                                  static_cast<cudaStream_t>(stream)));
}

moe_status moe_route_noaux_tc(const moe_shape* shape, int32_t n_group, int32_t topk_group,
                              const void* x, const float* w_router, const void* w_split,
                              const float* score_bias, float* logits, int32_t* topk_idx,
                              float* topk_w, int32_t* err_flag, void* stream) {
    moe_status st = check_shape(shape);
    if (st != MOE_OK) return st;
    const moe_shape& s = *shape;
    if (n_group < 1 || n_group > 32 || s.E % n_group != 0 || topk_group < 1 ||
        topk_group > n_group || s.k > topk_group * (s.E / n_group))
        return MOE_ERR_INVALID_ARG;
    if (s.T == 0) return MOE_OK;
    if (!logits) return MOE_ERR_INVALID_ARG;
    // bias-free logits (the softmax selection this also writes is replaced below)
    st = moe_route_split(shape, x, w_router, w_split, nullptr, logits, topk_idx, topk_w,
                         err_flag, stream);
    if (st != MOE_OK) return st;
    return cuda_status(moe::launch_route_noaux(s, n_group, topk_group, logits, score_bias,
                                               topk_idx, topk_w,
                                               static_cast<cudaStream_t>(stream)));
}

moe_status moe_permute(const moe_shape* shape, const int32_t* topk_idx, int32_t* counts,
                       int32_t* offsets, int32_t* perm, int32_t* inv, int32_t* err_flag,
                       void* workspace, size_t workspace_bytes, void* stream) {
    moe_status st = check_shape(shape);
    if (st != MOE_OK) return st;
    if (!counts || !offsets) return MOE_ERR_INVALID_ARG;
    if (shape->T > 0 && (!topk_idx || !perm || !inv)) return MOE_ERR_INVALID_ARG;
    const Workspace w = layout(*shape);
    if (w.total > 0 && (!workspace || workspace_bytes < w.total)) return MOE_ERR_WORKSPACE;
    void* blk = static_cast<char*>(workspace) + w.permute_off;
    return cuda_status(moe::launch_permute(*shape, topk_idx, counts, offsets, perm, inv, err_flag,
                                           blk, static_cast<cudaStream_t>(stream)));
}

moe_status moe_route_permute(const moe_shape* shape, const void* x, const float* w_router,
                             const void* w_split, const float* router_bias, float* logits,
                             int32_t* topk_idx, float* topk_w, int32_t* counts, int32_t* offsets,
                             int32_t* perm, int32_t* inv, int32_t* err_flag, void* workspace,
                             size_t workspace_bytes, void* stream) {
    moe_status st = check_shape(shape);
    if (st != MOE_OK) return st;
    if (!counts || !offsets) return MOE_ERR_INVALID_ARG;
    if (shape->T > 0 && (!x || !w_router || !topk_idx || !topk_w || !perm || !inv))
        return MOE_ERR_INVALID_ARG;
    const Workspace w = layout(*shape);
    if (w.total > 0 && (!workspace || workspace_bytes < w.total)) return MOE_ERR_WORKSPACE;
    // one token block: the cluster router writes the plan too
    if (shape->T > 0 && shape->T <= moe::kRoutePlanTokens && shape->H <= 32768 &&
        aligned16(w_router)) {
        const cudaError_t e = moe::launch_route_cluster(*shape, x, w_router, router_bias, logits,
                                                        topk_idx, topk_w, counts, offsets, perm,
                                                        inv, static_cast<cudaStream_t>(stream));
        if (e != cudaErrorNotSupported) return cuda_status(e);
    }
    st = moe_route_split(shape, x, w_router, w_split, router_bias, logits, topk_idx, topk_w,
                         err_flag, stream);
    if (st != MOE_OK) return st;
    return moe_permute(shape, topk_idx, counts, offsets, perm, inv, err_flag, workspace,
                       workspace_bytes, stream);
}

}  // extern "C"

namespace {

// The expert FFNs of routed experts [e_begin, e_end) (weights of those experts
// only: gate_up[e - e_begin], down[e - e_begin]) and, when with_shared, of the
// shared experts.  moe_forward is the whole range with the shared experts;
// moe_forward_experts is one expert-parallel rank's share.  The launches see
// a shape whose E is the range's width and whose offsets start at e_begin, so
// their group tables hold only the range's experts, with the rows of the
// global sorted order.
// Where the training forward keeps what the backward pass reads: the gate and
// up pre-activations, the SwiGLU outputs and the gathered x rows.
struct TrainState {
    void* gu;        // [T*k, 2I]
    void* gu_sh;     // [S*T, 2Is]
    void* h;         // [T*k, I]
    void* h_sh;      // [S*T, Is]
    void* x_perm;    // [T*k, H]
    size_t total;
};

TrainState train_state_layout(const moe_shape& s, void* base) {
    TrainState t{};
    char* b = static_cast<char*>(base);
    const size_t Tk = static_cast<size_t>(s.T * s.k);
    const size_t ST = static_cast<size_t>(s.n_shared) * static_cast<size_t>(s.T);
    const size_t Is = s.n_shared > 0 ? static_cast<size_t>(s.I_shared) : 0;
    size_t off = 0;
    t.gu = b + off;
    off += align_up(Tk * 2 * s.I * 2);
    t.gu_sh = b + off;
    off += align_up(ST * 2 * Is * 2);
    t.h = b + off;
    off += align_up(Tk * s.I * 2);
    t.h_sh = b + off;
    off += align_up(ST * Is * 2);
    t.x_perm = b + off;
    off += align_up(Tk * s.H * 2);
    t.total = off;
    return t;
}

moe_status forward_range(const moe_shape& s, int e_begin, int e_end, bool with_shared,
                         const void* x, const int32_t* offsets, const int32_t* perm,
                         const float* topk_w, const void* gate_up, const void* down,
                         const void* sh_gate_up, const void* sh_down, void* y_slots,
                         int32_t* err_flag, void* workspace, size_t workspace_bytes,
                         cudaStream_t cs, const TrainState* train = nullptr) {
    if (s.T == 0) return MOE_OK;
    const bool any_routed = e_end > e_begin;
    const bool shared = with_shared && s.n_shared > 0;
    if (!x || !offsets || !perm || !topk_w || !y_slots) return MOE_ERR_INVALID_ARG;
    if (any_routed && (!gate_up || !down)) return MOE_ERR_INVALID_ARG;
    if (shared && (!sh_gate_up || !sh_down)) return MOE_ERR_INVALID_ARG;
    const Workspace w = layout(s);
    if (!workspace || workspace_bytes < w.total) return MOE_ERR_WORKSPACE;
    if (!any_routed && !shared) return MOE_OK;
    moe_shape sl = s;
    sl.E = e_end - e_begin;
    sl.n_shared = shared ? s.n_shared : 0;
    if (!shared) sl.I_shared = 0;
    const int32_t* offs = offsets + e_begin;
    char* ws = static_cast<char*>(workspace);
    void* h_routed = train ? train->h : ws + w.h_routed_off;
    void* h_shared = train ? train->h_sh : ws + w.h_shared_off;
    void* gu_routed = train ? train->gu : nullptr;
    void* gu_shared = train && shared ? train->gu_sh : nullptr;
    if (s.dtype == MOE_F32) {
        return cuda_status(moe::launch_ffn_simt(sl, x, offs, perm, topk_w, gate_up, down,
                                                sh_gate_up, sh_down, h_routed, h_shared, y_slots,
                                                cs));
    }
    const void* ptrs[] = {x, y_slots, workspace};
    for (const void* p : ptrs)
        if (!aligned16(p)) return MOE_ERR_UNSUPPORTED;
    if (any_routed && (!aligned16(gate_up) || !aligned16(down))) return MOE_ERR_UNSUPPORTED;
    if (shared && (!aligned16(sh_gate_up) || !aligned16(sh_down))) return MOE_ERR_UNSUPPORTED;
    const int sms = num_sms();
    // decode batches (<= 8 rows per expert): stream the active experts' weights
    if (s.T <= 8)
        return cuda_status(moe::launch_ffn_decode(sl, x, offs, perm, topk_w, gate_up, down,
                                                  sh_gate_up, sh_down, h_routed, h_shared,
                                                  y_slots, sms, cs));
    void* x_perm = train ? train->x_perm : ws + w.x_perm_off;
    // x rows in sorted slot order for GEMM 1.  When x is too large to stay in
    // L2 between its k copies, gather token-major (each row of x read once,
    // written k times; measured 1.3-2.7 % faster per step on the 67-134 MB
    // batches); otherwise slot-major, which needs no inverse permutation.
    const bool by_token = static_cast<int64_t>(s.T) * s.H * 2 > (int64_t(48) << 20);
    if (any_routed) {
        cudaError_t e = by_token
                            ? moe::launch_gather_by_token(s, x, perm,
                                                          reinterpret_cast<int32_t*>(ws + w.inv_off),
                                                          x_perm, sms, cs)
                            : moe::launch_gather_rows(s, x, perm, x_perm, sms, cs);
        if (e != cudaSuccess) return MOE_ERR_CUDA;
    }
    // CTA pairs (256-row tiles) when the experts average at least 256 rows;
    // one CTA per tile otherwise (less padding on small groups).  The average
    // is over all E experts, a range's share of the rows being proportional.
    constexpr int kPairMinRows = 256;   // average rows per expert for CTA pairs
    constexpr int kPairGroupM = 16;     // m-tiles per rasterisation band
    if (s.T * s.k >= static_cast<int64_t>(kPairMinRows) * s.E)
        return cuda_status(moe::launch_ffn_sm100_pair(sl, x, x_perm, offs, perm, topk_w, gate_up,
                                                      down, sh_gate_up, sh_down, h_routed,
                                                      h_shared, y_slots, err_flag, sms,
                                                      kPairGroupM, cs, gu_routed, gu_shared));
    return cuda_status(moe::launch_ffn_sm100(sl, x, x_perm, offs, perm, topk_w, gate_up, down,
                                             sh_gate_up, sh_down, h_routed, h_shared, y_slots,
                                             err_flag, sms, 8, cs, gu_routed, gu_shared));
}

// Workspace of moe_backward, in 256-byte aligned regions.
struct BwdLayout {
    size_t poff, dO, dgu, dgu_sh, dX_sh, dw_raw, dl, part, partb, total;
};

BwdLayout bwd_layout(const moe_shape& s) {
    BwdLayout b{};
    const size_t P = moe::backward_pad_rows(s);
    const size_t ST = static_cast<size_t>(s.n_shared) * static_cast<size_t>(s.T);
    const size_t Is = s.n_shared > 0 ? static_cast<size_t>(s.I_shared) : 0;
    const size_t chunks = static_cast<size_t>(moe::router_wgrad_chunks(s));
    size_t off = 0;
    b.poff = off;
    off += align_up(static_cast<size_t>(s.E + 1) * 4);
    b.dO = off;
    off += align_up(P * s.H * 2);
    b.dgu = off;
    off += align_up(P * 2 * s.I * 2);
    b.dgu_sh = off;
    off += align_up(ST * 2 * Is * 2);
    b.dX_sh = off;
    off += align_up(ST * s.H * 2);
    b.dw_raw = off;
    off += align_up(static_cast<size_t>(s.T * s.k) * moe::backward_dw_tiles(s) * 4);
    b.dl = off;
    off += align_up(static_cast<size_t>(s.T) * s.E * 4);
    b.part = off;
    off += align_up(chunks * s.E * s.H * 4);
    b.partb = off;
    off += align_up(chunks * s.E * 4);
    b.total = off;
    return b;
}

// Shapes the training path (tensor-core GEMMs, bf16) supports.
moe_status check_train_shape(const moe_shape& s) {
    if (s.dtype != MOE_BF16 || s.T <= 8) return MOE_ERR_UNSUPPORTED;
    if (s.H % 64 || s.I % 32 || (s.n_shared > 0 && s.I_shared % 32)) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

}  // namespace

extern "C" {

moe_status moe_forward(const moe_shape* shape, const void* x, const int32_t* offsets,
                       const int32_t* perm, const float* topk_w, const void* gate_up,
                       const void* down, const void* sh_gate_up, const void* sh_down,
                       void* y_slots, int32_t* err_flag, void* workspace,
                       size_t workspace_bytes, void* stream) {
    moe_status st = check_shape(shape);
    if (st != MOE_OK) return st;
    const moe_shape& s = *shape;
    if (s.T == 0) return MOE_OK;
    if (!gate_up || !down) return MOE_ERR_INVALID_ARG;
    if (s.n_shared > 0 && (!sh_gate_up || !sh_down)) return MOE_ERR_INVALID_ARG;
    return forward_range(s, 0, s.E, true, x, offsets, perm, topk_w, gate_up, down, sh_gate_up,
                         sh_down, y_slots, err_flag, workspace, workspace_bytes,
                         static_cast<cudaStream_t>(stream));
}

moe_status moe_shared_merge(const moe_shape* shape, const void* sh_gate_up, const void* sh_down,
                            void* gate_up_merged, void* down_merged, void* stream) {
    moe_status st = check_shape(shape);
    if (st != MOE_OK) return st;
    const moe_shape& s = *shape;
    if (s.n_shared == 0 || !sh_gate_up || !sh_down || !gate_up_merged || !down_merged)
        return MOE_ERR_INVALID_ARG;
    const size_t eb = elem_bytes(s);
    const size_t S = static_cast<size_t>(s.n_shared), Is = static_cast<size_t>(s.I_shared);
    const size_t H = static_cast<size_t>(s.H);
    const size_t block = Is * H * eb;   // one expert's gate (or up) rows
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const auto* src_gu = static_cast<const uint8_t*>(sh_gate_up);
    auto* dst_gu = static_cast<uint8_t*>(gate_up_merged);
    for (size_t e = 0; e < S; ++e) {
        // gate rows of expert e, then its up rows, each one contiguous block
        if (cudaMemcpyAsync(dst_gu + e * block, src_gu + 2 * e * block, block,
                            cudaMemcpyDeviceToDevice, cs) != cudaSuccess ||
            cudaMemcpyAsync(dst_gu + (S + e) * block, src_gu + (2 * e + 1) * block, block,
                            cudaMemcpyDeviceToDevice, cs) != cudaSuccess)
            return MOE_ERR_CUDA;
        // expert e's [H, Is] down matrix into columns [e Is, (e+1) Is) of [H, S Is]
        if (cudaMemcpy2DAsync(static_cast<uint8_t*>(down_merged) + e * Is * eb, S * Is * eb,
                              static_cast<const uint8_t*>(sh_down) + e * block, Is * eb,
                              Is * eb, H, cudaMemcpyDeviceToDevice, cs) != cudaSuccess)
            return MOE_ERR_CUDA;
    }
    return MOE_OK;
}

moe_status moe_forward_experts(const moe_shape* shape, int32_t e_begin, int32_t e_end,
                               const void* x, const int32_t* offsets, const int32_t* perm,
                               const float* topk_w, const void* gate_up_local,
                               const void* down_local, const void* sh_gate_up,
                               const void* sh_down, void* y_slots, int32_t* err_flag,
                               void* workspace, size_t workspace_bytes, void* stream) {
    moe_status st = check_shape(shape);
    if (st != MOE_OK) return st;
    const moe_shape& s = *shape;
    if (e_begin < 0 || e_end < e_begin || e_end > s.E) return MOE_ERR_INVALID_ARG;
    if ((sh_gate_up == nullptr) != (sh_down == nullptr)) return MOE_ERR_INVALID_ARG;
    return forward_range(s, e_begin, e_end, sh_gate_up != nullptr, x, offsets, perm, topk_w,
                         gate_up_local, down_local, sh_gate_up, sh_down, y_slots, err_flag,
                         workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

moe_status moe_combine_experts(const moe_shape* shape, int32_t e_begin, int32_t e_end,
                               int32_t with_shared, const void* y_slots, const int32_t* inv,
                               const int32_t* topk_idx, float* y_partial, void* stream) {
    moe_status st = check_shape(shape);
    if (st != MOE_OK) return st;
    const moe_shape& s = *shape;
    if (e_begin < 0 || e_end < e_begin || e_end > s.E) return MOE_ERR_INVALID_ARG;
    if (s.T == 0) return MOE_OK;
    if (!y_slots || !inv || !topk_idx || !y_partial) return MOE_ERR_INVALID_ARG;
    if (s.dtype == MOE_BF16 && (!aligned16(y_slots) || !aligned16(y_partial)))
        return MOE_ERR_UNSUPPORTED;
    return cuda_status(moe::launch_combine_experts(s, e_begin, e_end, with_shared != 0, y_slots,
                                                   inv, topk_idx, y_partial, num_sms(),
                                                   static_cast<cudaStream_t>(stream)));
}

moe_status moe_cast_f32(const moe_shape* shape, const float* y32, void* y, void* stream) {
    moe_status st = check_shape(shape);
    if (st != MOE_OK) return st;
    const moe_shape& s = *shape;
    if (s.T == 0) return MOE_OK;
    if (!y32 || !y) return MOE_ERR_INVALID_ARG;
    const bool vec = (s.T * static_cast<int64_t>(s.H)) % 4 == 0;
    if (s.dtype == MOE_BF16 && vec &&
        (!aligned16(y32) || (reinterpret_cast<uintptr_t>(y) & 7u)))
        return MOE_ERR_UNSUPPORTED;
    return cuda_status(moe::launch_cast_f32(s, y32, y, num_sms(),
                                            static_cast<cudaStream_t>(stream)));
}

moe_status moe_train_state_size(const moe_shape* shape, size_t* bytes) {
    moe_status st = check_shape(shape);
    if (st != MOE_OK) return st;
    if (!bytes) return MOE_ERR_INVALID_ARG;
    *bytes = train_state_layout(*shape, nullptr).total;
    return MOE_OK;
}

moe_status moe_forward_train(const moe_shape* shape, const void* x, const int32_t* offsets,
                             const int32_t* perm, const float* topk_w, const void* gate_up,
                             const void* down, const void* sh_gate_up, const void* sh_down,
                             void* y_slots, void* state, size_t state_bytes, int32_t* err_flag,
                             void* workspace, size_t workspace_bytes, void* stream) {
    moe_status st = check_shape(shape);
    if (st != MOE_OK) return st;
    const moe_shape& s = *shape;
    if (s.T == 0) return MOE_OK;
    if ((st = check_train_shape(s)) != MOE_OK) return st;
    if (!gate_up || !down) return MOE_ERR_INVALID_ARG;
    if (s.n_shared > 0 && (!sh_gate_up || !sh_down)) return MOE_ERR_INVALID_ARG;
    const TrainState ts = train_state_layout(s, state);
    if (!state || state_bytes < ts.total) return MOE_ERR_WORKSPACE;
    if (!aligned16(state)) return MOE_ERR_UNSUPPORTED;
    return forward_range(s, 0, s.E, true, x, offsets, perm, topk_w, gate_up, down, sh_gate_up,
                         sh_down, y_slots, err_flag, workspace, workspace_bytes,
                         static_cast<cudaStream_t>(stream), &ts);
}

moe_status moe_backward_workspace_size(const moe_shape* shape, size_t* bytes) {
    moe_status st = check_shape(shape);
    if (st != MOE_OK) return st;
    if (!bytes) return MOE_ERR_INVALID_ARG;
    *bytes = bwd_layout(*shape).total;
    return MOE_OK;
}

moe_status moe_backward(const moe_shape* shape, const void* x, const float* w_router,
                        const int32_t* topk_idx, const float* topk_w, const int32_t* counts,
                        const int32_t* offsets, const int32_t* perm, const int32_t* inv,
                        const void* gate_up, const void* down, const void* sh_gate_up,
                        const void* sh_down, const void* state, const float* logits,
                        float aux_coef, const void* dy, void* dx, float* d_gate_up,
                        float* d_down, float* d_sh_gate_up, float* d_sh_down, float* d_w_router,
                        float* d_router_bias, float* d_topk_w, float* aux_loss,
                        int32_t* err_flag, void* workspace, size_t workspace_bytes,
                        void* stream) {
    moe_status st = check_shape(shape);
    if (st != MOE_OK) return st;
    const moe_shape& s = *shape;
    if (s.T == 0) return MOE_OK;
    if ((st = check_train_shape(s)) != MOE_OK) return st;
    if (!x || !w_router || !topk_idx || !topk_w || !counts || !offsets || !perm || !inv ||
        !gate_up || !down || !state || !dy || !dx || !d_gate_up || !d_down || !d_w_router)
        return MOE_ERR_INVALID_ARG;
    if (s.n_shared > 0 && (!sh_gate_up || !sh_down || !d_sh_gate_up || !d_sh_down))
        return MOE_ERR_INVALID_ARG;
    if (aux_coef != 0.f && !logits) return MOE_ERR_INVALID_ARG;
    const BwdLayout bl = bwd_layout(s);
    if (!workspace || workspace_bytes < bl.total) return MOE_ERR_WORKSPACE;
    const void* ptrs[] = {x, w_router, gate_up, down, state, dy, dx, d_gate_up, d_down,
                          d_w_router, workspace};
    for (const void* p : ptrs)
        if (!aligned16(p)) return MOE_ERR_UNSUPPORTED;
    if (s.n_shared > 0 && (!aligned16(sh_gate_up) || !aligned16(sh_down) ||
                           !aligned16(d_sh_gate_up) || !aligned16(d_sh_down)))
        return MOE_ERR_UNSUPPORTED;
    char* ws = static_cast<char*>(workspace);
    moe::BackwardBuffers b{};
    b.poffsets = reinterpret_cast<int32_t*>(ws + bl.poff);
    b.dO = ws + bl.dO;
    b.dgu = ws + bl.dgu;
    b.dgu_sh = ws + bl.dgu_sh;
    b.dX_sh = ws + bl.dX_sh;
    b.dw_raw = reinterpret_cast<float*>(ws + bl.dw_raw);
    b.dl = reinterpret_cast<float*>(ws + bl.dl);
    b.part = reinterpret_cast<float*>(ws + bl.part);
    b.partb = reinterpret_cast<float*>(ws + bl.partb);
    const TrainState ts = train_state_layout(s, const_cast<void*>(state));
    return cuda_status(moe::launch_backward(
        s, x, w_router, topk_idx, topk_w, counts, offsets, perm, inv, gate_up, down, sh_gate_up,
        sh_down, ts.gu, ts.gu_sh, ts.h, ts.h_sh, ts.x_perm, logits, aux_coef, dy, dx, d_gate_up,
        d_down, d_sh_gate_up, d_sh_down, d_w_router, d_router_bias, d_topk_w, aux_loss, b,
        err_flag, num_sms(), static_cast<cudaStream_t>(stream)));
}

moe_status moe_forward_mxfp4(const moe_shape* shape, const void* x, const int32_t* offsets,
                             const int32_t* perm, const float* topk_w, const uint8_t* gate_up_q,
                             const uint8_t* gate_up_s, const uint8_t* down_q,
                             const uint8_t* down_s, void* y_slots, int32_t* err_flag,
                             void* workspace, size_t workspace_bytes, void* stream) {
    moe_status st = check_shape(shape);
    if (st != MOE_OK) return st;
    const moe_shape& s = *shape;
    if (s.T == 0) return MOE_OK;
    if (s.dtype != MOE_BF16 || s.n_shared != 0 || s.T > 64 || s.H % 32 != 0 || s.I % 32 != 0)
        return MOE_ERR_UNSUPPORTED;
    if (!x || !offsets || !perm || !topk_w || !gate_up_q || !gate_up_s || !down_q || !down_s ||
        !y_slots)
        return MOE_ERR_INVALID_ARG;
    const Workspace w = layout(s);
    if (!workspace || workspace_bytes < w.total) return MOE_ERR_WORKSPACE;
    const void* ptrs[] = {x, gate_up_q, down_q, y_slots, workspace};
    for (const void* p : ptrs)
        if (!aligned16(p)) return MOE_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(gate_up_s) & 3u) || (reinterpret_cast<uintptr_t>(down_s) & 3u))
        return MOE_ERR_UNSUPPORTED;
    char* ws = static_cast<char*>(workspace);
    if (moe::mx_tc_supported(s, gate_up_q, down_q, false))
        return cuda_status(moe::launch_ffn_decode_mxfp4_tc(
            s, x, offsets, perm, topk_w, gate_up_q, gate_up_s, down_q, down_s, nullptr,
            reinterpret_cast<uint8_t*>(ws + w.mx_xq_off), reinterpret_cast<uint8_t*>(ws + w.mx_xsf_off),
            reinterpret_cast<uint8_t*>(ws + w.mx_hq_off), reinterpret_cast<uint8_t*>(ws + w.mx_hsf_off),
            reinterpret_cast<float*>(ws + w.mx_part_off), reinterpret_cast<int32_t*>(ws + w.mx_ctl_off),
            y_slots, err_flag, num_sms(), static_cast<cudaStream_t>(stream)));
    return cuda_status(moe::launch_ffn_decode_mxfp4(
        s, x, offsets, perm, topk_w, gate_up_q, gate_up_s, down_q, down_s, ws + w.h_routed_off,
        ws + w.mx_x16_off, reinterpret_cast<int32_t*>(ws + w.mx_xexp_off), ws + w.mx_h16_off,
        reinterpret_cast<int32_t*>(ws + w.mx_hexp_off), y_slots, err_flag, num_sms(),
        static_cast<cudaStream_t>(stream)));
}

moe_status moe_mxfp4_prepared_size(const moe_shape* shape, size_t* bytes) {
    moe_status st = check_shape(shape);
    if (st != MOE_OK) return st;
    if (!bytes) return MOE_ERR_INVALID_ARG;
    *bytes = static_cast<size_t>(moe::mx_tc_prepared_bytes(*shape));
    return MOE_OK;
}

moe_status moe_mxfp4_prepare(const moe_shape* shape, const uint8_t* gate_up_q,
                             const uint8_t* gate_up_s, const uint8_t* down_q,
                             const uint8_t* down_s, void* prepared, size_t prepared_bytes,
                             void* stream) {
    moe_status st = check_shape(shape);
    if (st != MOE_OK) return st;
    const size_t need = static_cast<size_t>(moe::mx_tc_prepared_bytes(*shape));
    if (need == 0) return MOE_ERR_UNSUPPORTED;
    if (!gate_up_q || !gate_up_s || !down_q || !down_s || !prepared) return MOE_ERR_INVALID_ARG;
    if (prepared_bytes < need) return MOE_ERR_WORKSPACE;
    if (!aligned16(prepared) || !aligned16(gate_up_q) || !aligned16(down_q))
        return MOE_ERR_UNSUPPORTED;
    return cuda_status(moe::launch_mx_tc_prepare(*shape, gate_up_q, gate_up_s, down_q, down_s,
                                                 prepared, num_sms(),
                                                 static_cast<cudaStream_t>(stream)));
}

moe_status moe_forward_mxfp4_prepared(const moe_shape* shape, const void* x,
                                      const int32_t* offsets, const int32_t* perm,
                                      const float* topk_w, const uint8_t* gate_up_q,
                                      const uint8_t* down_q, const void* prepared, void* y_slots,
                                      int32_t* err_flag, void* workspace, size_t workspace_bytes,
                                      void* stream) {
    moe_status st = check_shape(shape);
    if (st != MOE_OK) return st;
    const moe_shape& s = *shape;
    if (s.T == 0) return MOE_OK;
    if (s.dtype != MOE_BF16 || s.n_shared != 0 || s.T > 64 || s.H % 64 != 0 || s.I % 64 != 0)
        return MOE_ERR_UNSUPPORTED;
    if (!x || !offsets || !perm || !topk_w || !gate_up_q || !down_q || !prepared || !y_slots)
        return MOE_ERR_INVALID_ARG;
    const Workspace w = layout(s);
    if (!workspace || workspace_bytes < w.total) return MOE_ERR_WORKSPACE;
    const void* ptrs[] = {x, gate_up_q, down_q, prepared, y_slots, workspace};
    for (const void* p : ptrs)
        if (!aligned16(p)) return MOE_ERR_UNSUPPORTED;
    if (!moe::mx_tc_supported(s, gate_up_q, down_q, true)) return MOE_ERR_UNSUPPORTED;
    char* ws = static_cast<char*>(workspace);
    return cuda_status(moe::launch_ffn_decode_mxfp4_tc(
        s, x, offsets, perm, topk_w, gate_up_q, nullptr, down_q, nullptr, prepared,
        reinterpret_cast<uint8_t*>(ws + w.mx_xq_off), reinterpret_cast<uint8_t*>(ws + w.mx_xsf_off),
        reinterpret_cast<uint8_t*>(ws + w.mx_hq_off), reinterpret_cast<uint8_t*>(ws + w.mx_hsf_off),
        reinterpret_cast<float*>(ws + w.mx_part_off), reinterpret_cast<int32_t*>(ws + w.mx_ctl_off),
        y_slots, err_flag, num_sms(), static_cast<cudaStream_t>(stream)));
}

moe_status moe_combine(const moe_shape* shape, const void* y_slots, const int32_t* inv, void* y,
                       void* stream) {
    moe_status st = check_shape(shape);
    if (st != MOE_OK) return st;
    if (shape->T == 0) return MOE_OK;
    if (!y_slots || !inv || !y) return MOE_ERR_INVALID_ARG;
    if (shape->dtype == MOE_BF16 && (!aligned16(y_slots) || !aligned16(y)))
        return MOE_ERR_UNSUPPORTED;
    if (shape->dtype == MOE_F32 && shape->H % 4 == 0 && (!aligned16(y_slots) || !aligned16(y)))
        return MOE_ERR_UNSUPPORTED;
    return cuda_status(
        moe::launch_combine(*shape, y_slots, inv, y, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
