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
size_t permute_workspace_bytes(const moe_shape&);
cudaError_t launch_permute(const moe_shape&, const int32_t*, int32_t*, int32_t*, int32_t*,
                           int32_t*, int32_t*, void*, cudaStream_t);
cudaError_t launch_ffn_simt(const moe_shape&, const void*, const int32_t*, const int32_t*,
                            const float*, const void*, const void*, const void*, const void*,
                            void*, void*, void*, cudaStream_t);
cudaError_t launch_ffn_sm100(const moe_shape&, const void*, const void*, const int32_t*,
                             const int32_t*, const float*, const void*, const void*, const void*,
                             const void*, void*, void*, void*, int32_t*, int, int, cudaStream_t);
cudaError_t launch_ffn_decode(const moe_shape&, const void*, const int32_t*, const int32_t*,
                              const float*, const void*, const void*, const void*, const void*,
                              void*, void*, void*, int, cudaStream_t);
cudaError_t launch_ffn_sm100_pair(const moe_shape&, const void*, const void*, const int32_t*,
                                  const int32_t*, const float*, const void*, const void*,
                                  const void*, const void*, void*, void*, void*, int32_t*, int, int,
                                  cudaStream_t);
cudaError_t launch_ffn_decode_mxfp4(const moe_shape&, const void*, const int32_t*,
                                    const int32_t*, const float*, const uint8_t*, const uint8_t*,
                                    const uint8_t*, const uint8_t*, void*, void*, int32_t*, void*,
                                    int32_t*, void*, int32_t*, int, cudaStream_t);
cudaError_t launch_combine(const moe_shape&, const void*, const int32_t*, void*, cudaStream_t);
cudaError_t launch_gather_rows(const moe_shape&, const void*, const int32_t*, void*, int,
                               cudaStream_t);
cudaError_t launch_gather_by_token(const moe_shape&, const void*, const int32_t*, int32_t*, void*,
                                   int, cudaStream_t);
}  // namespace moe

namespace {

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

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

struct Workspace {
    size_t permute_off, h_routed_off, h_shared_off, x_perm_off, inv_off;
    size_t mx_x16_off, mx_xexp_off, mx_h16_off, mx_hexp_off;   // MXFP4 decode (T <= 8)
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
    if (s.dtype == MOE_BF16 && s.T <= 8) {
        w.mx_x16_off = off;
        off += align_up(static_cast<size_t>(s.T) * s.H * 2);
        w.mx_xexp_off = off;
        off += align_up(static_cast<size_t>(s.T) * 4);
        w.mx_h16_off = off;
        off += align_up(static_cast<size_t>(Tk) * s.I * 2);
        w.mx_hexp_off = off;
        off += align_up(static_cast<size_t>(Tk) * 4);
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
    // few tokens: one CTA per token; many tokens, bf16: tensor cores; else CUDA cores
    if (shape->T <= 256 && shape->H <= 32768 && aligned16(w_router))
        return cuda_status(moe::launch_route_small(*shape, x, w_router, router_bias, logits,
                                                   topk_idx, topk_w, cs));
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

moe_status moe_forward(const moe_shape* shape, const void* x, const int32_t* offsets,
                       const int32_t* perm, const float* topk_w, const void* gate_up,
                       const void* down, const void* sh_gate_up, const void* sh_down,
                       void* y_slots, int32_t* err_flag, void* workspace,
                       size_t workspace_bytes, void* stream) {
    moe_status st = check_shape(shape);
    if (st != MOE_OK) return st;
    const moe_shape& s = *shape;
    if (s.T == 0) return MOE_OK;
    if (!x || !offsets || !perm || !topk_w || !gate_up || !down || !y_slots)
        return MOE_ERR_INVALID_ARG;
    if (s.n_shared > 0 && (!sh_gate_up || !sh_down)) return MOE_ERR_INVALID_ARG;
    const Workspace w = layout(s);
    if (!workspace || workspace_bytes < w.total) return MOE_ERR_WORKSPACE;
    char* ws = static_cast<char*>(workspace);
    void* h_routed = ws + w.h_routed_off;
    void* h_shared = ws + w.h_shared_off;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (s.dtype == MOE_F32) {
        return cuda_status(moe::launch_ffn_simt(s, x, offsets, perm, topk_w, gate_up, down,
                                                sh_gate_up, sh_down, h_routed, h_shared, y_slots,
                                                cs));
    }
    const void* ptrs[] = {x, gate_up, down, y_slots, workspace};
    for (const void* p : ptrs)
        if (!aligned16(p)) return MOE_ERR_UNSUPPORTED;
    if (s.n_shared > 0 && (!aligned16(sh_gate_up) || !aligned16(sh_down)))
        return MOE_ERR_UNSUPPORTED;
    const int sms = num_sms();
    // decode batches (<= 8 rows per expert): stream the active experts' weights
    if (s.T <= 8)
        return cuda_status(moe::launch_ffn_decode(s, x, offsets, perm, topk_w, gate_up, down,
                                                  sh_gate_up, sh_down, h_routed, h_shared,
                                                  y_slots, sms, cs));
    void* x_perm = ws + w.x_perm_off;
    // x rows in sorted slot order for GEMM 1.  When x is too large to stay in
    // L2 between its k copies, gather token-major (each row of x read once,
    // written k times; measured 1.3-2.7 % faster per step on the 67-134 MB
    // batches); otherwise slot-major, which needs no inverse permutation.
    const bool by_token = static_cast<int64_t>(s.T) * s.H * 2 > (int64_t(48) << 20);
    cudaError_t e = by_token
                        ? moe::launch_gather_by_token(s, x, perm,
                                                      reinterpret_cast<int32_t*>(ws + w.inv_off),
                                                      x_perm, sms, cs)
                        : moe::launch_gather_rows(s, x, perm, x_perm, sms, cs);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    // CTA pairs (256-row tiles) when the experts average at least 256 rows;
    // one CTA per tile otherwise (less padding on small groups)
#ifndef MOE_PAIR_MIN_ROWS
#define MOE_PAIR_MIN_ROWS 256
#endif
#ifndef MOE_PAIR_GROUP_M
#define MOE_PAIR_GROUP_M 16
#endif
    if (s.T * s.k >= static_cast<int64_t>(MOE_PAIR_MIN_ROWS) * s.E)
        return cuda_status(moe::launch_ffn_sm100_pair(s, x, x_perm, offsets, perm, topk_w, gate_up,
                                                      down, sh_gate_up, sh_down, h_routed,
                                                      h_shared, y_slots, err_flag, sms,
                                                      MOE_PAIR_GROUP_M, cs));
    return cuda_status(moe::launch_ffn_sm100(s, x, x_perm, offsets, perm, topk_w, gate_up, down,
                                             sh_gate_up, sh_down, h_routed, h_shared, y_slots,
                                             err_flag, sms, 8, cs));
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
    if (s.dtype != MOE_BF16 || s.n_shared != 0 || s.T > 8 || s.H % 32 != 0 || s.I % 32 != 0)
        return MOE_ERR_UNSUPPORTED;
    if (!x || !offsets || !perm || !topk_w || !gate_up_q || !gate_up_s || !down_q || !down_s ||
        !y_slots)
        return MOE_ERR_INVALID_ARG;
    const Workspace w = layout(s);
    if (!workspace || workspace_bytes < w.total) return MOE_ERR_WORKSPACE;
    const void* ptrs[] = {x, gate_up_q, down_q, y_slots, workspace};
    for (const void* p : ptrs)
        if (!aligned16(p)) return MOE_ERR_UNSUPPORTED;
    char* ws = static_cast<char*>(workspace);
    return cuda_status(moe::launch_ffn_decode_mxfp4(
        s, x, offsets, perm, topk_w, gate_up_q, gate_up_s, down_q, down_s, ws + w.h_routed_off,
        ws + w.mx_x16_off, reinterpret_cast<int32_t*>(ws + w.mx_xexp_off), ws + w.mx_h16_off,
        reinterpret_cast<int32_t*>(ws + w.mx_hexp_off), y_slots, err_flag, num_sms(),
        static_cast<cudaStream_t>(stream)));
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
