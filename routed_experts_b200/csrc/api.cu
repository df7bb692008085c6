// api.cu - the C ABI (include/moe.h): argument checks, the workspace layout and
// the launch sequence of each call. Host code only; no allocation, no
// synchronisation except in moe_read_status.
#include <string.h>

#include "common.cuh"

using namespace moe;

namespace moe {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Validates cfg and fills the derived shape. INVALID_ARG for an ill-formed
// cfg, UNSUPPORTED for a well-formed one no kernel covers.
moe_status make_shape(const moe_config* cfg, Shape* s) {
    if (!cfg || !s) return MOE_ERR_INVALID_ARG;
    const moe_config c = *cfg;
    if (c.T <= 0 || c.d <= 0 || c.E <= 0 || c.K <= 0 || c.F <= 0 || c.R <= 0 || c.tile <= 0 || c.budget < 0)
        return MOE_ERR_INVALID_ARG;
    if (c.K > c.E || c.T % c.R != 0 || c.E % c.R != 0) return MOE_ERR_INVALID_ARG;
    if (c.dtype != MOE_BF16 && c.dtype != MOE_FP32) return MOE_ERR_INVALID_ARG;
    if (c.gating != MOE_GATE_SOFTMAX_TOPK && c.gating != MOE_GATE_SIGMOID_TOPK) return MOE_ERR_INVALID_ARG;
    if (c.plan_mode != MOE_PLAN_EXACT && c.plan_mode != MOE_PLAN_BLOCKS) return MOE_ERR_INVALID_ARG;
    if (c.plan_mode == MOE_PLAN_BLOCKS &&
        ((int64_t)c.E * c.R > 16384 || (int64_t)c.T > (int64_t)32767 * c.tile))
        return MOE_ERR_UNSUPPORTED;
    if (c.K > kMaxK || c.E > kMaxE || c.R > kMaxR || c.budget > kMaxBudget || (int64_t)c.R * c.budget > 1024)
        return MOE_ERR_UNSUPPORTED;
    if (c.dtype == MOE_BF16) {
        if (c.tile != 128 || c.F % 128 != 0 || c.d % 256 != 0) return MOE_ERR_UNSUPPORTED;
    } else {
        if (!(c.tile == 16 || c.tile == 32 || c.tile == 64 || c.tile == 128) || c.d % 64 != 0 || c.F % 64 != 0)
            return MOE_ERR_UNSUPPORTED;
    }
    s->T = c.T; s->d = c.d; s->E = c.E; s->K = c.K; s->F = c.F; s->R = c.R; s->tile = c.tile;
    s->budget = c.budget; s->dtype = c.dtype; s->gating = c.gating; s->plan_mode = c.plan_mode;
    s->N = (int64_t)c.T * c.K;
    s->C = (int64_t)(c.T / c.R) * c.K;
    s->per = c.E / c.R;
    s->max_pieces = (int64_t)c.E + (int64_t)c.R * c.budget;
    s->max_blocks = (s->N + c.tile - 1) / c.tile + s->max_pieces;
    s->rows_cap = s->N + s->max_pieces * c.tile;
    s->n_chunks = (c.T + kTokPerChunk - 1) / kTokPerChunk;
    s->eb = c.dtype == MOE_BF16 ? 2 : 4;
    if (s->rows_cap >= (int64_t)1 << 31) return MOE_ERR_UNSUPPORTED;   // int32 row indices
    return MOE_OK;
}

WsLayout make_layout(const Shape& s) {
    WsLayout L;
    int64_t o = 0;
    auto take = [&](int64_t bytes) { const int64_t at = o; o = align_up(o + bytes, 256); return at; };
    L.header = take(sizeof(uint32_t) * H_WORDS);
    L.chunk_counts = take(sizeof(int32_t) * (int64_t)s.n_chunks * s.E);
    L.chunk_base = take(sizeof(int32_t) * (int64_t)s.n_chunks * s.E);
    L.chunk_flags = take(sizeof(uint32_t) * (int64_t)s.n_chunks);
    L.pieces = take(sizeof(int32_t) * kPieceInts * s.max_pieces);
    L.exp_piece_off = take(sizeof(int32_t) * (s.E + 1));
    L.exp_piece_idx = take(sizeof(int32_t) * s.max_pieces);
    L.blocks = take(sizeof(int32_t) * kBlockInts * s.max_blocks);
    L.sched_off = take(sizeof(int32_t) * (s.E + 1));
    L.sched = take(sizeof(int32_t) * s.max_blocks);
    L.rank_load = take(sizeof(int32_t) * s.R);
    L.rank_replicas = take(sizeof(int32_t) * s.R);
    L.rank_row0 = take(sizeof(int32_t) * (s.R + 1));
    L.row_of = take(sizeof(int32_t) * s.N);
    L.src_of = take(sizeof(int32_t) * s.rows_cap);
    L.gemm_q = take(sizeof(int32_t) * kGemmQWords);
    L.pair_ready = take(sizeof(int32_t) * max_pairs(s));
    L.plan_end = o;
    L.idx = take(sizeof(int32_t) * s.N);
    L.w = take(sizeof(float) * s.N);
    L.counts = take(sizeof(int32_t) * s.E);
    L.arrivals = take(sizeof(int32_t) * (int64_t)s.T * (s.d / 32));
    L.xp = take((int64_t)s.eb * s.rows_cap * s.d);
    L.h = take((int64_t)s.eb * s.rows_cap * s.F);
    L.yp = take((int64_t)s.eb * s.rows_cap * s.d);
    L.layer_end = o;
    L.logits_dev = take(sizeof(float) * (int64_t)s.T * s.E);
    L.x_dev = take((int64_t)s.eb * s.T * s.d);
    L.out_dev = take((int64_t)s.eb * s.T * s.d);
    L.host_end = o;
    L.dy = take((int64_t)s.eb * s.rows_cap * s.d);
    L.ag = take((int64_t)s.eb * s.rows_cap * 2 * s.F);
    L.dag = take((int64_t)s.eb * s.rows_cap * 2 * s.F);
    L.dw = take(sizeof(float) * s.N);
    L.train_end = o;
    return L;
}

}  // namespace moe

namespace {

moe_status check_ws(const void* ws, size_t ws_bytes, int64_t need) {
    if (!ws || !aligned16(ws)) return MOE_ERR_INVALID_ARG;
    if ((int64_t)ws_bytes < need) return MOE_ERR_WORKSPACE;
    return MOE_OK;
}

moe_status from_cuda(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

moe_status plan_impl(const Shape& s, const WsLayout& L, const float* logits, int32_t* idx, float* w,
                     int32_t* counts, void* ws, cudaStream_t st) {
    const WsPtrs P = ws_ptrs(ws, L);
    cudaError_t e = launch_topk_hist(s, logits, idx, w, P, st);
    if (e == cudaSuccess) e = launch_plan(s, counts, P, st);
    if (e == cudaSuccess) e = launch_row_maps(s, idx, P, st);
    return from_cuda(e);
}

moe_status fc_impl(const Shape& s, const WsLayout& L, int which, const void* a_mat, const void* w, void* out,
                   void* ws, cudaStream_t st) {
    const WsPtrs P = ws_ptrs(ws, L);
    cudaError_t e = s.dtype == MOE_BF16 ? launch_ffn_tc(s, which, a_mat, w, out, P, st, kSpinBudget)
                                        : launch_ffn_simt(s, which, a_mat, w, out, P, st);
    return from_cuda(e);
}

moe_status ffn_impl(const Shape& s, const WsLayout& L, const void* xp, const void* wgu, const void* wdn,
                    void* h, void* yp, void* ws, cudaStream_t st) {
    moe_status r = fc_impl(s, L, 1, xp, wgu, h, ws, st);
    if (r != MOE_OK) return r;
    return fc_impl(s, L, 2, h, wdn, yp, ws, st);
}

// moe_layer_fwd reads FC1's token rows straight from x (no dispatch launch,
// no xp) when x is small enough to stay in L2 beside the streaming weights:
// there the gathered FC1 measured as fast as dispatch + FC1 or faster, and
// with a larger x (whose rows it reads scattered from DRAM) slower.
constexpr int64_t kGatherMaxXBytes = (int64_t)64 << 20;
bool layer_gathers(const Shape& s) { return s.dtype == MOE_BF16 && (int64_t)s.T * s.d * s.eb <= kGatherMaxXBytes; }

moe_status mx_shape(const moe_config* cfg, Shape* s) {
    moe_status r = make_shape(cfg, s);
    if (r != MOE_OK) return r;
    if (s->dtype != MOE_BF16 || s->tile != 128 || s->d % 256 != 0 || s->F % 128 != 0) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

bool wfmt_ok(int32_t wfmt) { return wfmt == MOE_MX_W_E4M3 || wfmt == MOE_MX_W_E2M1; }

int64_t mx_bytes(const Shape& s, int which, int wfmt = MOE_MX_W_E4M3) {
    const int64_t per = wfmt == MOE_MX_W_E2M1 ? 2 : 1;   // weight elements per code byte
    switch (which) {
        case MOE_MX_XQ: return s.rows_cap * s.d;
        case MOE_MX_XS: return mx_scale_bytes(s.rows_cap, s.d);
        case MOE_MX_HQ: return s.rows_cap * s.F;
        case MOE_MX_HS: return mx_scale_bytes(s.rows_cap, s.F);
        case MOE_MX_W1Q: return (int64_t)s.E * 2 * s.F * s.d / per;
        case MOE_MX_W1S: return mx_scale_bytes((int64_t)s.E * 2 * s.F, s.d);
        case MOE_MX_W2Q: return (int64_t)s.E * s.d * s.F / per;
        case MOE_MX_W2S: return mx_scale_bytes((int64_t)s.E * s.d, s.F);
    }
    return -1;
}

}  // namespace

extern "C" {

moe_status moe_workspace_size(const moe_config* cfg, int32_t kind, size_t* bytes) {
    Shape s;
    moe_status r = make_shape(cfg, &s);
    if (r != MOE_OK) return r;
    if (!bytes) return MOE_ERR_INVALID_ARG;
    const WsLayout L = make_layout(s);
    switch (kind) {
        case MOE_WS_PLAN: *bytes = (size_t)L.plan_end; return MOE_OK;
        case MOE_WS_LAYER: *bytes = (size_t)L.layer_end; return MOE_OK;
        case MOE_WS_LAYER_HOST: *bytes = (size_t)L.host_end; return MOE_OK;
        case MOE_WS_LAYER_TRAIN: *bytes = (size_t)L.train_end; return MOE_OK;
        default: return MOE_ERR_INVALID_ARG;
    }
}

moe_status moe_rows_capacity(const moe_config* cfg, int64_t* rows_cap) {
    Shape s;
    moe_status r = make_shape(cfg, &s);
    if (r != MOE_OK) return r;
    if (!rows_cap) return MOE_ERR_INVALID_ARG;
    *rows_cap = s.rows_cap;
    return MOE_OK;
}

moe_status moe_plan_view(const moe_config* cfg, moe_plan_layout* out) {
    Shape s;
    moe_status r = make_shape(cfg, &s);
    if (r != MOE_OK) return r;
    if (!out) return MOE_ERR_INVALID_ARG;
    const WsLayout L = make_layout(s);
    out->header = L.header;
    out->pieces = L.pieces;
    out->blocks = L.blocks;
    out->rank_load = L.rank_load;
    out->rank_replicas = L.rank_replicas;
    out->rank_row0 = L.rank_row0;
    out->row_of = L.row_of;
    out->src_of = L.src_of;
    out->max_pieces = s.max_pieces;
    out->max_blocks = s.max_blocks;
    out->rows_cap = s.rows_cap;
    return MOE_OK;
}

moe_status moe_plan(const moe_config* cfg, const float* logits, int32_t* topk_idx, float* topk_w,
                    int32_t* counts, void* ws, size_t ws_bytes, moe_stream_t stream) {
    Shape s;
    moe_status r = make_shape(cfg, &s);
    if (r != MOE_OK) return r;
    if (!logits || !topk_idx || !topk_w || !counts) return MOE_ERR_INVALID_ARG;
    if (!aligned16(logits) || !aligned16(topk_idx) || !aligned16(topk_w) || !aligned16(counts))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = make_layout(s);
    if ((r = check_ws(ws, ws_bytes, L.plan_end)) != MOE_OK) return r;
    return plan_impl(s, L, logits, topk_idx, topk_w, counts, ws, reinterpret_cast<cudaStream_t>(stream));
}

moe_status moe_dispatch(const moe_config* cfg, const void* x, void* xp, const void* ws, size_t ws_bytes,
                        moe_stream_t stream) {
    Shape s;
    moe_status r = make_shape(cfg, &s);
    if (r != MOE_OK) return r;
    if (!x || !xp || !aligned16(x) || !aligned16(xp)) return MOE_ERR_INVALID_ARG;
    const WsLayout L = make_layout(s);
    if ((r = check_ws(ws, ws_bytes, L.plan_end)) != MOE_OK) return r;
    const WsPtrs P = ws_ptrs(const_cast<void*>(ws), L);
    return from_cuda(launch_gather(s, x, xp, P, reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_expert_ffn(const moe_config* cfg, const void* xp, const void* w_gate_up, const void* w_down,
                          void* h, void* yp, void* ws, size_t ws_bytes, moe_stream_t stream) {
    Shape s;
    moe_status r = make_shape(cfg, &s);
    if (r != MOE_OK) return r;
    if (!xp || !w_gate_up || !w_down || !h || !yp) return MOE_ERR_INVALID_ARG;
    if (!aligned16(xp) || !aligned16(w_gate_up) || !aligned16(w_down) || !aligned16(h) || !aligned16(yp))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = make_layout(s);
    if ((r = check_ws(ws, ws_bytes, L.plan_end)) != MOE_OK) return r;
    return ffn_impl(s, L, xp, w_gate_up, w_down, h, yp, ws, reinterpret_cast<cudaStream_t>(stream));
}

moe_status moe_expert_ffn_fused(const moe_config* cfg, const void* xp, const void* w_gate_up, const void* w_down,
                                void* h, void* yp, void* ws, size_t ws_bytes, moe_stream_t stream) {
    Shape s;
    moe_status r = make_shape(cfg, &s);
    if (r != MOE_OK) return r;
    if (s.dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
    if (!xp || !w_gate_up || !w_down || !h || !yp) return MOE_ERR_INVALID_ARG;
    if (!aligned16(xp) || !aligned16(w_gate_up) || !aligned16(w_down) || !aligned16(h) || !aligned16(yp))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = make_layout(s);
    if ((r = check_ws(ws, ws_bytes, L.plan_end)) != MOE_OK) return r;
    const WsPtrs P = ws_ptrs(ws, L);
    return from_cuda(launch_ffn_fused(s, xp, w_gate_up, w_down, h, yp, P, reinterpret_cast<cudaStream_t>(stream),
                                      kSpinBudget));
}

moe_status moe_expert_ffn_fused_gather(const moe_config* cfg, const void* x, const void* w_gate_up,
                                       const void* w_down, void* h, void* yp, void* ws, size_t ws_bytes,
                                       moe_stream_t stream) {
    Shape s;
    moe_status r = make_shape(cfg, &s);
    if (r != MOE_OK) return r;
    if (s.dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
    if (!x || !w_gate_up || !w_down || !h || !yp) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w_gate_up) || !aligned16(w_down) || !aligned16(h) || !aligned16(yp))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = make_layout(s);
    if ((r = check_ws(ws, ws_bytes, L.plan_end)) != MOE_OK) return r;
    const WsPtrs P = ws_ptrs(ws, L);
    return from_cuda(launch_ffn_fused(s, x, w_gate_up, w_down, h, yp, P, reinterpret_cast<cudaStream_t>(stream),
                                      kSpinBudget, true));
}

moe_status moe_expert_fc1(const moe_config* cfg, const void* xp, const void* w_gate_up, void* h, void* ws,
                          size_t ws_bytes, moe_stream_t stream) {
    Shape s;
    moe_status r = make_shape(cfg, &s);
    if (r != MOE_OK) return r;
    if (!xp || !w_gate_up || !h || !aligned16(xp) || !aligned16(w_gate_up) || !aligned16(h))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = make_layout(s);
    if ((r = check_ws(ws, ws_bytes, L.plan_end)) != MOE_OK) return r;
    return fc_impl(s, L, 1, xp, w_gate_up, h, ws, reinterpret_cast<cudaStream_t>(stream));
}

moe_status moe_expert_fc1_gather(const moe_config* cfg, const void* x, const void* w_gate_up, void* h, void* ws,
                                 size_t ws_bytes, moe_stream_t stream) {
    Shape s;
    moe_status r = make_shape(cfg, &s);
    if (r != MOE_OK) return r;
    if (s.dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
    if (!x || !w_gate_up || !h || !aligned16(x) || !aligned16(w_gate_up) || !aligned16(h))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = make_layout(s);
    if ((r = check_ws(ws, ws_bytes, L.plan_end)) != MOE_OK) return r;
    return fc_impl(s, L, 3, x, w_gate_up, h, ws, reinterpret_cast<cudaStream_t>(stream));
}

moe_status moe_expert_fc2(const moe_config* cfg, const void* h, const void* w_down, void* yp, void* ws,
                          size_t ws_bytes, moe_stream_t stream) {
    Shape s;
    moe_status r = make_shape(cfg, &s);
    if (r != MOE_OK) return r;
    if (!h || !w_down || !yp || !aligned16(h) || !aligned16(w_down) || !aligned16(yp))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = make_layout(s);
    if ((r = check_ws(ws, ws_bytes, L.plan_end)) != MOE_OK) return r;
    return fc_impl(s, L, 2, h, w_down, yp, ws, reinterpret_cast<cudaStream_t>(stream));
}

moe_status moe_expert_fc2_combine(const moe_config* cfg, const void* h, const void* w_down, const float* topk_w,
                                  void* yp, void* out, void* ws, size_t ws_bytes, moe_stream_t stream) {
    Shape s;
    moe_status r = make_shape(cfg, &s);
    if (r != MOE_OK) return r;
    if (s.dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
    if (!h || !w_down || !topk_w || !yp || !out) return MOE_ERR_INVALID_ARG;
    if (!aligned16(h) || !aligned16(w_down) || !aligned16(topk_w) || !aligned16(yp) || !aligned16(out))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = make_layout(s);
    if ((r = check_ws(ws, ws_bytes, L.layer_end)) != MOE_OK) return r;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int32_t* arrivals = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + L.arrivals);
    if (cudaMemsetAsync(arrivals, 0, sizeof(int32_t) * (size_t)s.T * (s.d / 32), st) != cudaSuccess)
        return MOE_ERR_CUDA;
    const FoldArgs fold{topk_w, out, arrivals};
    return from_cuda(launch_ffn_tn(s, 2, h, w_down, yp, ws_ptrs(ws, L), st, kSpinBudget, &fold));
}

moe_status moe_combine(const moe_config* cfg, const void* yp, const float* topk_w, void* out, const void* ws,
                       size_t ws_bytes, moe_stream_t stream) {
    Shape s;
    moe_status r = make_shape(cfg, &s);
    if (r != MOE_OK) return r;
    if (!yp || !topk_w || !out || !aligned16(yp) || !aligned16(topk_w) || !aligned16(out))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = make_layout(s);
    if ((r = check_ws(ws, ws_bytes, L.plan_end)) != MOE_OK) return r;
    const WsPtrs P = ws_ptrs(const_cast<void*>(ws), L);
    return from_cuda(launch_combine(s, yp, topk_w, out, P, reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_layer_fwd(const moe_config* cfg, const float* logits, const void* x, const void* w_gate_up,
                         const void* w_down, void* out, void* ws, size_t ws_bytes, moe_stream_t stream) {
    Shape s;
    moe_status r = make_shape(cfg, &s);
    if (r != MOE_OK) return r;
    if (!logits || !x || !w_gate_up || !w_down || !out) return MOE_ERR_INVALID_ARG;
    if (!aligned16(logits) || !aligned16(x) || !aligned16(w_gate_up) || !aligned16(w_down) || !aligned16(out))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = make_layout(s);
    if ((r = check_ws(ws, ws_bytes, L.layer_end)) != MOE_OK) return r;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    char* b = static_cast<char*>(ws);
    int32_t* idx = reinterpret_cast<int32_t*>(b + L.idx);
    float* w = reinterpret_cast<float*>(b + L.w);
    int32_t* counts = reinterpret_cast<int32_t*>(b + L.counts);
    void* xp = b + L.xp;
    void* h = b + L.h;
    void* yp = b + L.yp;
    if ((r = plan_impl(s, L, logits, idx, w, counts, ws, st)) != MOE_OK) return r;
    const WsPtrs P = ws_ptrs(ws, L);
    if (layer_gathers(s)) {
        cudaError_t e = launch_ffn_tc(s, 3, x, w_gate_up, h, P, st, kSpinBudget);   // FC1 reading x
        if (e == cudaSuccess) e = launch_ffn_tc(s, 2, h, w_down, yp, P, st, kSpinBudget);
        if (e == cudaSuccess) e = launch_combine(s, yp, w, out, P, st);
        return from_cuda(e);
    }
    if ((r = from_cuda(launch_gather(s, x, xp, P, st))) != MOE_OK) return r;
    if ((r = ffn_impl(s, L, xp, w_gate_up, w_down, h, yp, ws, st)) != MOE_OK) return r;
    return from_cuda(launch_combine(s, yp, w, out, P, st));
}

moe_status moe_layer_path(const moe_config* cfg, int32_t* path) {
    Shape s;
    moe_status r = make_shape(cfg, &s);
    if (r != MOE_OK) return r;
    if (!path) return MOE_ERR_INVALID_ARG;
    *path = layer_gathers(s) ? MOE_PATH_GATHER_FC1 : MOE_PATH_DISPATCH;
    return MOE_OK;
}

moe_status moe_layer_fwd_train(const moe_config* cfg, const float* logits, const void* x, const void* w_gate_up,
                               const void* w_down, void* out, void* ws, size_t ws_bytes, moe_stream_t stream) {
    Shape s;
    moe_status r = make_shape(cfg, &s);
    if (r != MOE_OK) return r;
    if (s.dtype != MOE_BF16 || s.F % 256 != 0) return MOE_ERR_UNSUPPORTED;
    if (!logits || !x || !w_gate_up || !w_down || !out) return MOE_ERR_INVALID_ARG;
    if (!aligned16(logits) || !aligned16(x) || !aligned16(w_gate_up) || !aligned16(w_down) || !aligned16(out))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = make_layout(s);
    if ((r = check_ws(ws, ws_bytes, L.train_end)) != MOE_OK) return r;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    char* b = static_cast<char*>(ws);
    int32_t* idx = reinterpret_cast<int32_t*>(b + L.idx);
    float* w = reinterpret_cast<float*>(b + L.w);
    int32_t* counts = reinterpret_cast<int32_t*>(b + L.counts);
    if ((r = plan_impl(s, L, logits, idx, w, counts, ws, st)) != MOE_OK) return r;
    const WsPtrs P = ws_ptrs(ws, L);
    cudaError_t e = launch_gather(s, x, b + L.xp, P, st);
    if (e == cudaSuccess) e = launch_ffn_tc(s, 4, b + L.xp, w_gate_up, b + L.h, P, st, kSpinBudget, b + L.ag);
    if (e == cudaSuccess) e = launch_ffn_tc(s, 2, b + L.h, w_down, b + L.yp, P, st, kSpinBudget);
    if (e == cudaSuccess) e = launch_combine(s, b + L.yp, w, out, P, st);
    return from_cuda(e);
}

moe_status moe_layer_fwd_host(const moe_config* cfg, const float* logits_host, const void* x_host,
                              const void* w_gate_up, const void* w_down, void* out_host, void* ws,
                              size_t ws_bytes, moe_stream_t stream) {
    Shape s;
    moe_status r = make_shape(cfg, &s);
    if (r != MOE_OK) return r;
    if (!logits_host || !x_host || !out_host) return MOE_ERR_INVALID_ARG;
    const WsLayout L = make_layout(s);
    if ((r = check_ws(ws, ws_bytes, L.host_end)) != MOE_OK) return r;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    char* b = static_cast<char*>(ws);
    float* lg = reinterpret_cast<float*>(b + L.logits_dev);
    void* x = b + L.x_dev;
    void* out = b + L.out_dev;
    const size_t lg_bytes = sizeof(float) * (size_t)s.T * s.E;
    const size_t x_bytes = (size_t)s.eb * s.T * s.d;
    if (cudaMemcpyAsync(lg, logits_host, lg_bytes, cudaMemcpyHostToDevice, st) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemcpyAsync(x, x_host, x_bytes, cudaMemcpyHostToDevice, st) != cudaSuccess) return MOE_ERR_CUDA;
    if ((r = moe_layer_fwd(cfg, lg, x, w_gate_up, w_down, out, ws, ws_bytes, stream)) != MOE_OK) return r;
    if (cudaMemcpyAsync(out_host, out, x_bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
}

moe_status moe_layer_bwd(const moe_config* cfg, const float* logits, const void* w_gate_up, const void* w_down,
                         const void* d_out, void* dx, float* dw_gate_up, float* dw_down, float* dlogits, void* ws,
                         size_t ws_bytes, moe_stream_t stream) {
    Shape s;
    moe_status r = make_shape(cfg, &s);
    if (r != MOE_OK) return r;
    if (s.dtype != MOE_BF16 || s.F % 256 != 0) return MOE_ERR_UNSUPPORTED;
    if (!logits || !w_gate_up || !w_down || !d_out || !dx || !dw_gate_up || !dw_down) return MOE_ERR_INVALID_ARG;
    if (!aligned16(logits) || !aligned16(w_gate_up) || !aligned16(w_down) || !aligned16(d_out) || !aligned16(dx) ||
        !aligned16(dw_gate_up) || !aligned16(dw_down) || (dlogits && !aligned16(dlogits)))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = make_layout(s);
    if ((r = check_ws(ws, ws_bytes, L.train_end)) != MOE_OK) return r;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    char* b = static_cast<char*>(ws);
    const int32_t* idx = reinterpret_cast<const int32_t*>(b + L.idx);
    const float* w = reinterpret_cast<const float*>(b + L.w);
    void* xp = b + L.xp;
    const void* h = b + L.h;
    const void* yp = b + L.yp;
    void* dy = b + L.dy;   // dY, then dXp once WGrad of W2 has read dY
    const void* ag = b + L.ag;   // the pre-activations moe_layer_fwd_train stored
    void* dag = b + L.dag;
    float* dw = reinterpret_cast<float*>(b + L.dw);
    const WsPtrs P = ws_ptrs(ws, L);
    cudaError_t e = launch_bwd_scatter(s, d_out, yp, w, dy, dw, P, st);
    if (e == cudaSuccess) e = launch_zero_padding(s, xp, dy, (int64_t)s.eb * s.d, P, st);
    if (e == cudaSuccess) e = launch_bwd_tc(s, 0, dy, w_down, dag, ag, P, st, kSpinBudget);
    if (e == cudaSuccess) e = launch_bwd_tc(s, 2, dy, h, dw_down, nullptr, P, st, kSpinBudget);
    if (e == cudaSuccess) e = launch_bwd_tc(s, 1, dag, w_gate_up, dy, nullptr, P, st, kSpinBudget);
    if (e == cudaSuccess) e = launch_bwd_tc(s, 3, dag, xp, dw_gate_up, nullptr, P, st, kSpinBudget);
    if (e == cudaSuccess) e = launch_combine(s, dy, nullptr, dx, P, st);
    if (e == cudaSuccess && dlogits) e = launch_dlogits(s, logits, idx, w, dw, dlogits, st);
    return from_cuda(e);
}

moe_status moe_mx_buffer_bytes(const moe_config* cfg, int32_t which, int32_t wfmt, size_t* bytes) {
    Shape s;
    moe_status r = mx_shape(cfg, &s);
    if (r != MOE_OK) return r;
    if (!bytes || which < MOE_MX_XQ || which > MOE_MX_W2S || !wfmt_ok(wfmt)) return MOE_ERR_INVALID_ARG;
    *bytes = (size_t)mx_bytes(s, which, wfmt);
    return MOE_OK;
}

moe_status moe_mx_quantize_weights(const moe_config* cfg, const void* w_gate_up, const void* w_down, int32_t wfmt,
                                   void* w1q, void* w1s, void* w2q, void* w2s, moe_stream_t stream) {
    Shape s;
    moe_status r = mx_shape(cfg, &s);
    if (r != MOE_OK) return r;
    if (!w_gate_up || !w_down || !w1q || !w1s || !w2q || !w2s || !wfmt_ok(wfmt)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(w_gate_up) || !aligned16(w_down) || !aligned16(w1q) || !aligned16(w1s) || !aligned16(w2q) ||
        !aligned16(w2s))
        return MOE_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = launch_mx_quantize(w_gate_up, (int64_t)s.E * 2 * s.F, s.d, s.F, wfmt,
                                       static_cast<uint8_t*>(w1q), static_cast<uint8_t*>(w1s), st);
    if (e == cudaSuccess)
        e = launch_mx_quantize(w_down, (int64_t)s.E * s.d, s.F, 0, wfmt, static_cast<uint8_t*>(w2q),
                               static_cast<uint8_t*>(w2s), st);
    return from_cuda(e);
}

moe_status moe_dispatch_mx(const moe_config* cfg, const void* x, void* xq, void* xs, const void* ws,
                           size_t ws_bytes, moe_stream_t stream) {
    Shape s;
    moe_status r = mx_shape(cfg, &s);
    if (r != MOE_OK) return r;
    if (!x || !xq || !xs || !aligned16(x) || !aligned16(xq) || !aligned16(xs)) return MOE_ERR_INVALID_ARG;
    const WsLayout L = make_layout(s);
    if ((r = check_ws(ws, ws_bytes, L.plan_end)) != MOE_OK) return r;
    const WsPtrs P = ws_ptrs(const_cast<void*>(ws), L);
    return from_cuda(launch_dispatch_mx(s, x, static_cast<uint8_t*>(xq), static_cast<uint8_t*>(xs), P,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_expert_fc1_mx(const moe_config* cfg, const void* xq, const void* xs, const void* w1q,
                             const void* w1s, int32_t wfmt, void* hq, void* hs, void* ws, size_t ws_bytes,
                             moe_stream_t stream) {
    Shape s;
    moe_status r = mx_shape(cfg, &s);
    if (r != MOE_OK) return r;
    if (!xq || !xs || !w1q || !w1s || !hq || !hs || !wfmt_ok(wfmt)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(xq) || !aligned16(xs) || !aligned16(w1q) || !aligned16(w1s) || !aligned16(hq) || !aligned16(hs))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = make_layout(s);
    if ((r = check_ws(ws, ws_bytes, L.plan_end)) != MOE_OK) return r;
    const WsPtrs P = ws_ptrs(ws, L);
    return from_cuda(launch_ffn_mx(s, 1, static_cast<const uint8_t*>(xq), static_cast<const uint8_t*>(xs),
                                   static_cast<const uint8_t*>(w1q), static_cast<const uint8_t*>(w1s), wfmt, hq,
                                   static_cast<uint8_t*>(hs), P, reinterpret_cast<cudaStream_t>(stream),
                                   kSpinBudget));
}

moe_status moe_expert_fc2_mx(const moe_config* cfg, const void* hq, const void* hs, const void* w2q,
                             const void* w2s, int32_t wfmt, void* yp, void* ws, size_t ws_bytes,
                             moe_stream_t stream) {
    Shape s;
    moe_status r = mx_shape(cfg, &s);
    if (r != MOE_OK) return r;
    if (!hq || !hs || !w2q || !w2s || !yp || !wfmt_ok(wfmt)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(hq) || !aligned16(hs) || !aligned16(w2q) || !aligned16(w2s) || !aligned16(yp))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = make_layout(s);
    if ((r = check_ws(ws, ws_bytes, L.plan_end)) != MOE_OK) return r;
    const WsPtrs P = ws_ptrs(ws, L);
    return from_cuda(launch_ffn_mx(s, 2, static_cast<const uint8_t*>(hq), static_cast<const uint8_t*>(hs),
                                   static_cast<const uint8_t*>(w2q), static_cast<const uint8_t*>(w2s), wfmt, yp,
                                   nullptr, P, reinterpret_cast<cudaStream_t>(stream), kSpinBudget));
}

moe_status moe_layer_fwd_mx(const moe_config* cfg, const float* logits, const void* x, const void* w1q,
                            const void* w1s, const void* w2q, const void* w2s, int32_t wfmt, void* out, void* ws,
                            size_t ws_bytes, moe_stream_t stream) {
    Shape s;
    moe_status r = mx_shape(cfg, &s);
    if (r != MOE_OK) return r;
    if (!logits || !x || !w1q || !w1s || !w2q || !w2s || !out || !wfmt_ok(wfmt)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(logits) || !aligned16(x) || !aligned16(w1q) || !aligned16(w1s) || !aligned16(w2q) ||
        !aligned16(w2s) || !aligned16(out))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = make_layout(s);
    if ((r = check_ws(ws, ws_bytes, L.layer_end)) != MOE_OK) return r;
    // xq | xs in xp's place, hq | hs in h's place
    const int64_t xs_at = align_up(mx_bytes(s, MOE_MX_XQ), 256), hs_at = align_up(mx_bytes(s, MOE_MX_HQ), 256);
    if (xs_at + mx_bytes(s, MOE_MX_XS) > L.h - L.xp || hs_at + mx_bytes(s, MOE_MX_HS) > L.yp - L.h)
        return MOE_ERR_UNSUPPORTED;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    char* b = static_cast<char*>(ws);
    int32_t* idx = reinterpret_cast<int32_t*>(b + L.idx);
    float* w = reinterpret_cast<float*>(b + L.w);
    int32_t* counts = reinterpret_cast<int32_t*>(b + L.counts);
    uint8_t* xq = reinterpret_cast<uint8_t*>(b + L.xp);
    uint8_t* xs = xq + xs_at;
    uint8_t* hq = reinterpret_cast<uint8_t*>(b + L.h);
    uint8_t* hs = hq + hs_at;
    void* yp = b + L.yp;
    if ((r = plan_impl(s, L, logits, idx, w, counts, ws, st)) != MOE_OK) return r;
    const WsPtrs P = ws_ptrs(ws, L);
    cudaError_t e = launch_dispatch_mx(s, x, xq, xs, P, st);
    if (e == cudaSuccess)
        e = launch_ffn_mx(s, 1, xq, xs, static_cast<const uint8_t*>(w1q), static_cast<const uint8_t*>(w1s), wfmt, hq,
                          hs, P, st, kSpinBudget);
    if (e == cudaSuccess)
        e = launch_ffn_mx(s, 2, hq, hs, static_cast<const uint8_t*>(w2q), static_cast<const uint8_t*>(w2s), wfmt, yp,
                          nullptr, P, st, kSpinBudget);
    if (e == cudaSuccess) e = launch_combine(s, yp, w, out, P, st);
    return from_cuda(e);
}

moe_status moe_read_status(const void* ws, moe_stream_t stream, uint32_t* dev_bits) {
    if (!ws || !dev_bits) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
    uint32_t v = 0;
    if (cudaMemcpy(&v, ws, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
    *dev_bits = v;
    return MOE_OK;
}

moe_status moe_probe_bounded_wait(uint32_t* status_word, int64_t budget_cycles, moe_stream_t stream) {
    if (!status_word || budget_cycles < 0 || budget_cycles > ((int64_t)1 << 34)) return MOE_ERR_INVALID_ARG;
    return from_cuda(launch_bounded_wait_probe(status_word, (long long)budget_cycles,
                                               reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_probe_expert_ffn_timeout(const moe_config* cfg, const void* xp, const void* w_gate_up,
                                        const void* w_down, void* h, void* yp, void* ws, size_t ws_bytes,
                                        int64_t budget_cycles, moe_stream_t stream) {
    Shape s;
    moe_status r = make_shape(cfg, &s);
    if (r != MOE_OK) return r;
    if (s.dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
    if (budget_cycles < 1 || budget_cycles > ((int64_t)1 << 34)) return MOE_ERR_INVALID_ARG;
    if (!xp || !w_gate_up || !w_down || !h || !yp) return MOE_ERR_INVALID_ARG;
    if (!aligned16(xp) || !aligned16(w_gate_up) || !aligned16(w_down) || !aligned16(h) || !aligned16(yp))
        return MOE_ERR_INVALID_ARG;
    const WsLayout L = make_layout(s);
    if ((r = check_ws(ws, ws_bytes, L.plan_end)) != MOE_OK) return r;
    const WsPtrs P = ws_ptrs(ws, L);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = launch_ffn_tn(s, 1, xp, w_gate_up, h, P, st, (long long)budget_cycles);
    if (e == cudaSuccess) e = launch_ffn_tn(s, 2, h, w_down, yp, P, st, (long long)budget_cycles);
    return from_cuda(e);
}

moe_status moe_probe_fc1_gather_timeout(const moe_config* cfg, const void* x, const void* w_gate_up, void* h,
                                        void* ws, size_t ws_bytes, int64_t budget_cycles, moe_stream_t stream) {
    Shape s;
    moe_status r = make_shape(cfg, &s);
    if (r != MOE_OK) return r;
    if (s.dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
    if (budget_cycles < 1 || budget_cycles > ((int64_t)1 << 34)) return MOE_ERR_INVALID_ARG;
    if (!x || !w_gate_up || !h || !aligned16(x) || !aligned16(w_gate_up) || !aligned16(h)) return MOE_ERR_INVALID_ARG;
    const WsLayout L = make_layout(s);
    if ((r = check_ws(ws, ws_bytes, L.plan_end)) != MOE_OK) return r;
    return from_cuda(launch_ffn_tn(s, 3, x, w_gate_up, h, ws_ptrs(ws, L), reinterpret_cast<cudaStream_t>(stream),
                                   (long long)budget_cycles));
}

const char* moe_status_string(moe_status s) {
    switch (s) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
        case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
        case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    }
    return "MOE_ERR_UNKNOWN";
}

}  // extern "C"
