// common.cuh - shared definitions of the CUDA library: the workspace layout,
// device status handling and small device helpers.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "moe.h"

namespace moe {

constexpr int kTokPerChunk = 32;          // tokens per top-k CTA-chunk (histogram granularity)
constexpr int kMaxK = 16;
constexpr int kMaxE = 1024;
constexpr int kMaxR = 256;
constexpr int kMaxBudget = 32;
constexpr int kPieceInts = 5;             // expert, rank, start, len, row0
constexpr int kBlockInts = 4;             // expert, row0, valid, rank

// header words
enum { H_STATUS = 0, H_NPIECES = 1, H_NBLOCKS = 2, H_TOTAL_ROWS = 3, H_MOVES = 4,
       H_REPLICAS = 5, H_TAU = 6, H_CANDIDATE = 7, H_WORDS = 8 };

// Work-queue counters of the grouped GEMM: for FC1 then FC2, two queue
// heads and a count of clusters that finished (all zero between launches).
constexpr int kGemmQWords = 12;

// Default bound of a device-side spin (clock cycles, about 2 s at 1.9 GHz).
constexpr long long kSpinBudget = 4000000000LL;

struct Shape {
    int32_t T, d, E, K, F, R, tile, budget, dtype, gating, plan_mode;
    int64_t N;          // T*K
    int64_t C;          // (T/R)*K
    int32_t per;        // E/R
    int64_t max_pieces, max_blocks, rows_cap;
    int32_t n_chunks;
    int32_t eb;         // element bytes of activations / weights
};

// Byte offsets of every array in a workspace.
struct WsLayout {
    int64_t header, chunk_counts, chunk_base, chunk_flags, pieces, exp_piece_off, exp_piece_idx,
        blocks, sched_off, sched, rank_load, rank_replicas, rank_row0, row_of, src_of, gemm_q, pair_ready;
    int64_t plan_end;
    // MOE_WS_LAYER extras
    int64_t idx, w, counts, arrivals, xp, h, yp;
    int64_t layer_end;
    // MOE_WS_LAYER_HOST extras
    int64_t logits_dev, x_dev, out_dev;
    int64_t host_end;
    // MOE_WS_LAYER_TRAIN extras: dY (later dXp), the pre-activations, dA | dG, dw
    int64_t dy, ag, dag, dw;
    int64_t train_end;
};

__host__ __device__ inline int64_t align_up(int64_t v, int64_t a) { return (v + a - 1) / a * a; }

// Upper bound on block pairs: every expert's pairs are ceil(blocks / 2).
inline int64_t max_pairs(const Shape& s) { return (s.max_blocks + s.E) / 2 + 1; }

// Device pointers into a workspace, passed by value to kernels.
struct WsPtrs {
    uint32_t* header;
    int32_t* chunk_counts;
    int32_t* chunk_base;
    uint32_t* chunk_flags;
    int32_t* pieces;
    int32_t* exp_piece_off;
    int32_t* exp_piece_idx;
    int32_t* blocks;
    int32_t* sched_off;
    int32_t* sched;
    int32_t* rank_load;
    int32_t* rank_replicas;
    int32_t* rank_row0;
    int32_t* row_of;
    int32_t* src_of;
    int32_t* gemm_q;     // [kGemmQWords] work-queue counters of the two GEMM launches
    int32_t* pair_ready; // [max_pairs] fused FFN: FC1 tiles stored per block pair
};

inline WsPtrs ws_ptrs(void* ws, const WsLayout& L) {
    char* b = static_cast<char*>(ws);
    WsPtrs p;
    p.header = reinterpret_cast<uint32_t*>(b + L.header);
    p.chunk_counts = reinterpret_cast<int32_t*>(b + L.chunk_counts);
    p.chunk_base = reinterpret_cast<int32_t*>(b + L.chunk_base);
    p.chunk_flags = reinterpret_cast<uint32_t*>(b + L.chunk_flags);
    p.pieces = reinterpret_cast<int32_t*>(b + L.pieces);
    p.exp_piece_off = reinterpret_cast<int32_t*>(b + L.exp_piece_off);
    p.exp_piece_idx = reinterpret_cast<int32_t*>(b + L.exp_piece_idx);
    p.blocks = reinterpret_cast<int32_t*>(b + L.blocks);
    p.sched_off = reinterpret_cast<int32_t*>(b + L.sched_off);
    p.sched = reinterpret_cast<int32_t*>(b + L.sched);
    p.rank_load = reinterpret_cast<int32_t*>(b + L.rank_load);
    p.rank_replicas = reinterpret_cast<int32_t*>(b + L.rank_replicas);
    p.rank_row0 = reinterpret_cast<int32_t*>(b + L.rank_row0);
    p.row_of = reinterpret_cast<int32_t*>(b + L.row_of);
    p.src_of = reinterpret_cast<int32_t*>(b + L.src_of);
    p.gemm_q = reinterpret_cast<int32_t*>(b + L.gemm_q);
    p.pair_ready = reinterpret_cast<int32_t*>(b + L.pair_ready);
    return p;
}

// MXFP8 scales of a [rows, K] matrix (K a multiple of 128): one E8M0 byte per
// 32 elements of a row, kept in 512-byte chunks, one per (128-row group,
// 128-column group), chunk index (row / 128) * (K / 128) + column / 128.
// Inside a chunk the scale of row r and 32-block b (both taken mod 128 and
// mod 4) sits at byte 16 * (r % 32) + 4 * (r / 32) + b: 32 lines of 16 bytes,
// the form in which the tensor cores' scale operand is copied into TMEM.
__host__ __device__ inline int64_t mx_scale_offset(int64_t row, int64_t kblock, int64_t K) {
    return ((row >> 7) * (K >> 7) + (kblock >> 2)) * 512 + (row & 31) * 16 + ((row >> 5) & 3) * 4 + (kblock & 3);
}
inline int64_t mx_scale_bytes(int64_t rows, int64_t K) { return (rows + 127) / 128 * (K / 128) * 512; }

__device__ inline void set_status(uint32_t* header, uint32_t bits) {
    atomicOr(header + H_STATUS, bits);
}

// Programmatic dependent launch along the layer's chain of kernels. A kernel
// launched by launch_pdl may have its CTAs placed while the kernel before it
// in the stream is still running; it calls pdl_wait() first, which returns
// once that kernel has completed with its memory visible, and then
// pdl_trigger(), which lets the next kernel of the stream be placed. A kernel
// passes pdl_trigger() only after its own pdl_wait(), so when a kernel starts,
// every kernel two or more places before it has completed.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args&&... args) {
    cudaLaunchConfig_t lc = {};
    lc.gridDim = grid;
    lc.blockDim = block;
    lc.dynamicSmemBytes = smem;
    lc.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
    return cudaLaunchKernelEx(&lc, kernel, std::forward<Args>(args)...);
}

// ---- shape and workspace layout, defined in api.cu ----
bool aligned16(const void* p);
// Validates cfg and fills the derived shape: INVALID_ARG for an ill-formed
// cfg, UNSUPPORTED for a well-formed one no kernel covers.
moe_status make_shape(const moe_config* cfg, Shape* s);
WsLayout make_layout(const Shape& s);

// ---- launchers (one per kernel family), defined in the kernel files ----
cudaError_t launch_topk_hist(const Shape& s, const float* logits, int32_t* idx, float* w,
                             const WsPtrs& ws, cudaStream_t st);
cudaError_t launch_plan(const Shape& s, int32_t* counts_out, const WsPtrs& ws, cudaStream_t st);
cudaError_t launch_row_maps(const Shape& s, const int32_t* idx, const WsPtrs& ws, cudaStream_t st);
cudaError_t launch_gather(const Shape& s, const void* x, void* xp, const WsPtrs& ws,
                          cudaStream_t st);
cudaError_t launch_combine(const Shape& s, const void* yp, const float* w, void* out,
                           const WsPtrs& ws, cudaStream_t st);
// which = 1: FC1 + SwiGLU (a_mat = xp, w = w_gate_up, out = h);
// which = 2: FC2 (a_mat = h, w = w_down, out = yp);
// which = 3 (tensor cores only): FC1 + SwiGLU with a_mat = x, rows gathered by the row map;
// which = 4 (tensor cores only): FC1 + SwiGLU as which = 1, also storing the pre-activations
// [gate | up] into preact [rows_cap, 2F] (the training forward).
cudaError_t launch_ffn_simt(const Shape& s, int which, const void* a_mat, const void* w, void* out,
                            const WsPtrs& ws, cudaStream_t st);
cudaError_t launch_bounded_wait_probe(uint32_t* status, long long budget, cudaStream_t st);
// The combine folded into FC2: the top-k weights [T, K], the layer output
// y [T, d] and one arrival counter per (token, 32 columns of y), [T, d/32],
// all zero before the launch (the launch leaves them zero when it completes).
struct FoldArgs {
    const float* topk_w;
    void* y;
    int32_t* arrivals;
};
// The grouped GEMM with the token rows as the MMA's N (which = 1: FC1 + SwiGLU,
// 2: FC2, with fold also the combine; bf16): the MMA covers each block's valid
// rows rounded up to 16; rows of h and yp past a block's valid ones are not written.
cudaError_t launch_ffn_tn(const Shape& s, int which, const void* a_mat, const void* w, void* out,
                          const WsPtrs& ws, cudaStream_t st, long long spin_budget,
                          const FoldArgs* fold = nullptr);
cudaError_t launch_ffn_tc(const Shape& s, int which, const void* a_mat, const void* w, void* out,
                          const WsPtrs& ws, cudaStream_t st, long long spin_budget, void* preact = nullptr);
// FC1 then FC2 in one launch (bf16): h and yp as launch_ffn_tc's which = 1 and 2;
// a_src is xp, or x [T, d] read through the row map when gather is set
cudaError_t launch_ffn_fused(const Shape& s, const void* a_src, const void* w_gate_up, const void* w_down, void* h,
                             void* yp, const WsPtrs& ws, cudaStream_t st, long long spin_budget,
                             bool gather = false);
// backward (bf16): mode 0 DGrad W2 + SwiGLU derivative (a_mat = dY, b_mat = w_down, ag, out = dAG),
// 1 DGrad W1 (a_mat = dAG, b_mat = w_gate_up, out = dXp), 2 WGrad W2 (a_mat = dY, b_mat = h,
// out = dW2 fp32), 3 WGrad W1 (a_mat = dAG, b_mat = xp, out = dW1 fp32)
cudaError_t launch_bwd_tc(const Shape& s, int mode, const void* a_mat, const void* b_mat, void* out,
                          const void* ag, const WsPtrs& ws, cudaStream_t st, long long spin_budget);
cudaError_t launch_bwd_scatter(const Shape& s, const void* d_out, const void* yp, const float* w, void* dy,
                               float* dw, const WsPtrs& ws, cudaStream_t st);
cudaError_t launch_zero_padding(const Shape& s, void* a, void* b, int64_t row_bytes, const WsPtrs& ws,
                                cudaStream_t st);
cudaError_t launch_dlogits(const Shape& s, const float* logits, const int32_t* idx, const float* w, const float* dw,
                           float* dl, cudaStream_t st);
// MX quantization of a bf16 [rows, K] matrix (fmt MOE_MX_W_E4M3: codes
// [rows, K]; MOE_MX_W_E2M1: codes [rows, K/2], two per byte) with chunked
// scales; with interleave_F > 0 the rows are those of w_gate_up [E, 2F, K]
// reordered so that every 128 rows of an expert hold 64 gate rows then the
// 64 matching up rows (the FC1 column tiles of the MX GEMM).
cudaError_t launch_mx_quantize(const void* x, int64_t rows, int K, int interleave_F, int fmt, uint8_t* q,
                               uint8_t* sc, cudaStream_t st);
// The dispatch with MXFP8 quantization of each token row on the way.
cudaError_t launch_dispatch_mx(const Shape& s, const void* x, uint8_t* xq, uint8_t* xs, const WsPtrs& ws,
                               cudaStream_t st);
// MX grouped GEMM: which 1 = FC1 + SwiGLU (a = xq/xs, w = W1 in the
// interleaved MX layout, out = hq, out_sc = hs), 2 = FC2 (a = hq/hs, w = W2,
// out = yp in bf16, out_sc unused); wfmt: the weights' element format.
cudaError_t launch_ffn_mx(const Shape& s, int which, const uint8_t* a_q, const uint8_t* a_sc, const uint8_t* w_q,
                          const uint8_t* w_sc, int wfmt, void* out, uint8_t* out_sc, const WsPtrs& ws,
                          cudaStream_t st, long long spin_budget);

}  // namespace moe
