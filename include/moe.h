/*
 * moe.h - C ABI of the routed-expert MoE layer library (libmoe.so), sm_100a.
 *
 * The layer: router top-k and gating, an expert-load histogram, a greedy
 * replication planner that gives each of R virtual expert-parallel ranks
 * exactly S*K routed entries under a per-rank replica budget, a permute of
 * token rows into an expert-major, tile-padded buffer, a grouped SwiGLU
 * expert FFN on the tensor cores, and a weighted combine.
 *
 * Sources, cited by page title and section:
 *   [MegaFlux] "MegaFlux: Skew-Resilient MoE Megakernels via Pipelined
 *              Expert Replication"
 *   [MoonEP]   "MoonEP routing flow - live" (an explainer of MoonEP's
 *              planning kernel)
 *
 * Conventions for every call:
 *  - Pointers named as device buffers are device pointers (cudaMalloc or
 *    torch CUDA tensors), row-major and contiguous, 16-byte aligned. The
 *    caller allocates and owns every buffer, the workspace included; the
 *    library never allocates, frees or synchronises, except where a call
 *    says so (moe_read_status, moe_layer_fwd_host).
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 *    default stream). A return other than MOE_OK is synchronous and means
 *    nothing was launched. Conditions found on the device go to a status
 *    word in the workspace; moe_read_status returns them.
 *  - cfg->dtype applies to x, the expert weights, xp, h, yp and out
 *    (bf16 on the tensor-core path, fp32 on the CUDA-core path). Router
 *    logits and gating weights are always fp32.
 *  - The library keeps no state between calls: distinct workspaces may be
 *    used from distinct host threads at once. A workspace holds one plan;
 *    calls that read it must follow the moe_plan that wrote it, on the same
 *    stream (or after it in stream order), with the same cfg.
 *  - There is no CPU fallback: a cfg the kernels do not cover returns
 *    MOE_ERR_UNSUPPORTED.
 */
#ifndef ROUTED_EXPERTS_MOE_H
#define ROUTED_EXPERTS_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* a cudaStream_t */

/* Synchronous return codes (host-detected). */
typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,   /* null or misaligned pointer, inconsistent sizes */
    MOE_ERR_UNSUPPORTED = 2,   /* a valid cfg that no kernel here covers */
    MOE_ERR_WORKSPACE = 3,     /* ws_bytes smaller than moe_workspace_size asks */
    MOE_ERR_CUDA = 4           /* a CUDA runtime call failed (launch, copy, query) */
} moe_status;

/* Device status bits (read with moe_read_status). */
enum {
    MOE_DEV_PLAN_INEXACT = 1u, /* the planner could not give every rank exactly S*K
                                  entries within the replica budget; the plan is still a
                                  valid partition and the layer output is still correct */
    MOE_DEV_TIMEOUT = 2u,      /* a bounded device-side wait gave up; outputs are invalid */
    MOE_DEV_BAD_INDEX = 4u     /* a non-finite router logit or an out-of-range index */
};

typedef enum { MOE_BF16 = 0, MOE_FP32 = 1 } moe_dtype;
typedef enum { MOE_GATE_SOFTMAX_TOPK = 0, MOE_GATE_SIGMOID_TOPK = 1 } moe_gating;

/* Planner modes.
 * MOE_PLAN_EXACT: [MoonEP] "The greedy balance, step by step" - every rank
 *   gets exactly S*K entries; each piece is padded to whole tiles.
 * MOE_PLAN_BLOCKS: [MegaFlux] §3.1 "Bounded greedy search", App. A.1, A.2 -
 *   load counted in token blocks of `tile` rows, tau = ceil(sum_e b_e / R);
 *   four greedy candidates (donor priority: overload or largest home
 *   expert; fan-out: one new copy per expert per round or many), at most
 *   budget+2 rounds each; the one with the smallest maximum load wins (then
 *   fewer replicas); replicas whose blocks fit on another copy within that
 *   maximum are pruned, then single blocks move from the most- to the
 *   least-loaded rank while they share an expert. Blocks are cut from each
 *   expert's list owner first, then by rank, so only an expert's last block
 *   is partial. Requires E*R <= 16384 and T <= 32767*tile. */
typedef enum { MOE_PLAN_EXACT = 0, MOE_PLAN_BLOCKS = 1 } moe_plan_mode;

/* Workspace kinds for moe_workspace_size. */
typedef enum {
    MOE_WS_PLAN = 0,       /* plan, row maps and scratch: moe_plan .. moe_combine */
    MOE_WS_LAYER = 1,      /* MOE_WS_PLAN plus top-k, xp, h and yp: moe_layer_fwd */
    MOE_WS_LAYER_HOST = 2, /* MOE_WS_LAYER plus device copies of logits, x and out:
                              moe_layer_fwd_host */
    MOE_WS_LAYER_TRAIN = 3 /* MOE_WS_LAYER_HOST plus the backward's buffers (dY, the
                              pre-activations, dA | dG, dw): moe_layer_fwd_train then
                              moe_layer_bwd */
} moe_ws_kind;

/*
 * Layer shape. T tokens, hidden size d, E experts, top-K, expert FFN width
 * F, R virtual expert-parallel ranks, token-block rows `tile` (beta), and
 * `budget` replicas a rank may host. S = T/R tokens per rank; every rank's
 * capacity is C = S*K entries. Expert e is owned by rank e / (E/R).
 * Requirements: T % R == 0, E % R == 0, 1 <= K <= min(E, 16), E <= 1024,
 * R <= 256, 0 <= budget <= 32. bf16: tile == 128, F % 128 == 0,
 * d % 256 == 0. fp32: tile in {16, 32, 64, 128}, d % 64 == 0, F % 64 == 0.
 */
typedef struct {
    int32_t T, d, E, K, F, R, tile, budget;
    int32_t dtype;      /* moe_dtype */
    int32_t gating;     /* moe_gating */
    int32_t plan_mode;  /* moe_plan_mode */
} moe_config;

/*
 * Where moe_plan leaves the plan inside the workspace (byte offsets from
 * the workspace base) and the capacities those arrays are sized for.
 * All arrays are int32.
 *   header     [8]: device status bits, n_pieces, n_blocks, total_rows,
 *                   moves, replicas in total, then for MOE_PLAN_BLOCKS tau
 *                   and the winning candidate (2*priority + fan-out), else 0, 0
 *   pieces     [max_pieces][5]: expert, rank, start, len, row0 - rank
 *                   `rank` computes entries [start, start+len) of expert's
 *                   (token, slot)-ordered list at padded rows row0..;
 *                   ordered by (rank, expert)
 *   blocks     [max_blocks][4]: expert, row0, valid rows, rank - one
 *                   tile of one expert, in piece order
 *   rank_load  [R]: valid entries per rank (exactly S*K when exact)
 *   rank_replicas [R]: foreign experts hosted per rank (<= budget)
 *   rank_row0  [R+1]: first padded row of each rank; [R] = total rows
 *   row_of     [T*K]: padded row of entry (t, k)
 *   src_of     [rows_cap]: token of each padded row, -1 for padding;
 *                   defined for rows below total_rows
 */
typedef struct {
    int64_t header, pieces, blocks, rank_load, rank_replicas, rank_row0, row_of, src_of;
    int64_t max_pieces, max_blocks, rows_cap;
} moe_plan_layout;

/* Bytes of workspace a call sequence needs (see moe_ws_kind). */
moe_status moe_workspace_size(const moe_config* cfg, int32_t kind, size_t* bytes);

/* Rows of the padded expert-major buffers xp, h and yp:
 * T*K + (E + R*budget)*tile (each of at most E + R*budget pieces pads
 * fewer than tile rows). */
moe_status moe_rows_capacity(const moe_config* cfg, int64_t* rows_cap);

/* Offsets of the plan arrays inside a MOE_WS_PLAN workspace (host only). */
moe_status moe_plan_view(const moe_config* cfg, moe_plan_layout* out);

/*
 * moe_plan - steps A1 to A5: top-k, gating, histogram, planner, row maps.
 *   logits    fp32 [T, E] (device): router logits, any bias already added.
 *   topk_idx  int32 [T, K] (device, out): the K largest logits of each
 *             token, in descending order, ties to the lower expert id
 *             ([MegaFlux] §1; §4.1: k distinct experts per token).
 *   topk_w    fp32 [T, K] (device, out): softmax of the chosen logits
 *             renormalised over them, or their sigmoids normalised over
 *             them (cfg->gating).
 *   counts    int32 [E] (device, out): routed entries per expert, the
 *             routing profile the planner consumes ([MegaFlux] §3.1).
 *   ws        device workspace of at least moe_workspace_size(MOE_WS_PLAN)
 *             bytes; receives the plan (moe_plan_view) and scratch.
 * The planner ([MoonEP] "The greedy balance, step by step"; [MegaFlux]
 * §3.1, §4.1, App. A.1, A.2): starting from every expert on its owner,
 * each move refills the rank with the fewest entries from the rank with
 * the most, slicing the donor's largest experts (the tail of the entries
 * it still holds) until the receiver holds S*K; a receiver takes at most
 * `budget` foreign experts. Every piece is padded to whole tiles at a
 * tile-aligned row; pieces are laid out in (rank, expert) order. Token
 * counts, expert choices and routing weights are untouched.
 */
moe_status moe_plan(const moe_config* cfg, const float* logits, int32_t* topk_idx, float* topk_w,
                    int32_t* counts, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * moe_dispatch - step A6: xp[row] = x[src_of[row]] for every valid row
 * ([MegaFlux] §1: routed activations go to the ranks that compute their
 * experts). Padding rows of xp are not written. Whatever they hold never
 * reaches a valid row of h or yp, nor the output: every output element of
 * the expert FFN depends on its own token row alone.
 *   x   [T, d] (device), xp [rows_cap, d] (device, out).
 */
moe_status moe_dispatch(const moe_config* cfg, const void* x, void* xp, const void* ws,
                        size_t ws_bytes, moe_stream_t stream);

/*
 * moe_expert_ffn - steps A7 and A8, the grouped SwiGLU expert FFN over the
 * planned blocks ([MegaFlux] §2.1, §3.2 "Forward": FC1 then FC2 per token
 * block; §4.1: SwiGLU experts).
 *   xp         [rows_cap, d] (device)
 *   w_gate_up  [E, 2F, d] (device): rows 0..F-1 of expert e are the gate
 *              projection, rows F..2F-1 the up projection (K-major).
 *   w_down     [E, d, F] (device, K-major).
 *   h          [rows_cap, F] (device, out): silu(xp.gate) * (xp.up) on
 *              valid rows.
 *   yp         [rows_cap, d] (device, out): h . w_down on valid rows.
 * Rows of h and yp that no entry maps to (padding) hold unspecified values:
 * bf16 layers leave them as they were, fp32 layers write zero. fp32
 * accumulation; in bf16 mode h and yp are rounded to bf16 once.
 * bf16 layers run on the tensor cores with the token rows as the MMA's N
 * dimension, so each block costs its valid rows rounded up to 16 rather
 * than a whole tile.
 */
moe_status moe_expert_ffn(const moe_config* cfg, const void* xp, const void* w_gate_up,
                          const void* w_down, void* h, void* yp, void* ws, size_t ws_bytes,
                          moe_stream_t stream);

/*
 * moe_expert_fc1 / moe_expert_fc2 - the two halves of moe_expert_ffn, for
 * callers that schedule or time them apart: fc1 writes h from xp and
 * w_gate_up (step A7), fc2 writes yp from h and w_down (step A8). Same
 * arguments, layouts and rounding as moe_expert_ffn.
 */
moe_status moe_expert_fc1(const moe_config* cfg, const void* xp, const void* w_gate_up, void* h, void* ws,
                          size_t ws_bytes, moe_stream_t stream);
moe_status moe_expert_fc2(const moe_config* cfg, const void* h, const void* w_down, void* yp, void* ws,
                          size_t ws_bytes, moe_stream_t stream);

/*
 * moe_expert_ffn_fused - moe_expert_ffn in one persistent launch (bf16
 * layers; fp32 returns MOE_ERR_UNSUPPORTED): the work list holds all FC1
 * tiles, then all FC2 tiles, and an FC2 tile of a block pair starts once
 * every FC1 tile of that pair is in memory ([MegaFlux] §2.1 and §3.2
 * "Forward": FC2 waits only for the activation block it needs). The pair's
 * readiness is a count in the workspace, raised with a release by each
 * epilogue warp after its stores and read with an acquire by the scheduler;
 * the wait is bounded and reports MOE_DEV_TIMEOUT. Same arguments, outputs
 * on valid rows and rounding as moe_expert_ffn; padding rows of h and yp are
 * written as zero. It computes whole 128-row tiles (one-block experts on a
 * CTA pair beside an empty half).
 */
moe_status moe_expert_ffn_fused(const moe_config* cfg, const void* xp, const void* w_gate_up, const void* w_down,
                                void* h, void* yp, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * moe_expert_ffn_fused_gather - steps A6 to A8 in one launch (bf16 layers):
 * moe_expert_ffn_fused with FC1's activation rows read straight from x
 * [T, d] (device) through the plan's row map (TMA four-row gathers; padding
 * rows repeat their block's first token and are stored as zero h and yp
 * rows), so xp is never written. The same formula and rounding as
 * moe_dispatch followed by moe_expert_ffn on valid rows. Other dtypes
 * return MOE_ERR_UNSUPPORTED.
 */
moe_status moe_expert_ffn_fused_gather(const moe_config* cfg, const void* x, const void* w_gate_up,
                                       const void* w_down, void* h, void* yp, void* ws, size_t ws_bytes,
                                       moe_stream_t stream);

/*
 * moe_expert_fc1_gather - steps A6 and A7 in one launch (bf16 layers only):
 * FC1 + SwiGLU whose activation rows are read straight from x [T, d]
 * (device) through the plan's row map, so no xp buffer is written or read
 * ([MegaFlux] §2.1: token movement overlapped with the tiled FC1 work).
 * h [rows_cap, F] (device, out) holds, on valid rows, the bits
 * moe_dispatch + moe_expert_fc1 give; padding rows of h are not written.
 * It needs no xp buffer (rows_cap * d elements less memory) but is slower
 * than the two launches: its rows arrive by 16-byte copies from scattered
 * token rows instead of one tensor copy of consecutive rows.
 * fp32 layers return MOE_ERR_UNSUPPORTED.
 */
moe_status moe_expert_fc1_gather(const moe_config* cfg, const void* x, const void* w_gate_up, void* h, void* ws,
                                 size_t ws_bytes, moe_stream_t stream);

/*
 * moe_combine - step A9, the weighted top-k sum ([MegaFlux] §1, §2.1):
 * out[t] = sum over k in order of topk_w[t,k] * yp[row_of(t,k)], in fp32,
 * rounded once to cfg->dtype.
 *   yp [rows_cap, d] (device), topk_w fp32 [T, K] (device),
 *   out [T, d] (device, out).
 */
moe_status moe_combine(const moe_config* cfg, const void* yp, const float* topk_w, void* out,
                       const void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * moe_expert_fc2_combine - steps A8 and A9 in one launch (bf16 layers):
 * moe_expert_fc2 with the weighted top-k sum folded into its epilogue
 * ([MegaFlux] §2.1 "Fixed-placement MegaMoE forward": a token's output is
 * formed as soon as its expert rows are done; §1: the outputs are combined
 * by the routing weights). yp [rows_cap, d] (device, out) is written as by
 * moe_expert_fc2, and out [T, d] (device, out) is bit-identical to
 * moe_combine(yp, topk_w): the same fixed k order, fp32 sum and one
 * rounding. Each (token, 32 columns) has an arrival counter; the epilogue
 * whose rows complete a token's K rows of those columns sums them.
 *   h [rows_cap, F], w_down [E, d, F], topk_w fp32 [T, K] (device).
 *   ws  a MOE_WS_LAYER workspace holding the plan of moe_plan (the counters
 *       live in its layer part; the call clears them first).
 * Returns MOE_ERR_UNSUPPORTED for fp32 layers, MOE_ERR_WORKSPACE when
 * ws_bytes is below moe_workspace_size(MOE_WS_LAYER).
 * It is slower than moe_expert_fc2 followed by moe_combine on one GPU: FC2
 * walks the experts in order, so most tokens complete in its last items and
 * their sums fall on the epilogue warps there. moe_layer_fwd does not use it.
 */
moe_status moe_expert_fc2_combine(const moe_config* cfg, const void* h, const void* w_down, const float* topk_w,
                                  void* yp, void* out, void* ws, size_t ws_bytes, moe_stream_t stream);

/* Which FC1 input path moe_layer_fwd takes for a shape. */
enum {
    MOE_PATH_DISPATCH = 0,   /* moe_dispatch, then moe_expert_fc1 */
    MOE_PATH_GATHER_FC1 = 1  /* moe_expert_fc1_gather (no dispatch launch, xp unused) */
};
/* moe_layer_path - *path = the moe_layer_fwd FC1 input path of cfg (host only). */
moe_status moe_layer_path(const moe_config* cfg, int32_t* path);

/*
 * moe_layer_fwd - the whole layer, A1 to A9, on device buffers, with
 * top-k, xp, h and yp carved from a MOE_WS_LAYER workspace: the kernels of
 * moe_plan, then moe_dispatch and moe_expert_fc1 or, for bf16 layers whose
 * x [T, d] takes at most 64 MiB, moe_expert_fc1_gather in their place (x
 * then stays in L2 and the gathered FC1 is as fast or faster; the result is
 * bit-identical either way), then moe_expert_fc2 and moe_combine. The
 * launches are chained (programmatic dependent launch) on the stream.
 */
moe_status moe_layer_fwd(const moe_config* cfg, const float* logits, const void* x,
                         const void* w_gate_up, const void* w_down, void* out, void* ws,
                         size_t ws_bytes, moe_stream_t stream);

/*
 * moe_layer_fwd_host - the whole layer with the activations in host
 * memory: copies logits [T,E] and x [T,d] from host to the device copies
 * in a MOE_WS_LAYER_HOST workspace, runs moe_layer_fwd, and copies out
 * [T,d] back to host memory, all on `stream` with cudaMemcpyAsync (host
 * buffers should be pinned for the copies to be asynchronous). Expert
 * weights stay device-resident. Does not synchronise: out_host is valid
 * once the stream has reached the end of this call.
 */
moe_status moe_layer_fwd_host(const moe_config* cfg, const float* logits_host, const void* x_host,
                              const void* w_gate_up, const void* w_down, void* out_host,
                              void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * moe_layer_fwd_train - moe_layer_fwd on a MOE_WS_LAYER_TRAIN workspace
 * that also keeps what the backward needs: FC1's epilogue stores the gate
 * and up pre-activations, rounded to bf16, next to h. Same output bits as
 * moe_layer_fwd. bf16 layers with F % 256 == 0; others return
 * MOE_ERR_UNSUPPORTED.
 */
moe_status moe_layer_fwd_train(const moe_config* cfg, const float* logits, const void* x, const void* w_gate_up,
                               const void* w_down, void* out, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * moe_layer_bwd - the layer's backward on one GPU ([MegaFlux] §3.2
 * "Backward": DGrad through W2 then W1, WGrad per expert with the partial
 * gradients of an expert's replicas reduced into one). bf16 layers with
 * F % 256 == 0; others return MOE_ERR_UNSUPPORTED.
 *   ws         a MOE_WS_LAYER_TRAIN workspace on which moe_layer_fwd_train
 *              last ran with the same logits, x and weights (its top-k,
 *              plan, xp, h, yp and pre-activations are read; xp's padding
 *              rows are zeroed).
 *   logits     fp32 [T, E] (device), as given to moe_layer_fwd_train.
 *   w_gate_up  [E, 2F, d], w_down [E, d, F] (device), as given to moe_layer_fwd_train.
 *   d_out      [T, d] (device): the gradient of the loss with respect to out.
 *   dx         [T, d] (device, out): sum over k, in k order, of each entry's
 *              input gradient, in fp32, rounded once.
 *   dw_gate_up fp32 [E, 2F, d], dw_down fp32 [E, d, F] (device, out): every
 *              expert's weight gradients, zero for an expert no token chose.
 *   dlogits    fp32 [T, E] (device, out) or NULL: the gradient through the
 *              gating (softmax or sigmoid over the chosen logits); zero off
 *              each token's top-k (selection itself has no gradient).
 * Rounding points: each entry's dY = w * dOut is formed in fp32 and rounded
 * to bf16; FC1's pre-activations are the forward's, rounded to bf16;
 * dA | dG and each entry's dx row are rounded to bf16 once each; products
 * accumulate in fp32. Asynchronous on `stream`; 8 kernel launches.
 */
moe_status moe_layer_bwd(const moe_config* cfg, const float* logits, const void* w_gate_up, const void* w_down,
                         const void* d_out, void* dx, float* dw_gate_up, float* dw_down, float* dlogits, void* ws,
                         size_t ws_bytes, moe_stream_t stream);

/*
 * ---- MX forward: MXFP8 activations with MXFP4 or MXFP8 weights ([MegaFlux]
 * §2.1 'Persistent MoE execution': block-scaled MX tensor-core MMA; §4.1
 * 'Setup': the forward on MX operands with fp32 accumulation and bf16
 * outputs; [MoonEP] "A bandwidth-only model": one scale per 32 elements).
 *
 * MXFP8 matrix [rows, K] (K a multiple of 128): codes uint8 [rows, K], one
 * E4M3 byte per element, row-major; scales uint8, one E8M0 byte per 32
 * consecutive elements of a row (value 2^(s - 127)), in 512-byte chunks:
 * chunk (row / 128) * (K / 128) + col / 128 holds the scales of its 128 rows
 * and four 32-blocks, the scale of row r, block b at byte
 * 16 * (r % 32) + 4 * ((r % 128) / 32) + b % 4 of the chunk; that is
 * ceil(rows / 128) * (K / 128) * 512 bytes. Quantization (OCP Microscaling):
 * s = floor(log2 max|v|) - 8 + 127 clamped to [0, 254] (0 for an all-zero
 * block), each element v / 2^(s-127) rounded to E4M3, nearest with ties to
 * even, saturating at +-448.
 * The MX calls take bf16 layers (cfg->dtype == MOE_BF16, tile 128, d % 256 ==
 * 0, F % 128 == 0) and return MOE_ERR_UNSUPPORTED for others.
 */
/* Element format of MX expert weights: MXFP8 (E4M3, one byte per element) or
 * MXFP4 ([MegaFlux] §4.1's forward weights: E2M1, values 0, 0.5, 1, 1.5, 2, 3,
 * 4, 6 and their negatives, two codes per byte, element 2i in the low nibble
 * of byte i; scale s = floor(log2 max|v|) - 2 + 127 clamped to [0, 254];
 * nearest with ties to even, saturating at +-6). Activations and h are
 * always MXFP8. */
enum { MOE_MX_W_E4M3 = 0, MOE_MX_W_E2M1 = 1 };

enum {
    MOE_MX_XQ = 0,   /* dispatched token rows: codes [rows_cap, d] */
    MOE_MX_XS = 1,   /*   and their scales */
    MOE_MX_HQ = 2,   /* FC1 output h: codes [rows_cap, F] */
    MOE_MX_HS = 3,   /*   and their scales */
    MOE_MX_W1Q = 4,  /* W1 codes [E * 2F, d] (E4M3) or [E * 2F, d / 2] (E2M1), rows in FC1 tile order */
    MOE_MX_W1S = 5,  /*   and their scales */
    MOE_MX_W2Q = 6,  /* W2 codes [E * d, F] (E4M3) or [E * d, F / 2] (E2M1) */
    MOE_MX_W2S = 7   /*   and their scales */
};

/* Bytes of one of the MX buffers above for cfg and weight format wfmt (which
 * only the weight codes depend on). */
moe_status moe_mx_buffer_bytes(const moe_config* cfg, int32_t which, int32_t wfmt, size_t* bytes);

/*
 * moe_mx_quantize_weights - MX expert weights (wfmt: MOE_MX_W_E4M3 or
 * MOE_MX_W_E2M1), once, ahead of the layers.
 *   w_gate_up bf16 [E, 2F, d], w_down bf16 [E, d, F] (device): as for moe_layer_fwd.
 *   w1q, w1s (device, out): W1 along d. Rows are reordered for the MX GEMM's
 *            FC1 column tiles: row e*2F + 128*t + i holds gate row e*2F +
 *            64*t + i for i < 64 and up row e*2F + F + 64*t + (i - 64) for
 *            i >= 64 (t < F/64).
 *   w2q, w2s (device, out): W2 along F, rows unchanged.
 * Sizes from moe_mx_buffer_bytes. No workspace; asynchronous on `stream`.
 */
moe_status moe_mx_quantize_weights(const moe_config* cfg, const void* w_gate_up, const void* w_down, int32_t wfmt,
                                   void* w1q, void* w1s, void* w2q, void* w2s, moe_stream_t stream);

/*
 * moe_dispatch_mx - step A6 with MXFP8 quantization: each token row of x
 * (bf16 [T, d], device) is quantized along d once and its codes and scales
 * are stored to the K rows of the plan's row map. Padding rows of xq/xs are
 * not written. Needs the plan of moe_plan in ws (MOE_WS_PLAN or larger).
 *   xq, xs (device, out): MOE_MX_XQ / MOE_MX_XS buffers.
 */
moe_status moe_dispatch_mx(const moe_config* cfg, const void* x, void* xq, void* xs, const void* ws,
                           size_t ws_bytes, moe_stream_t stream);

/*
 * moe_expert_fc1_mx - step A7 on MX operands: per planned block,
 * h = silu(xq W1g^T) * (xq W1u^T) with the MMA's fp32 accumulation, rounded to
 * bf16, then quantized to MXFP8 along F into hq / hs (MOE_MX_HQ / MOE_MX_HS,
 * device, out). Padding rows of a block get zero codes and scale 0.
 *   xq, xs: from moe_dispatch_mx; w1q, w1s: from moe_mx_quantize_weights with
 *   weight format wfmt.
 */
moe_status moe_expert_fc1_mx(const moe_config* cfg, const void* xq, const void* xs, const void* w1q,
                             const void* w1s, int32_t wfmt, void* hq, void* hs, void* ws, size_t ws_bytes,
                             moe_stream_t stream);

/*
 * moe_expert_fc2_mx - step A8 on MX operands: yp = hq W2^T, fp32
 * accumulation, stored as bf16 [rows_cap, d] (device, out); padding rows are
 * zero. hq, hs: from moe_expert_fc1_mx; w2q, w2s: from moe_mx_quantize_weights
 * with weight format wfmt.
 */
moe_status moe_expert_fc2_mx(const moe_config* cfg, const void* hq, const void* hs, const void* w2q,
                             const void* w2s, int32_t wfmt, void* yp, void* ws, size_t ws_bytes,
                             moe_stream_t stream);

/*
 * moe_layer_fwd_mx - the whole layer on MX expert operands: moe_plan,
 * moe_dispatch_mx, moe_expert_fc1_mx, moe_expert_fc2_mx and moe_combine, on
 * a MOE_WS_LAYER workspace (xq/xs live where xp does, hq/hs where h does).
 *   logits fp32 [T, E], x bf16 [T, d] (device); w1q/w1s/w2q/w2s from
 *   moe_mx_quantize_weights with weight format wfmt (device); out bf16 [T, d]
 *   (device, out).
 */
moe_status moe_layer_fwd_mx(const moe_config* cfg, const float* logits, const void* x, const void* w1q,
                            const void* w1s, const void* w2q, const void* w2s, int32_t wfmt, void* out, void* ws,
                            size_t ws_bytes, moe_stream_t stream);

/*
 * moe_plan_noalloc - moe_plan for callers that cannot allocate device
 * memory. The papers have no counterpart: this is an interface for callers
 * that are handed only their inputs and outputs (a plugin inside another
 * framework's engine with no workspace to offer, or a serving loop whose
 * device memory is reserved up front by its own pool allocator, where
 * cudaMalloc can fail once the pool holds the free memory and can stall the
 * device mid-step).
 *   logits, topk_idx, topk_w, counts: as in moe_plan.
 *   row_of  int32 [T*K] (device, out): padded row of entry (t, k), as in
 *           moe_plan_layout.
 *   header  uint32 [8] (device, out): the header of moe_plan_layout: device
 *           status bits, n_pieces, n_blocks, total_rows, moves, replicas in
 *           total, then for MOE_PLAN_BLOCKS tau and the winning candidate,
 *           else 0, 0.
 * The planner's scratch lives in one static device array of
 * MOE_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that loads
 * the library keeps reserved until the process exits. A shape whose scratch
 * exceeds it returns MOE_ERR_WORKSPACE (moe_workspace_size with MOE_WS_PLAN
 * gives the bytes a shape needs). The call allocates and frees nothing.
 * Every call looks up the array's device address on the current device (a
 * lookup, not an allocation; it stays right after a cudaDeviceReset). The
 * first lookup on a device loads the library's device code there, so make
 * the first call on each device before any stream capture.
 * Every call shares the one array and it keeps the last call's contents;
 * calls that overlap on the GPU (for example on two streams at once) race
 * on it, so order them on one stream or with events.
 */
#define MOE_NOALLOC_SCRATCH_BYTES ((size_t)4 << 20)
moe_status moe_plan_noalloc(const moe_config* cfg, const float* logits, int32_t* topk_idx, float* topk_w,
                            int32_t* counts, int32_t* row_of, uint32_t* header, moe_stream_t stream);

/* Synchronises `stream`, then reads the device status bits of `ws`. */
moe_status moe_read_status(const void* ws, moe_stream_t stream, uint32_t* dev_bits);

/*
 * moe_probe_bounded_wait - a check of the device-side failure detection:
 * one CTA waits, through the same bounded wait the expert-FFN kernels use,
 * on an mbarrier that nothing ever arrives on. After budget_cycles clock
 * cycles (at most 2^34) the wait gives up, ORs MOE_DEV_TIMEOUT into
 * *status_word (a device uint32) and the kernel returns; the context stays
 * usable. No papers' counterpart: it exists so the timeout path can be
 * exercised without hanging or faulting a GPU.
 */
moe_status moe_probe_bounded_wait(uint32_t* status_word, int64_t budget_cycles, moe_stream_t stream);

/*
 * moe_probe_expert_ffn_timeout - a check of the expert FFN's failure
 * handling (bf16 layers; other dtypes return MOE_ERR_UNSUPPORTED):
 * moe_expert_ffn with every device-side wait of its tensor-core kernels
 * given budget_cycles clock cycles (1 .. 2^34) instead of about two seconds.
 * With a budget shorter than a copy or an MMA takes, waits run out: the
 * kernels OR MOE_DEV_TIMEOUT into the workspace's status word, stop both
 * CTAs of each pair, let every copy and MMA in flight finish, free their
 * tensor memory and return. h and yp are then undefined; the GEMM work
 * queues in the workspace are left at zero, so the next call runs normally
 * (moe_plan clears the status word). No papers' counterpart: it lets the
 * timeout path of the real kernels run on a GPU without a kernel broken on
 * purpose.
 */
moe_status moe_probe_expert_ffn_timeout(const moe_config* cfg, const void* xp, const void* w_gate_up,
                                        const void* w_down, void* h, void* yp, void* ws, size_t ws_bytes,
                                        int64_t budget_cycles, moe_stream_t stream);

/*
 * moe_probe_fc1_gather_timeout - the same check for moe_expert_fc1_gather
 * (FC1 reading x [T, d] through the row map; bf16 layers): every
 * device-side wait of its kernel, including those of its row-gather and
 * signal warps, gets budget_cycles clock cycles (1 .. 2^34). A stop drains
 * the row copies and the stage signals in flight before the CTAs leave. h
 * is then undefined; the next call runs normally. No papers' counterpart.
 */
moe_status moe_probe_fc1_gather_timeout(const moe_config* cfg, const void* x, const void* w_gate_up, void* h,
                                        void* ws, size_t ws_bytes, int64_t budget_cycles, moe_stream_t stream);

/* A static string naming a moe_status. */
const char* moe_status_string(moe_status s);

#ifdef __cplusplus
}
#endif

#endif /* ROUTED_EXPERTS_MOE_H */
