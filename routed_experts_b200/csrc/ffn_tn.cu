// ffn_tn.cu - the grouped SwiGLU expert FFN (steps A7, A8, bf16 layers) with
// the token rows as the N dimension of the tensor-core MMA: a persistent,
// warp-specialised tcgen05 GEMM over the planned token blocks, run by CTA
// pairs, fed by TMA, accumulating in TMEM.
//
// [MegaFlux] "MegaFlux: Skew-Resilient MoE Megakernels via Pipelined Expert
// Replication", §2.1 'Persistent MoE execution': persistent CTAs with
// warp-specialised workers (token movement, MMA, epilogue), tcgen05 MMA with
// fp32 accumulation in TMEM, operands staged by TMA, two-CTA MMA; §3.1
// 'Problem formulation': a token block is the FC1/FC2 token tile, and
// splitting an expert's rows over ranks can leave a partial block at every
// copy; §3.2 'Forward': FC1 needs W1 and an input block, FC2 needs W2 and the
// finished activation block.
//
// Why the tokens are the N dimension. A planned block holds up to 128 valid
// rows of one expert, and every piece of the plan ends in a partial block; on
// skewed layers with many small experts a quarter or more of the rows in the
// planned blocks are padding. With the weights as the MMA's M (256 rows over
// the CTA pair, 128 in each CTA) and the token rows as its N, the MMA covers
// only a block's valid rows rounded up to 16 (N may be any multiple of 16
// up to 256), so padding costs at most 15 rows per block instead of up to 127.
//
// Work item = (two planned blocks of one expert, weight slab j): one
// cta_group::2 MMA tile of M = 256 weight rows x N = 2n token rows, n being
// the larger of the two blocks' valid rows rounded up to 16. The planner
// lists an expert's whole blocks first and its partial blocks by decreasing
// size, so the two blocks of a pair are about the same size. An expert with
// an odd number of blocks gives its last item one block, the smallest, with
// N = its valid rows rounded up to 32 (half of them in each CTA).
//   FC1 + SwiGLU: slab j covers h columns 128j .. 128j+127; the even CTA
//     holds weight rows for h columns 128j + [0, 64), the odd CTA for
//     128j + 64 + [0, 64). Each CTA's 128 weight rows come from one 5-D TMA
//     box laid out in four groups of 32 rows, one group per TMEM lane
//     quarter: 16 gate rows, then the 16 up rows of the same h columns. So
//     the epilogue warp of each quarter holds gate (lanes 0-15) and up (lanes
//     16-31) of the same 16 h columns and forms SwiGLU with one warp shuffle.
//   FC2: slab j covers yp columns 256j .. 256j+255, 128 per CTA.
// The token rows (the MMA's B operand) are split between the CTAs: the even
// CTA holds block 0's first n rows, the odd CTA block 1's (or, for a single
// block, rows n .. 2n-1 of it). Each CTA brings its n rows with one TMA box
// per k-step (one tensor map per box height 16, 32, .., 128): a k-step is
// two copies per CTA, the weight rows and the token rows. (Copies per
// k-step, more than bytes, set the pace of the operand feed: an earlier
// version that built each CTA's rows from up to four exact boxes moved fewer
// bytes and ran slower.)
//
// The accumulator of an item holds, in each CTA, 128 lanes (its weight rows)
// x N columns (token rows). The epilogue drains it 32 token columns at a
// time, transposes through a per-warp staging tile in shared memory and
// stores whole row segments (32 or 64 bytes per token row) with vector
// stores. Only valid rows are written: padding rows of h and yp are left as
// they were.
//
// Scheduling is dynamic, as in the pair kernel of ffn_tc.cu: two atomic
// queues (one per half of the GPU, cut at an expert boundary) and a scheduler
// warp that decodes items into a 4-slot ring shared by both CTAs. Items are
// listed expert-major; inside an expert, its block pairs in groups of at most
// G, each group through every weight slab (slab-major inside the group). A
// group's token rows then stay in L2 while its slabs stream past, and each
// slab is read once per group: G is the most pairs whose token rows fit in
// 32 MiB (8 on a 7168-wide FC1), so the concurrent items of one half of the
// GPU keep their token rows and a few slabs within that half's L2. (Plain
// slab-major order re-read the token rows of experts with many pairs for
// every slab: 18.3 GB of DRAM reads for a 10.3 GB FC1.) CTA = 7 warps: TMA
// (warp 0), MMA (warp 1, even CTA), epilogue (warps 2-5), scheduler (warp 6
// of the even CTA) / release forwarder (warp 6 of the odd CTA). Every wait
// is bounded; a wait that runs out sets MOE_DEV_TIMEOUT, raises the CTA's
// abort flag, lets its in-flight copies and MMAs finish and returns; both
// CTAs then meet at the cluster barrier and free TMEM.
//
// MODE 3 is FC1 + SwiGLU with the token rows read straight from x [T, d]
// through the row map, so no dispatched copy xp is written or read: four
// more warps per CTA copy each k-step's rows (16-byte cp.async into the
// 128-byte-swizzled layout the TMA box would have produced) and arrive on the
// stage's local gather barrier as their copies land (cp.async.mbarrier
// arrive); a fifth warp waits on it, fences the async proxy and signals the
// stage's row barrier on the even CTA, which the MMA thread waits on beside
// the weights' TMA barrier. The copying warps never wait for their own
// copies, so all stages of the ring can be in flight, as with TMA. The even
// CTA's signal is a local arrive that also expects 16 bytes; the odd CTA's is
// a 16-byte shared-to-shared bulk copy into the even CTA that completes those
// bytes on the same barrier. (A cluster-scope release arrive from the odd
// CTA cost about a microsecond per stage, and the MMA waited on it nearly
// half of the time.) Padding rows are not copied: their accumulator columns
// are never stored.
#include <cudaTypedefs.h>
#include <string.h>

#include "common.cuh"
#include "ptx.cuh"
#include "tc_common.cuh"

namespace moe {
namespace {

using namespace tc;

// A stage holds kTnSlabs 64-wide K slabs of both operands, each operand
// brought by one TMA copy: fewer, larger copies feed the MMAs faster than one
// copy per operand per 64-wide slab.
constexpr int kTnSlabs = 2;
constexpr int kTnSlabA = 128 * kBK * 2;                    // 16 KB: 128 weight rows x 64 columns
constexpr int kTnBytesA = kTnSlabs * kTnSlabA;             // this CTA's weight rows of a stage
constexpr int kTnBytesB = kTnSlabs * 128 * kBK * 2;        // up to 128 token rows of a stage
constexpr int kTnStageBytes = kTnBytesA + kTnBytesB;
constexpr int kTnStages = 6 / kTnSlabs;
constexpr int kTnK = kTnSlabs * kBK;                       // K covered by a stage
constexpr int kTnMaps = 8;                                 // token-row boxes of 16 (i + 1) rows
constexpr int kTnStg = 32 * 33 * 4;                        // per epilogue warp: 32 x 32 fp32 (+1 pad)

struct TnSmem {
    uint64_t full[kTnStages], empty[kTnStages], acc_full[2], acc_empty[2], drain;
    uint64_t item_full[kItemSlots], item_empty[kItemSlots], fwd_empty[kItemSlots];
    int4 items[kItemSlots];       // expert (-1: no more work), weight slab, first row of block 0, of block 1 (-1: none)
    uint32_t valid[kItemSlots];   // valid rows of block 0 (low 16 bits) and of block 1 (high)
    // Copies in flight at an abort (even CTA): the odd CTA's producer stores
    // the bytes of its latest fill of each stage and, when it stops, its
    // count of fills, then arrives on odd_done; peer_bytes holds the odd
    // CTA's bytes the even CTA expected for its own latest fill of each stage.
    uint64_t odd_done;
    uint64_t bfull[kTnStages];    // MODE 3 (even CTA): both CTAs' gathered rows of the stage have landed
    uint64_t gfull[kTnStages];    // MODE 3: this CTA's gathered rows of the stage have landed
    int4 g_item;                  // MODE 3: the item the gather warps work on (x = -2: stop)
    uint32_t g_valid;
    int g_ok;
    int32_t g_tok[128];           // MODE 3: token of each of this CTA's rows of the item (-1: padding)
    alignas(16) uint32_t sig_src[4];              // MODE 3 (odd CTA): source of the 16-byte signal copies
    alignas(16) uint32_t sig_dst[kTnStages][4];   // MODE 3 (even CTA): their destinations, one per stage
    uint64_t sig_done;            // MODE 3 (even CTA): the odd CTA's signal thread has stopped
    long long sig_fills;          // MODE 3 (even CTA): how many signal copies it issued
    uint32_t odd_bytes[kTnStages], peer_bytes[kTnStages];
    long long odd_fills;
    uint32_t tmem_base;
    int abort_flag;
};

constexpr size_t kTnSmemBytes = 1024 /*align slack*/ + kTnStages * kTnStageBytes + 4 * kTnStg + sizeof(TnSmem) +
                                2 * sizeof(int32_t) * (kMaxE + 1);
static_assert(kTnSmemBytes <= 232448, "shared memory per CTA");

struct TnMaps {
    CUtensorMap w;                // FC1: w_gate_up as 5-D (64, 16, gate/up, 16-row group, K slab);
                                  // FC2: w_down as 3-D (64, row, K slab), 128-row box
    CUtensorMap b[kTnMaps];       // xp (FC1) or h (FC2) as 3-D (64, row, K slab), boxes of 16, 32, .., 128 rows
};

struct TnArgs {
    int Kdim;                     // d (FC1) or F (FC2)
    int n_tiles;                  // weight slabs per expert: F/128 (FC1) or d/256 (FC2)
    int d;                        // FC2: rows of one expert in w_down
    int F;                        // FC1: h columns (gate rows) of one expert
    int E;
    int ld_out;                   // row length of the output: F (h) or d (yp)
    int group;                    // block pairs per group of the item order (G)
    long long spin;
    const int32_t* blocks;
    const int32_t* sched;
    const int32_t* sched_off;
    uint32_t* header;
    int32_t* queue;               // [3]: head of queue 0, head of queue 1, clusters finished
    __nv_bfloat16* out;
    // FC2 with the combine folded in (MODE 2)
    int K;                        // experts per token
    int T;
    int64_t rows_cap;
    const float* topk_w;          // [T, K]
    const int32_t* row_of;        // [T*K] token entry -> row of yp
    const int32_t* src_of;        // [rows_cap] row of yp -> token
    int32_t* arrivals;            // [T, d/32] rows of the token stored, per 32-column chunk (zero between launches)
    __nv_bfloat16* y;             // [T, d] the layer's output
    const __nv_bfloat16* x;       // MODE 3: the token rows [T, d]
};

constexpr int kGatherWarp = 7;    // MODE 3: warps 7 .. 10 gather the token rows
constexpr int kGatherThreads = 128;
constexpr int kSignalWarp = 11;   // MODE 3: turns landed gathers into row-barrier arrivals
constexpr int kGatherExtra = kGatherThreads + 32;
static_assert(kTnSlabs == 2, "the row gather splits a 16-byte chunk index as (row, slab, chunk) = (i/16, i/8%2, i%8)");

__device__ __forceinline__ int round16(int v) { return (v + 15) & ~15; }

__device__ __forceinline__ int round32(int v) { return (v + 31) & ~31; }

// Work item -> (expert e, its two blocks b0, b1 (b1 = -1: one block), weight
// slab j). Expert e owns items [n_tiles*p_off[e], n_tiles*p_off[e+1]); inside
// them, its pairs in groups of G, group-major, then slab, then pair.
__device__ __forceinline__ void decode_grouped(long long it, int n_tiles, int G, const int32_t* s_off,
                                               const int32_t* p_off, int E, const int32_t* sched, int& e, int& b0,
                                               int& b1, int& j) {
    int lo = 0, hi = E;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if ((long long)n_tiles * p_off[mid] <= it) lo = mid; else hi = mid;
    }
    e = lo;
    const int np = p_off[lo + 1] - p_off[lo];
    const int nb = s_off[lo + 1] - s_off[lo];
    const int local = (int)(it - (long long)n_tiles * p_off[lo]);
    const int full = np / G;                       // whole groups
    int q;
    if (local < full * G * n_tiles) {
        const int g = local / (G * n_tiles), r = local % (G * n_tiles);
        j = r / G;
        q = g * G + r % G;
    } else {
        const int rest = np - full * G, r = local - full * G * n_tiles;
        j = r / rest;
        q = full * G + r % rest;
    }
    b0 = sched[s_off[lo] + 2 * q];
    b1 = 2 * q + 1 < nb ? sched[s_off[lo] + 2 * q + 1] : -1;
}

// Token rows per CTA of an item: the larger block's valid rows rounded up to
// 16 for a pair, half of the single block's valid rows rounded up to 32.
__device__ __forceinline__ int item_rows(int v0, int v1, bool pair) {
    return pair ? max(round16(v0), round16(v1)) : round32(v0) >> 1;
}

// The item's 32-column chunk at c0 for one epilogue warp (TMEM lane quarter
// `quad`): FC1 forms h = silu(gate) * up (gate in lanes 0-15, up in lanes
// 16-31 of the quarter: 16 h columns, 32 bytes of each token row); FC2 has
// 32 yp columns (64 bytes of each token row). The values go through the
// warp's staging tile in shared memory so that two (FC1) or four (FC2)
// neighbouring lanes write each token row's bytes with one 16-byte store
// each: every store instruction writes whole 32-byte sectors. Token column
// s of the accumulator is row r0 + s of block 0 for s < n, else row
// r1 + s - n of block 1 (r1 < 0: a single block, row r0 + s); only valid
// rows are stored.
template <bool kFC1>
__device__ __forceinline__ void tn_chunk(uint32_t t_acc, int c0, int lane, float* stg, __nv_bfloat16* out,
                                         int ld, int col, int r0, int r1, int n, int v0, int v1) {
    uint32_t v[32];
    ptx::tmem_ld32(t_acc + (uint32_t)c0, v);
    ptx::tmem_ld_wait();
    auto row_of = [&](int t, int64_t& row) -> bool {   // token column c0 + t
        const int s = c0 + t;
        const bool in0 = s < n || r1 < 0;
        const int r = in0 ? s : s - n;
        row = (int64_t)(in0 ? r0 : r1) + r;
        return r < (in0 ? v0 : v1);
    };
    if (kFC1) {
        const bool lo = lane < 16;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            // lanes l and l + 16 trade the half of their columns the other one finishes:
            // lane l < 16 forms tokens c0 + i, lane l + 16 tokens c0 + 16 + i, of h column l % 16
            const float send = __uint_as_float(lo ? v[16 + i] : v[i]);
            const float recv = __shfl_xor_sync(0xffffffffu, send, 16);
            const float own = __uint_as_float(lo ? v[i] : v[16 + i]);
            const float gate = lo ? own : recv, up = lo ? recv : own;
            stg[((lo ? 0 : 16) + i) * 17 + (lane & 15)] = silu(gate) * up;   // [token][column]
        }
        __syncwarp();
        // two lanes per token row: 8 columns (16 bytes) each
        const int half = lane & 1;
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
            const int t = 16 * rr + (lane >> 1);
            const float* src = stg + t * 17 + 8 * half;
            const uint4 pk = make_uint4(pack_bf16(src[0], src[1]), pack_bf16(src[2], src[3]),
                                        pack_bf16(src[4], src[5]), pack_bf16(src[6], src[7]));
            int64_t row;
            if (row_of(t, row)) *reinterpret_cast<uint4*>(out + row * ld + col + 8 * half) = pk;
        }
    } else {
        // lane l holds yp column l of the quarter for tokens c0 .. c0 + 31
#pragma unroll
        for (int i = 0; i < 32; ++i) stg[lane * 33 + i] = __uint_as_float(v[i]);   // [column][token]
        __syncwarp();
        // four lanes per token row: 8 columns (16 bytes) each
        const int q = lane & 3;
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {
            const int t = 8 * rr + (lane >> 2);
            const float* src = stg + (8 * q) * 33 + t;
            const uint4 pk = make_uint4(pack_bf16(src[0], src[33]), pack_bf16(src[2 * 33], src[3 * 33]),
                                        pack_bf16(src[4 * 33], src[5 * 33]), pack_bf16(src[6 * 33], src[7 * 33]));
            int64_t row;
            if (row_of(t, row)) *reinterpret_cast<uint4*>(out + row * ld + col + 8 * q) = pk;
        }
    }
    __syncwarp();   // the staging tile is free for the next chunk
}

// The combine folded into FC2 (MODE 2), after one epilogue warp has stored
// its 32 yp columns (chunk col / 32) of every valid token row of an item:
// each of those rows counts itself on its token's arrival counter of the
// chunk, and the warp whose count completes a token's K rows forms
// y[t, col .. col + 31] = sum over k = 0..K-1, in that order, of
// w[t,k] * yp[row_of(t,k), col ..] in fp32 (fmaf from 0, one rounding to
// bf16: the arithmetic of combine.cu, so the result is bit-identical), then
// clears the counter for the next launch. The warp's stores, a warp barrier
// and a GPU-scope fence come before its counts (the release side); a warp
// that completes tokens fences once after its counts and reads the rows
// through L2 (ld.global.cg: another SM stored them during this launch).
// Eight completed tokens at a time, four lanes per token, 16 bytes (8
// columns) per lane.
__device__ __forceinline__ void tn_fold_combine(const TnArgs& a, int lane, int col, int r0, int r1, int n, int v0,
                                                int v1) {
    __syncwarp();
    __threadfence();
    const int n_chunks = a.d >> 5, chunk = col >> 5;
    const int rows = 2 * n;   // token columns of the item: block 0 then block 1 (or one block's 2n rows)
    int tok[8], old[8];
    bool bad = false;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        tok[i] = -1;
        old[i] = -1;
        const int s_ = 32 * i + lane;
        if (s_ < rows) {
            const bool in0 = s_ < n || r1 < 0;
            const int r = in0 ? s_ : s_ - n;
            if (r < (in0 ? v0 : v1)) {
                const int t = __ldg(a.src_of + (int64_t)(in0 ? r0 : r1) + r);
                if (t >= 0 && t < a.T) tok[i] = t; else bad = true;
            }
        }
        if (tok[i] >= 0) old[i] = atomicAdd(a.arrivals + (int64_t)tok[i] * n_chunks + chunk, 1);
    }
    const int g = lane >> 2, q = lane & 3;
    if (__any_sync(0xffffffffu, (old[0] == a.K - 1) | (old[1] == a.K - 1) | (old[2] == a.K - 1) |
                                    (old[3] == a.K - 1) | (old[4] == a.K - 1) | (old[5] == a.K - 1) |
                                    (old[6] == a.K - 1) | (old[7] == a.K - 1))) {
        __threadfence();
        __syncwarp();
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        unsigned m = __ballot_sync(0xffffffffu, old[i] == a.K - 1);
        while (m) {
            // the g-th completed token of this group of (up to) 8 goes to lanes 4g .. 4g+3
            unsigned mm = m;
            for (int x = 0; x < g && mm; ++x) mm &= mm - 1;
            const int src = mm ? __ffs(mm) - 1 : 0;
            const int t = __shfl_sync(0xffffffffu, tok[i], src);
            for (int x = 0; x < 8 && m; ++x) m &= m - 1;
            if (!mm) continue;
            if (q == 0) a.arrivals[(int64_t)t * n_chunks + chunk] = 0;
            float acc[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = 0.f;
            for (int k0 = 0; k0 < a.K; k0 += 8) {
                uint4 v[8];
                float wk[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    wk[u] = 0.f;
                    v[u] = make_uint4(0u, 0u, 0u, 0u);
                    if (k0 + u < a.K) {
                        const int64_t e = (int64_t)t * a.K + k0 + u;
                        const int row = __ldg(a.row_of + e);
                        if (row >= 0 && row < a.rows_cap) {
                            wk[u] = __ldg(a.topk_w + e);
                            v[u] = __ldcg(reinterpret_cast<const uint4*>(a.out + (int64_t)row * a.d + col + 8 * q));
                        } else {
                            bad = true;
                        }
                    }
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    if (k0 + u >= a.K) break;
                    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v[u]);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float2 f = __bfloat1622float2(p[j]);
                        acc[2 * j] = fmaf(wk[u], f.x, acc[2 * j]);
                        acc[2 * j + 1] = fmaf(wk[u], f.y, acc[2 * j + 1]);
                    }
                }
            }
            uint4 o;
            __nv_bfloat162* po = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
            for (int j = 0; j < 4; ++j) po[j] = __floats2bfloat162_rn(acc[2 * j], acc[2 * j + 1]);
            *reinterpret_cast<uint4*>(a.y + (int64_t)t * a.d + col + 8 * q) = o;
        }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) set_status(a.header, MOE_DEV_BAD_INDEX);
}

// MODE 0: FC1 + SwiGLU (B = xp, out = h); MODE 1: FC2 (B = h, out = yp);
// MODE 2: FC2 with the combine folded in (also y); MODE 3: FC1 + SwiGLU with
// B gathered from x.
template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(MODE == 3 ? kThreads + kGatherExtra : kThreads, 1)
ffn_tn_kernel(const __grid_constant__ TnMaps maps, TnArgs a) {
    constexpr bool kFC1 = MODE == 0 || MODE == 3;
    constexpr bool kFold = MODE == 2;
    constexpr bool kGather = MODE == 3;
    pdl_wait();
    pdl_trigger();
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* epi_base = reinterpret_cast<float*>(base + kTnStages * kTnStageBytes);
    TnSmem* S = reinterpret_cast<TnSmem*>(reinterpret_cast<uint8_t*>(epi_base) + 4 * kTnStg);
    int32_t* s_off = reinterpret_cast<int32_t*>(S + 1);
    int32_t* p_off = s_off + (a.E + 1);
    volatile int* abort_flag = &S->abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = ptx::cluster_ctarank();
    const bool even = rank == 0;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kTnStages; ++s) { ptx::mbar_init(&S->full[s], 1); ptx::mbar_init(&S->empty[s], 1); }
        for (int q = 0; q < 2; ++q) { ptx::mbar_init(&S->acc_full[q], 1); ptx::mbar_init(&S->acc_empty[q], 8); }
        for (int q = 0; q < kItemSlots; ++q) {
            ptx::mbar_init(&S->item_full[q], 1);
            // + the gather leader and the signal thread
            ptx::mbar_init(&S->item_empty[q], kItemConsumers + (kGather ? 2 : 0));
            ptx::mbar_init(&S->fwd_empty[q], kOddConsumers + (kGather ? 2 : 0));
        }
        for (int s_ = 0; s_ < kTnStages; ++s_) {
            ptx::mbar_init(&S->bfull[s_], 1);                 // the even signal, + 16 bytes from the odd CTA
            ptx::mbar_init(&S->gfull[s_], kGatherThreads);    // one per gather thread
        }
        ptx::mbar_init(&S->drain, 1);
        ptx::mbar_init(&S->odd_done, 1);
        ptx::mbar_init(&S->sig_done, 1);
        S->abort_flag = 0;
        ptx::fence_barrier_init();
    }
    for (int i = threadIdx.x; i <= a.E; i += blockDim.x) s_off[i] = a.sched_off[i];
    __syncthreads();
    if (warp == 0) {
        // pair offsets: p_off[e] = sum over e' < e of ceil(blocks of e' / 2)
        int carry = 0;
        if (lane == 0) p_off[0] = 0;
        for (int b = 0; b < a.E; b += 32) {
            const int i = b + lane;
            int x = i < a.E ? (s_off[i + 1] - s_off[i] + 1) >> 1 : 0;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, x, off);
                if (lane >= off) x += y;
            }
            if (i < a.E) p_off[i + 1] = carry + x;
            carry += __shfl_sync(0xffffffffu, x, 31);
        }
        if (lane == 0) {
            ptx::prefetch_tmap(&maps.w);
#pragma unroll
            for (int m = 0; m < kTnMaps; ++m) ptx::prefetch_tmap(&maps.b[m]);
        }
    }
    __syncthreads();
    ptx::cluster_sync();   // the peer's barriers exist before any remote arrive, store or copy
    if (warp == 1) { ptx::tmem_alloc_pair(&S->tmem_base, kTmemCols); ptx::tmem_relinquish_pair(); }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = S->tmem_base;
    const int n_items = p_off[a.E] * a.n_tiles;
    const int kb_count = a.Kdim / kTnK;

    auto slot_of = [](int k) { return k % kItemSlots; };
    auto parity_of = [](int k) { return (uint32_t)((k / kItemSlots) & 1); };
    auto take_item = [&](int k, int4& item, uint32_t& valid) -> bool {
        const bool ok = even ? role_wait(&S->item_full[slot_of(k)], parity_of(k), a.spin, abort_flag, a.header)
                             : role_wait_cluster(&S->item_full[slot_of(k)], parity_of(k), a.spin, abort_flag, a.header);
        if (!ok) return false;
        item = S->items[slot_of(k)];
        valid = S->valid[slot_of(k)];
        return true;
    };
    auto release_item = [&](int k) { ptx::mbar_arrive(even ? &S->item_empty[slot_of(k)] : &S->fwd_empty[slot_of(k)]); };
    // a role that gave up stops both CTAs of the pair (role_wait raised this CTA's flag)
    auto abort_pair = [&]() {
        *abort_flag = 1;
        ptx::st_cluster_u32(ptx::map_to_rank(ptx::smem_addr(&S->abort_flag), rank ^ 1u), 1u);
    };

    if (warp == kSchedWarp) {
        // ------------------------------------------------ scheduler (even CTA)
        if (even) {
            const int g = ptx::smid() >= (ptx::nsmid() >> 1) ? 1 : 0;
            int lo = 0, hi = a.E;   // first expert whose pairs start at or after half of all pairs
            const int half = p_off[a.E] / 2;
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (p_off[mid] < half) lo = mid + 1; else hi = mid;
            }
            const int split = p_off[lo] * a.n_tiles;
            int next = lane == 0 ? fetch_item(a.queue, g, split, n_items) : 0;
            for (int k = 0;; ++k) {
                const bool ok = role_wait_cluster(&S->item_empty[slot_of(k)], parity_of(k) ^ 1, a.spin, abort_flag,
                                                  a.header);
                if (lane == 0) {
                    int4 item = make_int4(-1, 0, -1, -1);
                    uint32_t valid = 0;
                    if (ok && next >= 0) {
                        int e, b0, b1, j;
                        decode_grouped(next, a.n_tiles, a.group, s_off, p_off, a.E, a.sched, e, b0, b1, j);
                        const int ra = a.blocks[kBlockInts * b0 + 1], va = a.blocks[kBlockInts * b0 + 2];
                        const int rb = b1 >= 0 ? a.blocks[kBlockInts * b1 + 1] : -1;
                        const int vb = b1 >= 0 ? a.blocks[kBlockInts * b1 + 2] : 0;
                        item = make_int4(e, j, ra, rb);
                        valid = (uint32_t)va | ((uint32_t)vb << 16);
                    }
                    // publish to both CTAs
                    S->items[slot_of(k)] = item;
                    S->valid[slot_of(k)] = valid;
                    ptx::st_cluster_v4(ptx::map_to_rank(ptx::smem_addr(&S->items[slot_of(k)]), 1), item);
                    ptx::st_cluster_u32(ptx::map_to_rank(ptx::smem_addr(&S->valid[slot_of(k)]), 1), valid);
                    ptx::mbar_arrive(&S->item_full[slot_of(k)]);
                    ptx::mbar_arrive_cluster(ptx::map_to_rank(ptx::smem_addr(&S->item_full[slot_of(k)]), 1));
                    if (item.x >= 0) next = fetch_item(a.queue, g, split, n_items);   // latency hides behind the ring
                    else next = -2;
                }
                if (__shfl_sync(0xffffffffu, next, 0) == -2) {
                    if (lane == 0 && !ok) abort_pair();
                    break;
                }
            }
            if (lane == 0) {
                // the last cluster to finish resets the queues for the next launch
                __threadfence();
                const int done = atomicAdd(&a.queue[2], 1);
                if (done == (int)ptx::cluster_count_x() - 1) {
                    a.queue[0] = 0;
                    a.queue[1] = 0;
                    __threadfence();
                    a.queue[2] = 0;
                }
            }
        } else if (lane == 0) {
            // forwarder (odd CTA): once this CTA's consumers have all released a
            // slot, release it to the even CTA's scheduler at cluster scope
            for (int k = 0;; ++k) {
                int4 item;
                uint32_t valid;
                if (!take_item(k, item, valid) ||
                    !role_wait(&S->fwd_empty[slot_of(k)], parity_of(k), a.spin, abort_flag, a.header)) {
                    abort_pair();
                    break;
                }
                ptx::mbar_arrive_cluster(ptx::map_to_rank(ptx::smem_addr(&S->item_empty[slot_of(k)]), 0));
                if (item.x < 0) break;
            }
        }
    } else if (warp == 0) {
        // ------------------------------------------------ TMA producer (both CTAs, lane 0)
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            long long fills = 0;
            bool ok = true;
            const uint32_t bar0 = ptx::map_to_rank(ptx::smem_addr(&S->full[0]), 0);
            for (int k = 0; ok; ++k) {
                int4 item;
                uint32_t valid;
                if (!take_item(k, item, valid)) { ok = false; break; }
                release_item(k);
                if (item.x < 0) break;
                const int e = item.x, j = item.y;
                const int n = item_rows((int)(valid & 0xffffu), (int)(valid >> 16), item.w >= 0);
                // this CTA's token rows: block 0's first n, then block 1's (or the single block's next n)
                const int brow = rank == 0 ? item.z : (item.w >= 0 ? item.w : item.z + n);
                const CUtensorMap* bmap = &maps.b[(n >> 4) - 1];
                const uint32_t cta_bytes = (uint32_t)(kTnBytesA + (kGather ? 0 : kTnSlabs * n * kBK * 2));
                const uint32_t tx = 2 * cta_bytes;   // both CTAs' copies count on the even CTA's barrier
                // FC1: the 64 h columns 128j + 64 rank .. as 4 groups of (16 gate rows, 16 up rows),
                // the first being 16-row group e*F/8 + (128j + 64 rank)/16 of w_gate_up
                const int fg = e * (a.F >> 3) + ((j * 128 + (int)rank * 64) >> 4);
                const int wrow = e * a.d + j * 256 + (int)rank * 128;   // FC2: this CTA's weight rows
                for (int kb = 0; kb < kb_count; ++kb) {
                    if (!role_wait(&S->empty[stage], phase ^ 1, a.spin, abort_flag, a.header)) { ok = false; break; }
                    const uint32_t bar = bar0 + (uint32_t)(stage * sizeof(uint64_t));
                    uint8_t* st = base + stage * kTnStageBytes;
                    if (even) {
                        ptx::mbar_arrive_expect_tx(&S->full[stage], tx);
                        S->peer_bytes[stage] = cta_bytes;
                    } else {
                        ptx::st_cluster_u32(ptx::map_to_rank(ptx::smem_addr(&S->odd_bytes[stage]), 0), cta_bytes);
                    }
                    if (kFC1) ptx::tma_load_5d_pair(st, &maps.w, 0, 0, 0, fg, kb * kTnSlabs, bar);
                    else ptx::tma_load_3d_pair(st, &maps.w, 0, wrow, kb * kTnSlabs, bar);
                    if (!kGather) ptx::tma_load_3d_pair(st + kTnBytesA, bmap, 0, brow, kb * kTnSlabs, bar);
                    ++fills;
                    if (++stage == kTnStages) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok) abort_pair();
            if (!even) {
                // tell the even CTA how far this producer got
                const uint32_t fa = ptx::map_to_rank(ptx::smem_addr(&S->odd_fills), 0);
                ptx::st_cluster_u32(fa, (uint32_t)(fills & 0xffffffffll));
                ptx::st_cluster_u32(fa + 4, (uint32_t)(fills >> 32));
                ptx::mbar_arrive_cluster(ptx::map_to_rank(ptx::smem_addr(&S->odd_done), 0));
            } else if (!ok) {
                // An abort: every copy either CTA issued must land before the
                // CTAs leave. Both producers fill the same sequence of stages;
                // the odd one can be at most one fill per stage past the even
                // one (it waits for the MMAs of the stage's previous fill,
                // which need the even CTA's arm) or behind it.
                long long fo = -1;
                if (ptx::mbar_wait_cluster(&S->odd_done, 0, kDrainBudget))
                    fo = *reinterpret_cast<volatile long long*>(&S->odd_fills);
                bool landed = true;
                const long long first = fills > kTnStages ? fills - kTnStages : 0;
                for (long long f = first; f < fills; ++f) {
                    const int s_ = (int)(f % kTnStages);
                    // a fill the odd producer never issued: count its half as arrived
                    if (fo >= 0 && f >= fo) ptx::mbar_complete_tx(&S->full[s_], S->peer_bytes[s_]);
                    landed &= ptx::mbar_wait(&S->full[s_], (uint32_t)((f / kTnStages) & 1), kDrainBudget);
                }
                // fills the odd producer issued into stages the even CTA never armed
                for (long long f = fills; landed && f < fo; ++f) {
                    const int s_ = (int)(f % kTnStages);
                    ptx::mbar_arrive_expect_tx(&S->full[s_], S->odd_bytes[s_]);
                    landed &= ptx::mbar_wait(&S->full[s_], (uint32_t)((f / kTnStages) & 1), kDrainBudget);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (even CTA)
        if (lane == 0 && even) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true, issued = false;
            for (int k = 0; ok; ++k) {
                int4 item;
                uint32_t valid;
                if (!take_item(k, item, valid)) { ok = false; break; }
                release_item(k);
                if (item.x < 0) break;
                const int N = 2 * item_rows((int)(valid & 0xffffu), (int)(valid >> 16), item.w >= 0);
                const uint32_t idesc = ptx::idesc_bf16_f32(2 * kBM, N);
                const int acc = k & 1;
                const uint32_t acc_phase = (uint32_t)((k >> 1) & 1);
                if (!role_wait_cluster(&S->acc_empty[acc], acc_phase ^ 1, a.spin, abort_flag, a.header)) { ok = false; break; }
                ptx::tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(acc * kN);
                for (int kb = 0; kb < kb_count; ++kb) {
                    if (!role_wait(&S->full[stage], phase, a.spin, abort_flag, a.header)) { ok = false; break; }
                    if (kGather && !role_wait_cluster(&S->bfull[stage], phase, a.spin, abort_flag, a.header)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t a_addr = ptx::smem_addr(base + stage * kTnStageBytes);
                    const uint32_t b_addr = a_addr + kTnBytesA;
#pragma unroll
                    for (int sl = 0; sl < kTnSlabs; ++sl) {
                        // slab sl: weight rows at sl * 16 KB, token rows at sl * (N/2 rows) * 128 B
                        const uint32_t as = a_addr + sl * kTnSlabA, bs = b_addr + sl * (N >> 1) * (kBK * 2);
#pragma unroll
                        for (int ks = 0; ks < kBK / 16; ++ks)
                            ptx::mma_bf16_pair(d_tmem, ptx::sdesc_k_sw128(as + ks * 32), ptx::sdesc_k_sw128(bs + ks * 32),
                                               idesc, (kb | sl | ks) != 0 ? 1u : 0u);
                    }
                    issued = true;
                    const uint32_t empty_addr = ptx::smem_addr(&S->empty[stage]);
                    ptx::mma_commit_pair(empty_addr);
                    ptx::mma_commit_pair(ptx::map_to_rank(empty_addr, 1));
                    if (++stage == kTnStages) { stage = 0; phase ^= 1; }
                }
                if (ok) {
                    const uint32_t full_addr = ptx::smem_addr(&S->acc_full[acc]);
                    ptx::mma_commit_pair(full_addr);
                    ptx::mma_commit_pair(ptx::map_to_rank(full_addr, 1));
                }
            }
            if (!ok) abort_pair();
            if (!ok && issued) {
                // wait for every MMA issued so far before TMEM is freed
                ptx::mma_commit_pair(ptx::smem_addr(&S->drain));
                ptx::mbar_wait(&S->drain, 0, kDrainBudget);
            }
        }
    } else if (kGather && warp == kSignalWarp) {
        // ------------------------------------------------ gather signal (MODE 3), warp 11 of both CTAs
        if (lane == 0) {
            const uint32_t bfull0 = ptx::map_to_rank(ptx::smem_addr(&S->bfull[0]), 0);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            long long fills = 0;   // stages signalled
            for (int k = 0; ok; ++k) {
                int4 item;
                uint32_t valid;
                if (!take_item(k, item, valid)) { ok = false; break; }
                release_item(k);
                if (item.x < 0) break;
                for (int kb = 0; kb < kb_count; ++kb, ++fills) {
                    if (!role_wait(&S->gfull[stage], phase, a.spin, abort_flag, a.header)) { ok = false; break; }
                    // the rows reached shared memory through the generic proxy; the MMAs read them
                    // through the async proxy
                    ptx::fence_proxy_async_shared();
                    if (even) {
                        ptx::mbar_arrive_expect_tx(&S->bfull[stage], 16u);
                    } else {
                        ptx::bulk_copy_s2c(ptx::map_to_rank(ptx::smem_addr(&S->sig_dst[stage][0]), 0),
                                           ptx::smem_addr(&S->sig_src[0]), 16u,
                                           bfull0 + (uint32_t)(stage * sizeof(uint64_t)));
                    }
                    if (++stage == kTnStages) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok) abort_pair();
            if (!even) {
                // tell the even CTA how many signal copies this CTA issued
                const uint32_t fa = ptx::map_to_rank(ptx::smem_addr(&S->sig_fills), 0);
                ptx::st_cluster_u32(fa, (uint32_t)(fills & 0xffffffffll));
                ptx::st_cluster_u32(fa + 4, (uint32_t)(fills >> 32));
                ptx::mbar_arrive_cluster(ptx::map_to_rank(ptx::smem_addr(&S->sig_done), 0));
            } else {
                // Every signal copy of the odd CTA lands before the CTAs leave. After a
                // complete run the MMA thread has waited for every stage; after a stop,
                // wait for the phases the odd CTA sent bytes to: this thread's last
                // arrival on each stage, and (armed here) the odd CTA's signals past them.
                if (ptx::mbar_wait_cluster(&S->sig_done, 0, kDrainBudget)) {
                    const long long fo = *reinterpret_cast<volatile long long*>(&S->sig_fills);
                    const long long first = fills > kTnStages ? fills - kTnStages : 0;
                    for (long long f = first; f < fills && f < fo; ++f)
                        ptx::mbar_wait(&S->bfull[f % kTnStages], (uint32_t)((f / kTnStages) & 1), kDrainBudget);
                    for (long long f = fills; f < fo; ++f) {
                        ptx::mbar_arrive_expect_tx(&S->bfull[f % kTnStages], 16u);
                        ptx::mbar_wait(&S->bfull[f % kTnStages], (uint32_t)((f / kTnStages) & 1), kDrainBudget);
                    }
                }
            }
        }
    } else if (kGather && warp >= kGatherWarp) {
        // ------------------------------------------------ row gather (MODE 3), warps 7..10 of both CTAs
        const int gt = threadIdx.x - kGatherWarp * 32;
        auto gsync = [] { asm volatile("bar.sync 1, %0;" ::"n"(kGatherThreads) : "memory"); };
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true, bad = false;
        for (int k = 0; ok; ++k) {
            if (gt == 0) {
                int4 item = make_int4(-2, 0, -1, -1);
                uint32_t valid = 0;
                const bool got = take_item(k, item, valid);
                if (got) release_item(k);
                S->g_item = got ? item : make_int4(-2, 0, -1, -1);
                S->g_valid = valid;
            }
            gsync();   // also: every thread is done with the previous item's g_tok
            const int4 item = S->g_item;
            const uint32_t valid = S->g_valid;
            if (item.x == -2) { ok = false; break; }
            if (item.x < 0) break;
            const int n = item_rows((int)(valid & 0xffffu), (int)(valid >> 16), item.w >= 0);
            const int brow = rank == 0 ? item.z : (item.w >= 0 ? item.w : item.z + n);
            for (int r = gt; r < n; r += kGatherThreads) {
                int t = __ldg(a.src_of + brow + r);
                if (t >= a.T) { bad = true; t = -1; }
                S->g_tok[r] = t;
            }
            gsync();
            // this thread's 16-byte chunks of the item, the same in every k-step: source row
            // (null for a padding row) and place in the B tile
            constexpr int kPer = 128 * 8 * kTnSlabs / kGatherThreads;
            const __nv_bfloat16* srcp[kPer];
            uint32_t dsto[kPer];
#pragma unroll
            for (int j = 0; j < kPer; ++j) {
                const int i = gt + j * kGatherThreads;
                const int r = i >> 4, sl = (i >> 3) & 1, c = i & 7;
                const int t = i < n * 16 ? S->g_tok[r] : -1;
                srcp[j] = t >= 0 ? a.x + (int64_t)t * a.d + sl * kBK + c * 8 : nullptr;
                dsto[j] = (uint32_t)((sl * n + r) * 128 + ((c ^ (r & 7)) << 4));
            }
            for (int kb = 0; kb < kb_count; ++kb) {
                if (gt == 0) S->g_ok = role_wait(&S->empty[stage], phase ^ 1, a.spin, abort_flag, a.header) ? 1 : 0;
                gsync();
                if (!S->g_ok) { ok = false; break; }
                // n rows x kTnSlabs slabs x 8 chunks of 16 bytes; slab sl of row r at
                // (sl*n + r)*128, chunk c at position c ^ (r % 8) (128-byte swizzle)
                const uint32_t bs = ptx::smem_addr(base + stage * kTnStageBytes + kTnBytesA);
#pragma unroll
                for (int j = 0; j < kPer; ++j)
                    if (srcp[j]) ptx::cp_async16(bs + dsto[j], srcp[j] + (int64_t)kb * kTnK);
                ptx::cp_async_mbar_arrive_noinc(&S->gfull[stage]);
                if (++stage == kTnStages) { stage = 0; phase ^= 1; }
            }
        }
        ptx::cp_async_commit();
        ptx::cp_async_wait<0>();   // nothing may land after the CTA leaves
        if (!ok && gt == 0) abort_pair();
        if (bad) set_status(a.header, MOE_DEV_BAD_INDEX);
    } else {
        // ------------------------------------------------ epilogue, warps 2..5 of both CTAs
        const int quad = warp & 3;                 // TMEM lanes 32*quad .. 32*quad+31
        float* stg = epi_base + quad * (kTnStg / 4);
        for (int k = 0;; ++k) {
            // lane 0 waits and the warp follows its outcome, so the lanes never part ways
            int4 item = make_int4(-1, 0, -1, -1);
            uint32_t valid = 0;
            int got = 0;
            if (lane == 0) got = take_item(k, item, valid) ? 1 : 0;
            if (!__shfl_sync(0xffffffffu, got, 0)) {
                if (lane == 0) abort_pair();
                break;
            }
            item.x = __shfl_sync(0xffffffffu, item.x, 0);
            item.y = __shfl_sync(0xffffffffu, item.y, 0);
            item.z = __shfl_sync(0xffffffffu, item.z, 0);
            item.w = __shfl_sync(0xffffffffu, item.w, 0);
            valid = __shfl_sync(0xffffffffu, valid, 0);
            if (lane == 0) release_item(k);
            if (item.x < 0) break;
            const int v0 = (int)(valid & 0xffffu), v1 = (int)(valid >> 16);
            const int n = item_rows(v0, v1, item.w >= 0);
            const int acc = k & 1;
            const uint32_t acc_phase = (uint32_t)((k >> 1) & 1);
            int full = 0;
            if (lane == 0) full = role_wait(&S->acc_full[acc], acc_phase, a.spin, abort_flag, a.header) ? 1 : 0;
            if (!__shfl_sync(0xffffffffu, full, 0)) {
                if (lane == 0) abort_pair();
                break;
            }
            __syncwarp();
            ptx::tc_fence_after();
            const uint32_t t_acc = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * kN);
            // FC1: h columns 128j + 64 rank + 16 quad ..; FC2: yp columns 256j + 128 rank + 32 quad ..
            const int col = kFC1 ? item.y * 128 + (int)rank * 64 + quad * 16 : item.y * 256 + (int)rank * 128 + quad * 32;
            for (int c0 = 0; c0 < 2 * n; c0 += 32)
                tn_chunk<kFC1>(t_acc, c0, lane, stg, a.out, a.ld_out, col, item.z, item.w, n, v0, v1);
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (even) ptx::mbar_arrive(&S->acc_empty[acc]);
                else ptx::mbar_arrive_cluster(ptx::map_to_rank(ptx::smem_addr(&S->acc_empty[acc]), 0));
            }
            // the accumulator is free: the next item's MMAs overlap the combine
            if (kFold) tn_fold_combine(a, lane, col, item.z, item.w, n, v0, v1);
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();   // no CTA leaves while its peer may still signal it
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc_pair(tmem, kTmemCols);
    }
}

// w_gate_up [E, 2F, d] as 5-D (64, 16, 2, E*F/8, d/64): dims 0 and 4 are a
// row's K position split into 64-column slabs (128 bytes apart), dim 1 the
// row inside a 16-row group, dim 3 the 16-row group over all experts, and
// dim 2 steps F rows, from a gate row to the up row of the same h column.
// One box of (64, 16, 2, 4, kTnSlabs) at group e*F/8 + c/16 brings h columns
// c .. c+63 as four groups of 16 gate rows followed by the 16 matching up
// rows, for kTnSlabs K slabs (slab after slab).
bool make_tmap_w1_groups(CUtensorMap* tm, const void* w, int E, int F, int d) {
    auto fn = encode_fn();
    if (!fn) return false;
    const uint64_t row = (uint64_t)d * 2;
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    cuuint64_t dims[5] = {(cuuint64_t)kBK, 16, 2, (cuuint64_t)E * F / 8, (cuuint64_t)d / kBK};
    cuuint64_t strides[4] = {row, (uint64_t)F * row, 16 * row, (uint64_t)kBK * 2};
    cuuint32_t box[5] = {(cuuint32_t)kBK, 16, 2, 4, (cuuint32_t)kTnSlabs};
    return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(w), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A row-major [rows, K] bf16 matrix as 3-D (64, row, K/64), box (64,
// box_rows, kTnSlabs): kTnSlabs 64-column slabs of box_rows rows, slab after
// slab, 128-byte swizzle.
bool make_tmap_slabs(CUtensorMap* tm, const void* p, uint64_t K, uint64_t rows, uint32_t box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)kBK, rows, K / kBK};
    cuuint64_t strides[2] = {K * 2, (cuuint64_t)kBK * 2};
    cuuint32_t box[3] = {(cuuint32_t)kBK, box_rows, (cuuint32_t)kTnSlabs};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(p), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// which = 1: FC1 + SwiGLU, xp [rows_cap, d] x w_gate_up -> h [rows_cap, F];
// which = 2: FC2, h [rows_cap, F] x w_down -> yp [rows_cap, d], and with
// fold also the weighted top-k sum of the yp rows into fold->y [T, d];
// which = 3: FC1 + SwiGLU with the token rows gathered from x [T, d].
cudaError_t launch_ffn_tn(const Shape& s, int which, const void* a_mat, const void* w, void* out,
                          const WsPtrs& ws, cudaStream_t st, long long spin_budget, const FoldArgs* fold) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    sms &= ~1;   // whole CTA pairs
    const bool gather = which == 3;
    const bool fc1 = which == 1 || gather;
    const int K = fc1 ? s.d : s.F;
    TnMaps maps;
    memset(&maps, 0, sizeof(maps));
    for (int m = 0; m < kTnMaps && !gather; ++m)
        if (!make_tmap_slabs(&maps.b[m], a_mat, (uint64_t)K, (uint64_t)s.rows_cap, 16u * (m + 1)))
            return cudaErrorInvalidValue;
    if (fc1 ? !make_tmap_w1_groups(&maps.w, w, s.E, s.F, s.d)
            : !make_tmap_slabs(&maps.w, w, (uint64_t)s.F, (uint64_t)s.E * s.d, 128))
        return cudaErrorInvalidValue;
    TnArgs a;
    a.Kdim = K;
    a.n_tiles = fc1 ? s.F / 128 : s.d / 256;
    a.d = s.d;
    a.F = s.F;
    a.E = s.E;
    a.ld_out = fc1 ? s.F : s.d;
    {
        const int64_t pair_bytes = (int64_t)2 * kBM * K * 2;   // token rows of one block pair
        const int64_t g = ((int64_t)32 << 20) / pair_bytes;
        a.group = (int)(g < 1 ? 1 : (g > (1 << 20) ? (1 << 20) : g));
    }
    a.spin = spin_budget;
    a.blocks = ws.blocks;
    a.sched = ws.sched;
    a.sched_off = ws.sched_off;
    a.header = ws.header;
    a.queue = ws.gemm_q + (fc1 ? 0 : 4);
    a.out = static_cast<__nv_bfloat16*>(out);
    a.K = s.K;
    a.T = s.T;
    a.rows_cap = s.rows_cap;
    a.row_of = ws.row_of;
    a.src_of = ws.src_of;
    a.topk_w = fold ? fold->topk_w : nullptr;
    a.arrivals = fold ? fold->arrivals : nullptr;
    a.y = fold ? static_cast<__nv_bfloat16*>(fold->y) : nullptr;
    a.x = gather ? static_cast<const __nv_bfloat16*>(a_mat) : nullptr;
    if (fold && (fc1 || !fold->topk_w || !fold->arrivals || !fold->y)) return cudaErrorInvalidValue;
    cudaError_t err;
    if (gather) {
        err = cudaFuncSetAttribute(ffn_tn_kernel<3>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kTnSmemBytes);
        if (err != cudaSuccess) return err;
        return launch_pdl(ffn_tn_kernel<3>, dim3(sms), dim3(kThreads + kGatherExtra), kTnSmemBytes, st, maps, a);
    }
    if (fc1) {
        err = cudaFuncSetAttribute(ffn_tn_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kTnSmemBytes);
        if (err != cudaSuccess) return err;
        return launch_pdl(ffn_tn_kernel<0>, dim3(sms), dim3(kThreads), kTnSmemBytes, st, maps, a);
    } else if (!fold) {
        err = cudaFuncSetAttribute(ffn_tn_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kTnSmemBytes);
        if (err != cudaSuccess) return err;
        return launch_pdl(ffn_tn_kernel<1>, dim3(sms), dim3(kThreads), kTnSmemBytes, st, maps, a);
    } else {
        err = cudaFuncSetAttribute(ffn_tn_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kTnSmemBytes);
        if (err != cudaSuccess) return err;
        return launch_pdl(ffn_tn_kernel<2>, dim3(sms), dim3(kThreads), kTnSmemBytes, st, maps, a);
    }
}

}  // namespace moe
