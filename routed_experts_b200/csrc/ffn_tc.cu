// ffn_tc.cu - the grouped SwiGLU expert FFN on the 5th-generation tensor cores
// (steps A7, A8 for bf16 layers) with the token rows as the MMA's M: a
// persistent, warp-specialised tcgen05 GEMM over the planned token blocks, run
// by CTA pairs, fed by TMA, accumulating in TMEM. It computes whole 128-row
// blocks, and serves the launches that need that: the training forward (which
// keeps the pre-activations and zero padding rows for the backward) and the
// fused FC1 -> FC2 launches. The layer's FC1 (also the one gathering x) and
// FC2 run on ffn_tn.cu, which covers each block's valid rows rounded up to 16
// instead.
//
// [MegaFlux] "MegaFlux: Skew-Resilient MoE Megakernels via Pipelined Expert
// Replication", §2.1 'Persistent MoE execution': persistent CTAs with
// warp-specialised workers (token movement, MMA, epilogue), tcgen05 MMA with
// fp32 accumulation in TMEM, operands staged by TMA, and two-CTA MMA; §3.1
// 'Problem formulation': the token blocks of the plan match the FC1/FC2 token
// tile (128 rows here); §3.2 'Forward': FC1 needs W1 and an input block, FC2
// needs W2 and the finished activation block.
//
// Work item = (two planned blocks of one expert, column tile), computed by a
// cluster of two CTAs on neighbouring SMs as one 256 x 256 MMA tile
// (tcgen05.mma.cta_group::2, M = 256, N = 256, K = 16): each CTA holds its own
// block's 128 activation rows and half (128 rows) of the weight tile in its
// shared memory, and receives its 128 rows of the accumulator in its own TMEM.
// So every CTA loads 32 KB per 64-deep k-step instead of 48 KB for a 128 x 256
// tile of its own. FC1 tiles are 128 gate columns (even CTA's weight half)
// plus the matching 128 up columns (odd CTA's half), so both halves of SwiGLU
// sit side by side in each CTA's accumulator; FC2 tiles are 256 columns of d.
// An expert with an odd number of blocks gives its last pair one block: the
// odd CTA then reloads the even CTA's rows and stores nothing. Rows of a
// block past its valid ones (padding) are stored as zero, whatever the
// activation rows held there.
//
// The fused launch with the dispatch folded in (mode 5) reads FC1's
// activation rows straight from x: each 128-row A tile is built by 32
// four-row TMA gathers (tile::gather4, one per lane of the TMA warp) of the
// token rows the plan's row map names; padding rows repeat the block's first
// token.
//
// Scheduling is dynamic. Items are listed expert-major (then column tile,
// then block pair), so consecutive items share an expert's weight tiles and a
// pair's activation rows. The list is cut at an expert boundary into two
// halves with a queue each (global atomic counters in the workspace); a
// cluster takes items from the queue of its half of the GPU (by the SM index
// of its even CTA) and steals from the other queue once its own is empty. The
// even CTA's TMA thread fetches each item and hands it to every consumer of
// both CTAs through a small ring in shared memory (a remote store plus a
// remote mbarrier arrive for the odd CTA). A scheduler warp of the even CTA
// fetches and decodes items several ahead (expert, column tile, first rows of
// both blocks), so no role waits on a global load at an item boundary. The
// last cluster to finish resets the counters for the next launch.
//
// CTA = 7 warps: warp 0 issues TMA loads into a 6-stage ring of 32 KB stages
// (128-byte swizzle), counted on the even CTA's "full" barrier; warp 6 of the
// even CTA fetches and decodes work items, warp 6 of the odd CTA hands its
// CTA's releases of item slots back to it; warp 1 of the
// even CTA issues the pair MMAs into one of two 256-column accumulators and
// commits to the "empty"/"full" barriers of both CTAs; warps 2-5 of each CTA
// drain the other accumulator (tcgen05.ld), apply the epilogue and store bf16
// rows, then arrive on the even CTA's "accumulator empty" barrier. Every wait
// is bounded: a wait that runs out sets MOE_DEV_TIMEOUT, raises the CTA's
// abort flag, lets its in-flight copies and MMAs finish and returns; both CTAs
// then meet at the cluster barrier and free TMEM.
#include <cudaTypedefs.h>
#include <math.h>

#include <mutex>

#include "common.cuh"
#include "ptx.cuh"
#include "tc_common.cuh"

namespace moe {
namespace {

using namespace tc;

struct TcArgs {
    const int32_t* src_of;    // row -> token (gathered FC1 only)
    int Kdim;                 // d or F
    int n_tiles;              // F/128 (FC1) or d/256 (FC2)
    int F;                    // FC1: row offset of the up projection inside an expert
    int b_rows;               // rows of one expert in the 2D weight view: 2F or d
    int E;
    long long spin;
    const int32_t* blocks;
    const int32_t* sched;
    const int32_t* sched_off;
    uint32_t* header;
    int32_t* queue;           // [3]: head of queue 0, head of queue 1, clusters finished
    int lone_apart;           // 1: experts with a single block are left to the single-CTA kernel
    // fused FFN (MODE 4): FC2's contraction length, column tiles and weight rows per expert, and
    // the per-pair counts of FC1 tiles stored
    int Kdim2, n_tiles2, b_rows2;
    int32_t* ready;
};

// The epilogue of one work item for one warp (rows 32*quad .. 32*quad+31 of
// the CTA's block): drain the accumulator at t_row 32 columns at a time,
// apply FC1's SwiGLU (MODE 0, 2, 3) or nothing (FC2), and store bf16 tiles
// through the warp's two staging tiles with TMA. MODE 3 first stores the
// pre-activations through tmP. Rows past the block's valid ones are zero.
template <int MODE>
__device__ __forceinline__ void epilogue_item(uint32_t t_row, int lane, int quad, uint8_t* stg, int& buf,
                                              const CUtensorMap* tmO, const CUtensorMap* tmP, int F, int j,
                                              int row0, bool pad) {
    constexpr bool kFC1 = MODE != 1;
    constexpr bool kPreact = MODE == 3;
    constexpr int kColTile = kFC1 ? 128 : 256;
#pragma unroll 1
    for (int c = 0; c < kColTile; c += 32) {
        uint32_t pk[16];
        if (kFC1) {
            uint32_t gt[32], up[32];
            ptx::tmem_ld32(t_row + c, gt);
            ptx::tmem_ld32(t_row + 128 + c, up);
            ptx::tmem_ld_wait();
            if (kPreact) {
                // the pre-activations first: gate at column j*128 + c, up at F + j*128 + c,
                // through both staging tiles
                uint32_t pg[16], pu[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    pg[i] = pad ? 0u : pack_bf16(__uint_as_float(gt[2 * i]), __uint_as_float(gt[2 * i + 1]));
                    pu[i] = pad ? 0u : pack_bf16(__uint_as_float(up[2 * i]), __uint_as_float(up[2 * i + 1]));
                }
                if (lane == 0) ptx::bulk_wait_group_read<0>();
                __syncwarp();
                uint4* sg = reinterpret_cast<uint4*>(stg + lane * 64);
                uint4* su = reinterpret_cast<uint4*>(stg + kEpiBuf + lane * 64);
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    sg[v] = make_uint4(pg[4 * v], pg[4 * v + 1], pg[4 * v + 2], pg[4 * v + 3]);
                    su[v] = make_uint4(pu[4 * v], pu[4 * v + 1], pu[4 * v + 2], pu[4 * v + 3]);
                }
                ptx::fence_proxy_async_shared();
                __syncwarp();
                if (lane == 0) {
                    ptx::tma_store_2d(tmP, stg, j * kColTile + c, row0 + quad * 32);
                    ptx::tma_store_2d(tmP, stg + kEpiBuf, F + j * kColTile + c, row0 + quad * 32);
                    ptx::bulk_commit_group();
                    ptx::bulk_wait_group_read<0>();   // both tiles free again for h below
                }
                __syncwarp();
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float h0 = silu(__uint_as_float(gt[2 * i])) * __uint_as_float(up[2 * i]);
                const float h1 = silu(__uint_as_float(gt[2 * i + 1])) * __uint_as_float(up[2 * i + 1]);
                pk[i] = pad ? 0u : pack_bf16(h0, h1);
            }
        } else {
            uint32_t y[32];
            ptx::tmem_ld32(t_row + c, y);
            ptx::tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i)
                pk[i] = pad ? 0u : pack_bf16(__uint_as_float(y[2 * i]), __uint_as_float(y[2 * i + 1]));
        }
        // this staging tile's previous store has finished reading it
        if (lane == 0) ptx::bulk_wait_group_read<1>();
        __syncwarp();
        uint8_t* tile = stg + buf * kEpiBuf;
        uint4* srow = reinterpret_cast<uint4*>(tile + lane * 64);   // row m: 32 bf16
#pragma unroll
        for (int v = 0; v < 4; ++v) srow[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        ptx::fence_proxy_async_shared();
        __syncwarp();
        if (lane == 0) {
            ptx::tma_store_2d(tmO, tile, j * kColTile + c, row0 + quad * 32);
            ptx::bulk_commit_group();
        }
        buf ^= 1;
    }
}

// MODE 0: FC1 + SwiGLU -> h (A = xp); MODE 1: FC2 -> yp (A = h);
// MODE 2: FC1 + SwiGLU -> h with A gathered from x;
// MODE 3: FC1 + SwiGLU -> h, also storing the pre-activations [gate | up]
// (rounded to bf16) for the backward's SwiGLU derivative (training forward);
// MODE 4: FC1 and FC2 in one launch (fused FFN): the work list holds every
// FC1 item, then every FC2 item (per half of the GPU); the scheduler hands
// out an FC2 item of a block pair only once all FC1 column tiles of that pair
// are stored (a per-pair count each epilogue warp raises with a release add
// after its TMA stores complete; bounded wait, acquire), so FC2 reads h while
// it is still in L2. tmA2 / tmB2 / tmO2 are FC2's operands and output;
// MODE 5: MODE 4 with FC1's A gathered from x as in MODE 2 (dispatch, FC1
// and FC2 in one launch).
template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
ffn_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmP,
              const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
              const __grid_constant__ CUtensorMap tmO2, TcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* epi_base = base + kStages * kStageBytes;
    Smem* S = reinterpret_cast<Smem*>(epi_base + kEpiBytes);
    int32_t* s_off = reinterpret_cast<int32_t*>(S + 1);
    int32_t* p_off = s_off + (a.E + 1);
    volatile int* abort_flag = &S->abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = ptx::cluster_ctarank();
    const bool even = rank == 0;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) { ptx::mbar_init(&S->full[s], 1); ptx::mbar_init(&S->empty[s], 1); }
        for (int q = 0; q < 2; ++q) { ptx::mbar_init(&S->acc_full[q], 1); ptx::mbar_init(&S->acc_empty[q], 8); }
        for (int q = 0; q < kItemSlots; ++q) {
            ptx::mbar_init(&S->item_full[q], 1);
            ptx::mbar_init(&S->item_empty[q], kItemConsumers);
            ptx::mbar_init(&S->fwd_empty[q], kOddConsumers);
        }
        ptx::mbar_init(&S->drain, 1);
        S->abort_flag = 0;
        ptx::fence_barrier_init();
    }
    for (int i = threadIdx.x; i <= a.E; i += kThreads) s_off[i] = a.sched_off[i];
    __syncthreads();
    if (warp == 0) {
        // pair offsets: p_off[e] = sum over e' < e of the pairs of e' (ceil(blocks / 2);
        // none for a one-block expert left to the single-CTA kernel)
        int carry = 0;
        if (lane == 0) p_off[0] = 0;
        for (int b = 0; b < a.E; b += 32) {
            const int i = b + lane;
            const int nb = i < a.E ? s_off[i + 1] - s_off[i] : 0;
            const int v = (a.lone_apart && nb == 1) ? 0 : (nb + 1) >> 1;
            int x = v;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, x, off);
                if (lane >= off) x += y;
            }
            if (i < a.E) p_off[i + 1] = carry + x;
            carry += __shfl_sync(0xffffffffu, x, 31);
        }
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tmap(&tmA);
        ptx::prefetch_tmap(&tmB);
        ptx::prefetch_tmap(&tmO);
        if (MODE == 3) ptx::prefetch_tmap(&tmP);
        if (MODE >= 4) { ptx::prefetch_tmap(&tmA2); ptx::prefetch_tmap(&tmB2); ptx::prefetch_tmap(&tmO2); }
    }
    __syncthreads();
    ptx::cluster_sync();   // the peer's barriers exist before any remote arrive, store or copy
    if (warp == 1) { ptx::tmem_alloc_pair(&S->tmem_base, kTmemCols); ptx::tmem_relinquish_pair(); }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = S->tmem_base;
    constexpr bool kFused = MODE == 4 || MODE == 5;
    const int n_items = p_off[a.E] * (a.n_tiles + (kFused ? a.n_tiles2 : 0));
    const int kb_count = a.Kdim / kBK;
    constexpr bool kGather = MODE == 2 || MODE == 5;   // FC1 items only
    // an item's phase (fused FFN: FC2 items carry it in the column field's bit 16)
    auto is_fc2 = [&](const int4& item) { return kFused ? (item.y >> 16) != 0 : MODE == 1; };

    // the ring slot of the k-th item, and the parity of its phase
    auto slot_of = [](int k) { return k % kItemSlots; };
    auto parity_of = [](int k) { return (uint32_t)((k / kItemSlots) & 1); };
    // take item k from the ring (both CTAs; the odd CTA's copy is written by
    // the even CTA's scheduler). Returns false when the wait gave up.
    auto take_item = [&](int k, int4& item) -> bool {
        const bool ok = even ? role_wait(&S->item_full[slot_of(k)], parity_of(k), a.spin, abort_flag, a.header)
                             : role_wait_cluster(&S->item_full[slot_of(k)], parity_of(k), a.spin, abort_flag, a.header);
        if (!ok) return false;
        item = S->items[slot_of(k)];
        return true;
    };
    // a local arrive (release at CTA scope) on this CTA's "slot empty" barrier
    auto release_item = [&](int k) { ptx::mbar_arrive(even ? &S->item_empty[slot_of(k)] : &S->fwd_empty[slot_of(k)]); };

    if (warp == kSchedWarp) {
        // ------------------------------------------------ scheduler (even CTA)
        if (even) {
            // group of this cluster: the half of the GPU its even CTA runs on
            const int g = ptx::smid() >= (ptx::nsmid() >> 1) ? 1 : 0;
            int lo = 0, hi = a.E;   // first expert whose pairs start at or after half of all pairs
            const int half = p_off[a.E] / 2;
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (p_off[mid] < half) lo = mid + 1; else hi = mid;
            }
            const int n_t = a.n_tiles + (kFused ? a.n_tiles2 : 0);   // items per block pair
            const int split = p_off[lo] * n_t;
            int next = lane == 0 ? fetch_item(a.queue, g, split, n_items) : 0;
            for (int k = 0;; ++k) {
                bool ok = role_wait_cluster(&S->item_empty[slot_of(k)], parity_of(k) ^ 1, a.spin, abort_flag, a.header);
                int4 item = make_int4(-1, 0, -1, -1);
                uint32_t valid = 0;
                int pair = 0;
                if (lane == 0 && ok && next >= 0) {
                    int e, b0, b1, j;
                    bool fc2 = false;
                    if (kFused) {
                        // this half's FC1 items, then its FC2 items
                        const int pb = next < split ? 0 : p_off[lo];              // first pair of the half
                        const int np = next < split ? p_off[lo] : p_off[a.E] - p_off[lo];
                        const int local = next < split ? next : next - split;
                        fc2 = local >= np * a.n_tiles;
                        const int idx = fc2 ? pb * a.n_tiles2 + (local - np * a.n_tiles) : pb * a.n_tiles + local;
                        decode_item(idx, fc2 ? a.n_tiles2 : a.n_tiles, s_off, p_off, a.E, a.sched, e, b0, b1, j, &pair);
                        if (fc2) {
                            // every FC1 tile of this pair stored (8 epilogue warps per FC1 item)
                            const int target = 8 * a.n_tiles;
                            const long long t0 = clock64();
                            while (ptx::ld_acquire_gpu(a.ready + pair) < target) {
                                if (*abort_flag) { ok = false; break; }
                                if (clock64() - t0 > a.spin) {
                                    *abort_flag = 1;
                                    atomicOr(a.header + H_STATUS, (uint32_t)MOE_DEV_TIMEOUT);
                                    ok = false;
                                    break;
                                }
                                __nanosleep(128);
                            }
                            ptx::fence_proxy_async_global();
                        }
                    } else {
                        decode_item(next, a.n_tiles, s_off, p_off, a.E, a.sched, e, b0, b1, j);
                    }
                    if (ok) {
                        item = make_int4(e, j | (fc2 ? 0x10000 : 0), a.blocks[kBlockInts * b0 + 1],
                                         b1 >= 0 ? a.blocks[kBlockInts * b1 + 1] : -1);
                        valid = (uint32_t)a.blocks[kBlockInts * b0 + 2] |
                                (b1 >= 0 ? (uint32_t)a.blocks[kBlockInts * b1 + 2] << 16 : 0u);
                    }
                }
                item.x = __shfl_sync(0xffffffffu, item.x, 0);
                item.y = __shfl_sync(0xffffffffu, item.y, 0);
                item.z = __shfl_sync(0xffffffffu, item.z, 0);
                item.w = __shfl_sync(0xffffffffu, item.w, 0);
                if (kGather && item.x >= 0 && (item.y >> 16) == 0) {
                    // tokens of the rows of both blocks; a padding row takes its block's first token
                    const int r_even = item.z, r_odd = item.w >= 0 ? item.w : item.z;
                    const int first_even = __ldg(a.src_of + r_even), first_odd = __ldg(a.src_of + r_odd);
                    int4 ve, vo;
                    ve.x = __ldg(a.src_of + r_even + 4 * lane + 0); vo.x = __ldg(a.src_of + r_odd + 4 * lane + 0);
                    ve.y = __ldg(a.src_of + r_even + 4 * lane + 1); vo.y = __ldg(a.src_of + r_odd + 4 * lane + 1);
                    ve.z = __ldg(a.src_of + r_even + 4 * lane + 2); vo.z = __ldg(a.src_of + r_odd + 4 * lane + 2);
                    ve.w = __ldg(a.src_of + r_even + 4 * lane + 3); vo.w = __ldg(a.src_of + r_odd + 4 * lane + 3);
                    ve.x = ve.x < 0 ? first_even : ve.x; vo.x = vo.x < 0 ? first_odd : vo.x;
                    ve.y = ve.y < 0 ? first_even : ve.y; vo.y = vo.y < 0 ? first_odd : vo.y;
                    ve.z = ve.z < 0 ? first_even : ve.z; vo.z = vo.z < 0 ? first_odd : vo.z;
                    ve.w = ve.w < 0 ? first_even : ve.w; vo.w = vo.w < 0 ? first_odd : vo.w;
                    *reinterpret_cast<int4*>(&S->rows[slot_of(k)][4 * lane]) = ve;
                    ptx::st_cluster_v4(ptx::map_to_rank(ptx::smem_addr(&S->rows[slot_of(k)][4 * lane]), 1), vo);
                    ptx::fence_acq_rel_cluster();
                }
                __syncwarp();
                if (lane == 0) {
                    // publish to both CTAs
                    S->items[slot_of(k)] = item;
                    S->valid[slot_of(k)] = valid;
                    S->pair_idx[slot_of(k)] = pair;
                    const uint32_t peer = ptx::map_to_rank(ptx::smem_addr(&S->items[slot_of(k)]), 1);
                    ptx::st_cluster_v4(peer, item);
                    ptx::st_cluster_u32(ptx::map_to_rank(ptx::smem_addr(&S->valid[slot_of(k)]), 1), valid);
                    if (kFused)
                        ptx::st_cluster_u32(ptx::map_to_rank(ptx::smem_addr(&S->pair_idx[slot_of(k)]), 1),
                                            (uint32_t)pair);
                    ptx::mbar_arrive(&S->item_full[slot_of(k)]);
                    ptx::mbar_arrive_cluster(ptx::map_to_rank(ptx::smem_addr(&S->item_full[slot_of(k)]), 1));
                }
                if (item.x < 0) break;
                if (lane == 0) next = fetch_item(a.queue, g, split, n_items);   // latency hides behind the ring
            }
            if (lane == 0) {
                // the last cluster to finish resets the queues for the next launch
                __threadfence();
                const int done = atomicAdd(&a.queue[2], 1);
                if (done == (int)ptx::cluster_count_x() - 1) {
                    a.queue[0] = 0;
                    a.queue[1] = 0;
                    if (kFused)   // every FC2 item was handed out, so every count is final
                        for (int q = 0; q < p_off[a.E]; ++q) a.ready[q] = 0;
                    __threadfence();
                    a.queue[2] = 0;
                }
            }
        } else if (lane == 0) {
            // forwarder (odd CTA): once this CTA's consumers have all released a
            // slot, release it to the even CTA's scheduler at cluster scope
            for (int k = 0;; ++k) {
                int4 item;
                if (!take_item(k, item)) break;
                if (!role_wait(&S->fwd_empty[slot_of(k)], parity_of(k), a.spin, abort_flag, a.header)) break;
                ptx::mbar_arrive_cluster(ptx::map_to_rank(ptx::smem_addr(&S->item_empty[slot_of(k)]), 0));
                if (item.x < 0) break;
            }
        }
    } else if (warp == 0) {
        // ------------------------------------------------ TMA producer (both CTAs, whole warp)
        int stage = 0;
        uint32_t phase = 0;
        long long fills = 0;
        bool ok = true;
        for (int k = 0; ok; ++k) {
            int4 item;
            if (!take_item(k, item)) { ok = false; break; }
            int4 tok = make_int4(0, 0, 0, 0);   // gathered FC1: tokens of this lane's four rows
            const bool gath = kGather && item.x >= 0 && (item.y >> 16) == 0;   // warp-uniform
            if (gath) tok = *reinterpret_cast<const int4*>(&S->rows[slot_of(k)][4 * lane]);
            __syncwarp();
            if (lane == 0) release_item(k);
            if (item.x < 0) break;
            const int e = item.x, j = item.y & 0xffff;
            const bool fc2 = is_fc2(item);
            const int row0 = even ? item.z : (item.w >= 0 ? item.w : item.z);
            const int brow = fc2 ? e * (kFused ? a.b_rows2 : a.b_rows) + j * kN + (even ? 0 : kHalfN)
                                 : e * a.b_rows + j * 128 + (even ? 0 : a.F);
            const CUtensorMap* mA = (kFused && fc2) ? &tmA2 : &tmA;
            const CUtensorMap* mB = (kFused && fc2) ? &tmB2 : &tmB;
            const int kbc = (kFused && fc2) ? a.Kdim2 / kBK : kb_count;
            if (kFused && fc2) ptx::fence_proxy_async_global();   // h was stored by other CTAs' TMA
            for (int kb = 0; kb < kbc; ++kb) {
                if (!role_wait(&S->empty[stage], phase ^ 1, a.spin, abort_flag, a.header)) { ok = false; break; }
                const uint32_t bar = ptx::map_to_rank(ptx::smem_addr(&S->full[stage]), 0);
                uint8_t* st = base + stage * kStageBytes;
                if (lane == 0) {
                    if (even) ptx::mbar_arrive_expect_tx(&S->full[stage], 2 * kStageBytes);
                    if (!gath) ptx::tma_load_2d_pair(st, mA, kb * kBK, row0, bar);
                    ptx::tma_load_2d_pair(st + kABytes, mB, kb * kBK, brow, bar);
                }
                if (gath) ptx::tma_gather4_pair(st + 4 * 128 * lane, &tmA, kb * kBK, tok.x, tok.y, tok.z, tok.w, bar);
                ++fills;
                if (++stage == kStages) { stage = 0; phase ^= 1; }
            }
        }
        if (!ok && even && lane == 0) {
            // let the copies still in flight land before the CTA exits
            const long long first = fills > kStages ? fills - kStages : 0;
            for (long long f = first; f < fills; ++f)
                ptx::mbar_wait(&S->full[f % kStages], (uint32_t)((f / kStages) & 1), kDrainBudget);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (even CTA)
        if (lane == 0 && even) {
            const uint32_t idesc = ptx::idesc_bf16_f32(2 * kBM, kN);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true, issued = false;
            for (int k = 0; ok; ++k) {
                int4 item;
                if (!take_item(k, item)) { ok = false; break; }
                release_item(k);
                if (item.x < 0) break;
                const int kbc = (kFused && is_fc2(item)) ? a.Kdim2 / kBK : kb_count;
                const int acc = k & 1;
                const uint32_t acc_phase = (uint32_t)((k >> 1) & 1);
                if (!role_wait_cluster(&S->acc_empty[acc], acc_phase ^ 1, a.spin, abort_flag, a.header)) { ok = false; break; }
                ptx::tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(acc * kN);
                for (int kb = 0; kb < kbc; ++kb) {
                    if (!role_wait(&S->full[stage], phase, a.spin, abort_flag, a.header)) { ok = false; break; }
                    ptx::tc_fence_after();
                    const uint32_t a_addr = ptx::smem_addr(base + stage * kStageBytes);
                    const uint32_t b_addr = a_addr + kABytes;
#pragma unroll
                    for (int ks = 0; ks < kBK / 16; ++ks) {
                        ptx::mma_bf16_pair(d_tmem, ptx::sdesc_k_sw128(a_addr + ks * 32),
                                           ptx::sdesc_k_sw128(b_addr + ks * 32), idesc, (kb | ks) != 0 ? 1u : 0u);
                    }
                    issued = true;
                    const uint32_t empty_addr = ptx::smem_addr(&S->empty[stage]);
                    ptx::mma_commit_pair(empty_addr);
                    ptx::mma_commit_pair(ptx::map_to_rank(empty_addr, 1));
                    if (++stage == kStages) { stage = 0; phase ^= 1; }
                }
                if (ok) {
                    const uint32_t full_addr = ptx::smem_addr(&S->acc_full[acc]);
                    ptx::mma_commit_pair(full_addr);
                    ptx::mma_commit_pair(ptx::map_to_rank(full_addr, 1));
                }
            }
            if (!ok && issued) {
                // wait for every MMA issued so far before TMEM is freed
                ptx::mma_commit_pair(ptx::smem_addr(&S->drain));
                ptx::mbar_wait(&S->drain, 0, kDrainBudget);
            }
        }
    } else {
        // ------------------------------------------------ epilogue, warps 2..5 of both CTAs
        const int quad = warp & 3;                 // TMEM lanes 32*quad .. 32*quad+31
        const int m = quad * 32 + lane;            // row inside this CTA's block
        uint8_t* stg = epi_base + quad * 2 * kEpiBuf;
        int buf = 0;
        for (int k = 0;; ++k) {
            int4 item;
            if (!take_item(k, item)) break;
            const uint32_t vv = S->valid[slot_of(k)];
            const int pidx = S->pair_idx[slot_of(k)];
            __syncwarp();
            if (lane == 0) release_item(k);
            if (item.x < 0) break;
            const int j = item.y & 0xffff;
            const bool fc2 = is_fc2(item);
            // rows of the block past its valid ones are padding: written as zero
            const bool pad = m >= (int)(even ? (vv & 0xffffu) : (vv >> 16));
            const int row0 = even ? item.z : item.w;   // -1: this CTA's half of the pair is empty
            const int acc = k & 1;
            const uint32_t acc_phase = (uint32_t)((k >> 1) & 1);
            if (!role_wait(&S->acc_full[acc], acc_phase, a.spin, abort_flag, a.header)) break;
            ptx::tc_fence_after();
            const uint32_t t_acc = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * kN);
            if (!kFused) {
                if (row0 >= 0) epilogue_item<MODE>(t_acc, lane, quad, stg, buf, &tmO, &tmP, a.F, j, row0, pad);
            } else if (fc2) {
                if (row0 >= 0) epilogue_item<1>(t_acc, lane, quad, stg, buf, &tmO2, &tmO2, a.F, j, row0, pad);
            } else {
                if (row0 >= 0) epilogue_item<0>(t_acc, lane, quad, stg, buf, &tmO, &tmO, a.F, j, row0, pad);
                // this warp's rows of the FC1 tile are in memory: count them for the pair
                if (lane == 0) {
                    ptx::bulk_wait_group<0>();
                    ptx::fence_proxy_async_global();
                    ptx::red_release_gpu_add(a.ready + pidx, 1);
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (even) ptx::mbar_arrive(&S->acc_empty[acc]);
                else ptx::mbar_arrive_cluster(ptx::map_to_rank(ptx::smem_addr(&S->acc_empty[acc]), 0));
            }
        }
        if (lane == 0) ptx::bulk_wait_group<0>();   // the stores are done before the CTA exits
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();   // no CTA leaves while its peer may still signal it
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc_pair(tmem, kTmemCols);
    }
    // launched as a dependent of the lone-block kernel before it, this kernel may
    // start while that one runs; it completes only after it, so the launches
    // that follow see every row of the output (a no-op for a plain launch)
    ptx::griddep_wait();
}

// ---------------------------------------------------------------- lone blocks
// An expert with a single planned block would run on a CTA pair beside an
// empty half. Those blocks run here instead, one CTA per item with
// tcgen05.mma.cta_group::1 (M = 128, N = 256; a kernel keeps to one
// CTA-group size): the CTA loads the block's 128 rows and both halves of the
// weight tile (256 rows), 48 KB per k-step, into a 4-stage ring, and the
// same epilogue stores the result. Warp roles as in the pair kernel (TMA,
// MMA, 4 epilogue warps, scheduler); items (lone block, column tile) come
// from one atomic queue. The odd last block of an expert with three or more
// blocks stays in the pair kernel: its weight tiles are in L2 while the
// expert's pairs run there, and a later launch would read them again from
// memory.
constexpr int kSStages = 4;
constexpr int kSStageBytes = kABytes + 2 * kBBytes;   // 48 KB
constexpr uint32_t kSItemConsumers = 6;               // TMA thread, MMA thread, 4 epilogue warps

struct SSmem {
    uint64_t full[kSStages], empty[kSStages], acc_full[2], acc_empty[2], drain;
    uint64_t item_full[kItemSlots], item_empty[kItemSlots];
    int4 items[kItemSlots];   // expert (-1: no more work), column tile, first row of the block, valid rows
    uint32_t tmem_base;
    int abort_flag;
};

constexpr size_t kSSmemBytes = 1024 /*align slack*/ + kSStages * kSStageBytes + kEpiBytes + sizeof(SSmem) +
                               2 * sizeof(int32_t) * (kMaxE + 1);
static_assert(kSSmemBytes <= 232448, "shared memory per CTA");

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
ffn_tc_single_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmP, TcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* epi_base = base + kSStages * kSStageBytes;
    SSmem* S = reinterpret_cast<SSmem*>(epi_base + kEpiBytes);
    int32_t* s_off = reinterpret_cast<int32_t*>(S + 1);
    int32_t* q_off = s_off + (a.E + 1);
    volatile int* abort_flag = &S->abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kSStages; ++s) { ptx::mbar_init(&S->full[s], 1); ptx::mbar_init(&S->empty[s], 1); }
        for (int q = 0; q < 2; ++q) { ptx::mbar_init(&S->acc_full[q], 1); ptx::mbar_init(&S->acc_empty[q], 4); }
        for (int q = 0; q < kItemSlots; ++q) {
            ptx::mbar_init(&S->item_full[q], 1);
            ptx::mbar_init(&S->item_empty[q], kSItemConsumers);
        }
        ptx::mbar_init(&S->drain, 1);
        S->abort_flag = 0;
        ptx::fence_barrier_init();
    }
    for (int i = threadIdx.x; i <= a.E; i += kThreads) s_off[i] = a.sched_off[i];
    // the pair kernel launched after this one may take every SM this one does not hold
    if (threadIdx.x == 0) ptx::griddep_launch_dependents();
    __syncthreads();
    if (warp == 0) {
        // q_off[e]: one-block experts before e
        int carry = 0;
        if (lane == 0) q_off[0] = 0;
        for (int b = 0; b < a.E; b += 32) {
            const int i = b + lane;
            int x = i < a.E && s_off[i + 1] - s_off[i] == 1 ? 1 : 0;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, x, off);
                if (lane >= off) x += y;
            }
            if (i < a.E) q_off[i + 1] = carry + x;
            carry += __shfl_sync(0xffffffffu, x, 31);
        }
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tmap(&tmA);
        ptx::prefetch_tmap(&tmB);
        ptx::prefetch_tmap(&tmO);
        if (MODE == 3) ptx::prefetch_tmap(&tmP);
    }
    __syncthreads();
    if (warp == 1) { ptx::tmem_alloc(&S->tmem_base, kTmemCols); ptx::tmem_relinquish(); }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = S->tmem_base;
    const int n_items = q_off[a.E] * a.n_tiles;
    const int kb_count = a.Kdim / kBK;
    constexpr bool kFC1 = MODE != 1;
    constexpr int kColTile = kFC1 ? 128 : 256;

    auto slot_of = [](int k) { return k % kItemSlots; };
    auto parity_of = [](int k) { return (uint32_t)((k / kItemSlots) & 1); };
    auto take_item = [&](int k, int4& item) -> bool {
        if (!role_wait(&S->item_full[slot_of(k)], parity_of(k), a.spin, abort_flag, a.header)) return false;
        item = S->items[slot_of(k)];
        return true;
    };
    auto release_item = [&](int k) { ptx::mbar_arrive(&S->item_empty[slot_of(k)]); };

    if (warp == kSchedWarp) {
        // ------------------------------------------------ scheduler
        if (lane == 0) {
            for (int k = 0;; ++k) {
                const bool ok = role_wait(&S->item_empty[slot_of(k)], parity_of(k) ^ 1, a.spin, abort_flag, a.header);
                const int it = ok ? atomicAdd(&a.queue[0], 1) : n_items;
                int4 item = make_int4(-1, 0, 0, 0);
                if (it < n_items) {
                    const int q = it / a.n_tiles, j = it % a.n_tiles;
                    int lo = 0, hi = a.E;   // the expert of lone block q: q_off[lo] <= q < q_off[lo + 1]
                    while (hi - lo > 1) {
                        const int mid = (lo + hi) >> 1;
                        if (q_off[mid] <= q) lo = mid; else hi = mid;
                    }
                    const int b = a.sched[s_off[lo]];   // the expert's only block
                    item = make_int4(lo, j, a.blocks[kBlockInts * b + 1], a.blocks[kBlockInts * b + 2]);
                }
                S->items[slot_of(k)] = item;
                ptx::mbar_arrive(&S->item_full[slot_of(k)]);
                if (item.x < 0) break;
            }
            // the last CTA to finish resets the queue for the next launch
            __threadfence();
            if (atomicAdd(&a.queue[1], 1) == (int)gridDim.x - 1) {
                a.queue[0] = 0;
                __threadfence();
                a.queue[1] = 0;
            }
        }
    } else if (warp == 0) {
        // ------------------------------------------------ TMA producer
        int stage = 0;
        uint32_t phase = 0;
        long long fills = 0;
        bool ok = true;
        for (int k = 0; ok; ++k) {
            int4 item;
            if (!take_item(k, item)) { ok = false; break; }
            __syncwarp();
            if (lane == 0) release_item(k);
            if (item.x < 0) break;
            const int e = item.x, j = item.y, row0 = item.z;
            // both halves of the weight tile: FC1 gate rows j*128.. and up rows F + j*128..,
            // FC2 rows j*256 .. j*256 + 255
            const int brow0 = e * a.b_rows + j * kColTile;
            const int brow1 = brow0 + (kFC1 ? a.F : kHalfN);
            for (int kb = 0; kb < kb_count; ++kb) {
                if (!role_wait(&S->empty[stage], phase ^ 1, a.spin, abort_flag, a.header)) { ok = false; break; }
                uint8_t* st = base + stage * kSStageBytes;
                if (lane == 0) {
                    ptx::mbar_arrive_expect_tx(&S->full[stage], kSStageBytes);
                    ptx::tma_load_2d(st, &tmA, kb * kBK, row0, &S->full[stage]);
                    ptx::tma_load_2d(st + kABytes, &tmB, kb * kBK, brow0, &S->full[stage]);
                    ptx::tma_load_2d(st + kABytes + kBBytes, &tmB, kb * kBK, brow1, &S->full[stage]);
                }
                ++fills;
                if (++stage == kSStages) { stage = 0; phase ^= 1; }
            }
        }
        if (!ok && lane == 0) {
            const long long first = fills > kSStages ? fills - kSStages : 0;
            for (long long f = first; f < fills; ++f)
                ptx::mbar_wait(&S->full[f % kSStages], (uint32_t)((f / kSStages) & 1), kDrainBudget);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = ptx::idesc_bf16_f32(kBM, kN);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true, issued = false;
            for (int k = 0; ok; ++k) {
                int4 item;
                if (!take_item(k, item)) { ok = false; break; }
                release_item(k);
                if (item.x < 0) break;
                const int acc = k & 1;
                const uint32_t acc_phase = (uint32_t)((k >> 1) & 1);
                if (!role_wait(&S->acc_empty[acc], acc_phase ^ 1, a.spin, abort_flag, a.header)) { ok = false; break; }
                ptx::tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(acc * kN);
                for (int kb = 0; kb < kb_count; ++kb) {
                    if (!role_wait(&S->full[stage], phase, a.spin, abort_flag, a.header)) { ok = false; break; }
                    ptx::tc_fence_after();
                    const uint32_t a_addr = ptx::smem_addr(base + stage * kSStageBytes);
                    const uint32_t b_addr = a_addr + kABytes;
#pragma unroll
                    for (int ks = 0; ks < kBK / 16; ++ks)
                        ptx::mma_bf16(d_tmem, ptx::sdesc_k_sw128(a_addr + ks * 32), ptx::sdesc_k_sw128(b_addr + ks * 32),
                                      idesc, (kb | ks) != 0 ? 1u : 0u);
                    issued = true;
                    ptx::mma_commit(&S->empty[stage]);
                    if (++stage == kSStages) { stage = 0; phase ^= 1; }
                }
                if (ok) ptx::mma_commit(&S->acc_full[acc]);
            }
            if (!ok && issued) {
                ptx::mma_commit(&S->drain);
                ptx::mbar_wait(&S->drain, 0, kDrainBudget);
            }
        }
    } else {
        // ------------------------------------------------ epilogue, warps 2..5
        const int quad = warp & 3;
        const int m = quad * 32 + lane;
        uint8_t* stg = epi_base + quad * 2 * kEpiBuf;
        int buf = 0;
        for (int k = 0;; ++k) {
            int4 item;
            if (!take_item(k, item)) break;
            __syncwarp();
            if (lane == 0) release_item(k);
            if (item.x < 0) break;
            const int acc = k & 1;
            const uint32_t acc_phase = (uint32_t)((k >> 1) & 1);
            if (!role_wait(&S->acc_full[acc], acc_phase, a.spin, abort_flag, a.header)) break;
            ptx::tc_fence_after();
            epilogue_item<MODE>(tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * kN), lane, quad, stg, buf,
                                &tmO, &tmP, a.F, item.y, item.z, m >= item.w);
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&S->acc_empty[acc]);
        }
        if (lane == 0) ptx::bulk_wait_group<0>();
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

// One CTA waits, through the same bounded wait as the GEMM's roles, on an
// mbarrier no thread ever arrives on; when the wait runs out it reports
// MOE_DEV_TIMEOUT in *status and returns.
__global__ void bounded_wait_probe_kernel(uint32_t* status, long long budget) {
    __shared__ uint64_t never;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        ptx::mbar_init(&never, 1);
        abort_flag = 0;
        ptx::fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) role_wait(&never, 0, budget, &abort_flag, status);
}

// The single-CTA kernel over the one-block experts (with its own queue
// words), then the pair kernel as its programmatic dependent: the lone
// kernel's CTAs that find no work leave at once and the pair kernel's
// clusters take their SMs, so the two run side by side. The gathered FC1 and
// the fused FFN keep every block in pairs and launch the pair kernel alone.
template <int MODE>
cudaError_t launch_mode(const CUtensorMap& tA, const CUtensorMap& tB, const CUtensorMap& tO, const CUtensorMap& tP,
                        TcArgs a, int grid, cudaStream_t st, int32_t* single_queue,
                        const CUtensorMap* t2 = nullptr) {
    constexpr bool kSingles = MODE != 2 && MODE != 4 && MODE != 5;
    a.lone_apart = kSingles ? 1 : 0;
    cudaError_t err = cudaFuncSetAttribute(ffn_tc_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)kSmemBytes);
    if (err != cudaSuccess) return err;
    const CUtensorMap& tA2 = t2 ? t2[0] : tA;
    const CUtensorMap& tB2 = t2 ? t2[1] : tB;
    const CUtensorMap& tO2 = t2 ? t2[2] : tO;
    if constexpr (!kSingles) {
        ffn_tc_kernel<MODE><<<grid, kThreads, kSmemBytes, st>>>(tA, tB, tO, tP, tA2, tB2, tO2, a);
        return cudaGetLastError();
    } else {
        err = cudaFuncSetAttribute(ffn_tc_single_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)kSSmemBytes);
        if (err != cudaSuccess) return err;
        TcArgs lone = a;
        lone.queue = single_queue;
        ffn_tc_single_kernel<MODE><<<grid, kThreads, kSSmemBytes, st>>>(tA, tB, tO, tP, lone);
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
        cudaLaunchConfig_t lc = {};
        lc.gridDim = dim3(grid);
        lc.blockDim = dim3(kThreads);
        lc.dynamicSmemBytes = kSmemBytes;
        lc.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        lc.attrs = attr;
        lc.numAttrs = 1;
        return cudaLaunchKernelEx(&lc, ffn_tc_kernel<MODE>, tA, tB, tO, tP, tA2, tB2, tO2, a);
    }
}

}  // namespace

cudaError_t launch_bounded_wait_probe(uint32_t* status, long long budget, cudaStream_t st) {
    bounded_wait_probe_kernel<<<1, 32, 0, st>>>(status, budget);
    return cudaGetLastError();
}

cudaError_t launch_ffn_tc(const Shape& s, int which, const void* a_mat, const void* w, void* out,
                          const WsPtrs& ws, cudaStream_t st, long long spin_budget, void* preact) {
    // FC1 + SwiGLU (which = 1) and FC2 (which = 2) run on the token-N kernel (ffn_tn.cu)
    if (which == 1 || which == 2 || which == 3) return launch_ffn_tn(s, which, a_mat, w, out, ws, st, spin_budget);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    sms &= ~1;   // whole CTA pairs
    TcArgs a;
    a.E = s.E;
    a.spin = spin_budget;
    a.blocks = ws.blocks;
    a.sched = ws.sched;
    a.sched_off = ws.sched_off;
    a.header = ws.header;
    a.queue = ws.gemm_q + (which == 2 ? 4 : 0);
    a.src_of = ws.src_of;
    CUtensorMap tA, tB, tO, tP;
    if (which == 4) {
        // FC1 + SwiGLU -> h [rows_cap, F], and the pre-activations -> preact [rows_cap, 2F]
        if (!preact || !make_tmap(&tA, a_mat, (uint64_t)s.d, (uint64_t)s.rows_cap, kBM) ||
            !make_tmap(&tB, w, (uint64_t)s.d, (uint64_t)s.E * 2 * s.F, kHalfN) ||
            !make_tmap_out(&tO, out, (uint64_t)s.F, (uint64_t)s.rows_cap) ||
            !make_tmap_out(&tP, preact, (uint64_t)2 * s.F, (uint64_t)s.rows_cap))
            return cudaErrorInvalidValue;
        a.Kdim = s.d;
        a.n_tiles = s.F / 128;
        a.F = s.F;
        a.b_rows = 2 * s.F;
        return launch_mode<3>(tA, tB, tO, tP, a, sms, st, ws.gemm_q + 8);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_ffn_fused(const Shape& s, const void* a_src, const void* w_gate_up, const void* w_down, void* h,
                             void* yp, const WsPtrs& ws, cudaStream_t st, long long spin_budget, bool gather) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    sms &= ~1;
    TcArgs a{};
    a.E = s.E;
    a.spin = spin_budget;
    a.blocks = ws.blocks;
    a.sched = ws.sched;
    a.sched_off = ws.sched_off;
    a.header = ws.header;
    a.queue = ws.gemm_q;
    a.src_of = ws.src_of;
    a.ready = ws.pair_ready;
    // FC1: xp [rows_cap, d] (or x [T, d] gathered through the row map) x w_gate_up [E*2F, d] -> h;
    // FC2: h [rows_cap, F] x w_down [E*d, F] -> yp
    CUtensorMap tA, tB, tO, t2[3];
    const bool a_ok = gather ? make_tmap(&tA, a_src, (uint64_t)s.d, (uint64_t)s.T, 1)
                             : make_tmap(&tA, a_src, (uint64_t)s.d, (uint64_t)s.rows_cap, kBM);
    if (!a_ok || !make_tmap(&tB, w_gate_up, (uint64_t)s.d, (uint64_t)s.E * 2 * s.F, kHalfN) ||
        !make_tmap_out(&tO, h, (uint64_t)s.F, (uint64_t)s.rows_cap) ||
        !make_tmap(&t2[0], h, (uint64_t)s.F, (uint64_t)s.rows_cap, kBM) ||
        !make_tmap(&t2[1], w_down, (uint64_t)s.F, (uint64_t)s.E * s.d, kHalfN) ||
        !make_tmap_out(&t2[2], yp, (uint64_t)s.d, (uint64_t)s.rows_cap))
        return cudaErrorInvalidValue;
    a.Kdim = s.d;
    a.n_tiles = s.F / 128;
    a.F = s.F;
    a.b_rows = 2 * s.F;
    a.Kdim2 = s.F;
    a.n_tiles2 = s.d / kN;
    a.b_rows2 = s.d;
    return gather ? launch_mode<5>(tA, tB, tO, tO, a, sms, st, nullptr, t2)
                  : launch_mode<4>(tA, tB, tO, tO, a, sms, st, nullptr, t2);
}

}  // namespace moe
