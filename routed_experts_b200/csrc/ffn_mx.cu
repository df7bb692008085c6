// ffn_mx.cu - the grouped SwiGLU expert FFN with MXFP8 operands on the
// block-scaled 5th-generation tensor cores (steps A7, A8 of the MX layer).
//
// [MegaFlux] "MegaFlux: Skew-Resilient MoE Megakernels via Pipelined Expert
// Replication", §2.1 'Persistent MoE execution': tcgen05 MMA with native
// block scaling (MXFP8 / MXFP4), fp32 accumulation in TMEM, two-CTA MMA,
// operands staged by TMA; §4.1 'Setup': the forward runs on MX operands with
// fp32 accumulation and bf16 outputs.
//
// The kernel is the bf16 pair kernel's schedule (ffn_tc.cu: persistent CTA
// pairs, work items = (two planned blocks of one expert, column tile) from
// two die-split queues, a scheduler warp feeding a 4-slot item ring, a
// TMA warp, an MMA warp and four epilogue warps per CTA, every wait bounded)
// with these differences:
//   - operands are E4M3 bytes: one 128-byte swizzled row holds 128 K
//     elements, so a k-step is 128 deep: four K = 32 slices of
//     tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale (M = 256);
//   - each k-step also brings the scale factors of its 128 A rows and 256 B
//     rows (512 bytes per 128 rows, already in the chunked layout of
//     mx_scale_offset) into a small ring beside the operand stages, on the
//     same TMA barrier; the MMA thread copies them to TMEM (tcgen05.cp
//     32x128b.warpx4, four columns per 128 rows) ahead of the k-step's MMAs,
//     alternating between two column sets;
//   - an item is 256 rows x 256 columns held in two 128-column TMEM
//     half-buffers. Three half-buffers rotate (item k takes buffers 2k mod 3
//     and 2k+1 mod 3) and the epilogue frees each half as soon as it has read
//     it, so the next item's MMAs wait only for the first half of the
//     previous item's epilogue; two full 256-column accumulators would leave
//     no TMEM for the scales. When the item's half-buffers are adjacent (two
//     items in three) one N = 256 MMA per K slice covers both and each CTA
//     holds 128 consecutive weight rows of the item; otherwise two N = 128
//     MMAs per K slice fill them and each CTA holds 64 rows of each half;
//   - FC1's weight rows are stored with every 128 rows of an expert holding
//     64 gate rows then the matching 64 up rows, so either way a half-buffer
//     holds [64 gate | 64 up] columns and is SwiGLU-complete: 64 h columns
//     per half, 128 per item. An FC2 item is 256 columns of d;
//   - the FC1 epilogue applies SwiGLU, rounds h to bf16 (FC1's bf16 output)
//     and quantizes it to MXFP8 along F right away: each thread holds 32
//     consecutive h values of its row, exactly one scale block, so the
//     block maximum needs no communication. Codes are stored by TMA (32 x 32
//     byte tiles), scales by plain byte stores into the chunked layout. FC2
//     stores bf16 yp as the bf16 kernel does.
// Weights may be MXFP4 instead ([MegaFlux] §4.1: MXFP4 weights, MXFP8
// activations): E2M1 codes packed two per byte in memory, which TMA unpacks
// (CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B) into the same 128-byte shared-memory
// rows, one element per byte; the MMA reads them as E2M1 (B format field)
// and the barrier counts the packed bytes.
// Experts with a single block run in a pair beside an empty half.
#include <cuda_fp8.h>
#include <cudaTypedefs.h>
#include <math.h>

#include "common.cuh"
#include "ptx.cuh"
#include "tc_common.cuh"

namespace moe {
namespace {

using namespace tc;

constexpr int kMxBK = 128;                                  // K elements (bytes) per slab
constexpr int kMxHalf = 128;                                // accumulator columns of one half-item MMA (N)
constexpr int kMxItemN = 2 * kMxHalf;                       // accumulator columns per item
constexpr int kMxHalfRows = 64;                             // weight rows each CTA holds per half
// A stage holds kMxSlabs 128-deep K slabs, each operand (and each scale
// operand) brought by one TMA copy covering all of them: the operand feed
// is paced by copies more than by bytes.
constexpr int kMxSlabs = 2;
constexpr int kMxStages = 6 / kMxSlabs;
constexpr int kMxSlabA = kBM * kMxBK;                       // 16 KB: 128 activation rows of one slab
constexpr int kMxSlabB = 2 * kMxHalfRows * kMxBK;           // 16 KB: the two halves' weight rows of one slab
constexpr int kMxABytes = kMxSlabs * kMxSlabA;
constexpr int kMxBBytes = kMxSlabs * kMxSlabB;
constexpr int kMxStageBytes = kMxABytes + kMxBBytes;
constexpr int kMxSfBytes = 512;                             // 128 rows x 4 scales of one slab
constexpr int kMxSfOp = kMxSlabs * kMxSfBytes;              // one scale operand's chunks of a stage
constexpr int kMxSfStage = 3 * kMxSfOp;                     // A, B of half 0, B of half 1
constexpr int kMxBufs = 3;                                  // 128-column TMEM half-buffers
constexpr uint32_t kMxTmemCols = 512;                       // allocation: a power of two >= 3*128 + 24
constexpr uint32_t kMxSfCol = kMxBufs * kMxHalf;            // two sets of 12 scale columns from here

// The control block: the bf16 kernel's, with one full / empty barrier pair
// per stage of this kernel's ring and per TMEM half-buffer.
struct MxSmem {
    uint64_t full[kMxStages], empty[kMxStages], hfull[kMxBufs], hempty[kMxBufs], drain;
    uint64_t item_full[kItemSlots], item_empty[kItemSlots], fwd_empty[kItemSlots];
    int4 items[kItemSlots];       // expert (-1: no more work), column tile, first row of each CTA's block (-1: none)
    uint32_t valid[kItemSlots];   // valid rows of the even CTA's block (low 16 bits) and the odd CTA's (high)
    uint32_t tmem_base;
    int abort_flag;
};

constexpr size_t kMxSmemBytes = 1024 /*align slack*/ + kMxStages * (kMxStageBytes + kMxSfStage) + kEpiBytes +
                                sizeof(MxSmem) + 2 * sizeof(int32_t) * (kMaxE + 1);
static_assert(kMxSmemBytes <= 232448, "shared memory per CTA");
static_assert(kMxStageBytes % 1024 == 0, "stages keep the 1024-byte alignment of swizzled tiles");

struct MxArgs {
    int Kdim;               // d (FC1) or F (FC2)
    int n_tiles;            // F/128 (FC1) or d/256 (FC2)
    int b_rows;             // rows of one expert in the weight matrix: 2F or d
    int E;
    int out_K;              // FC1: F, the row length of h (for its scale layout)
    long long spin;
    const int32_t* blocks;
    const int32_t* sched;
    const int32_t* sched_off;
    uint32_t* header;
    int32_t* queue;         // [3]: head of queue 0, head of queue 1, clusters finished
    uint8_t* out_sc;        // FC1: scales of h
};

__device__ __forceinline__ uint32_t mx_scale_of(float amax) {
    const uint32_t field = (__float_as_uint(amax) >> 23) & 0xFFu;
    return field > 8u ? field - 8u : 0u;
}

// The epilogue of one half-item for one warp (rows 32*quad .. 32*quad+31 of
// the CTA's block), reading the half-buffer at t_half. MODE 0: columns
// [0, 64) gate and [64, 128) up -> h codes of columns col0 .. col0+63 and
// their two scales; MODE 1: 128 columns -> bf16 yp columns col0 .. col0+127.
template <int MODE>
__device__ __forceinline__ void mx_epilogue_half(uint32_t t_half, int lane, int quad, uint8_t* stg, int& buf,
                                                 const CUtensorMap* tmO, const MxArgs& a, int col0, int row0,
                                                 bool pad) {
    if (MODE == 0) {
#pragma unroll 1
        for (int c = 0; c < kMxHalfRows; c += 32) {
            uint32_t gt[32], up[32];
            ptx::tmem_ld32(t_half + c, gt);
            ptx::tmem_ld32(t_half + kMxHalfRows + c, up);
            ptx::tmem_ld_wait();
            float h[32];
            float amax = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const float v = silu(__uint_as_float(gt[i])) * __uint_as_float(up[i]);
                h[i] = __bfloat162float(__float2bfloat16_rn(v));   // FC1's bf16 output
                amax = fmaxf(amax, fabsf(h[i]));
            }
            const uint32_t s = pad ? 0u : mx_scale_of(amax);
            const float inv = __uint_as_float((254u - s) << 23);
            uint32_t pk[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t lo = (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(h[4 * i] * inv, h[4 * i + 1] * inv),
                                                                       __NV_SATFINITE, __NV_E4M3);
                const uint32_t hi = (uint32_t)__nv_cvt_float2_to_fp8x2(
                    make_float2(h[4 * i + 2] * inv, h[4 * i + 3] * inv), __NV_SATFINITE, __NV_E4M3);
                pk[i] = pad ? 0u : (lo | (hi << 16));
            }
            if (lane == 0) ptx::bulk_wait_group_read<1>();
            __syncwarp();
            uint8_t* tile = stg + buf * kEpiBuf;
            uint4* srow = reinterpret_cast<uint4*>(tile + lane * 32);   // row m: 32 codes
            srow[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            srow[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            ptx::fence_proxy_async_shared();
            __syncwarp();
            if (lane == 0) {
                ptx::tma_store_2d(tmO, tile, col0 + c, row0 + quad * 32);
                ptx::bulk_commit_group();
            }
            buf ^= 1;
            const int64_t row = (int64_t)row0 + quad * 32 + lane;
            a.out_sc[mx_scale_offset(row, (col0 + c) / 32, a.out_K)] = (uint8_t)s;
        }
    } else {
#pragma unroll 1
        for (int c = 0; c < kMxHalf; c += 32) {
            uint32_t y[32];
            ptx::tmem_ld32(t_half + c, y);
            ptx::tmem_ld_wait();
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
                pk[i] = pad ? 0u : pack_bf16(__uint_as_float(y[2 * i]), __uint_as_float(y[2 * i + 1]));
            if (lane == 0) ptx::bulk_wait_group_read<1>();
            __syncwarp();
            uint8_t* tile = stg + buf * kEpiBuf;
            uint4* srow = reinterpret_cast<uint4*>(tile + lane * 64);   // row m: 32 bf16
#pragma unroll
            for (int v = 0; v < 4; ++v) srow[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
            ptx::fence_proxy_async_shared();
            __syncwarp();
            if (lane == 0) {
                ptx::tma_store_2d(tmO, tile, col0 + c, row0 + quad * 32);
                ptx::bulk_commit_group();
            }
            buf ^= 1;
        }
    }
}

// MODE 0: FC1 + SwiGLU -> MXFP8 h; MODE 1: FC2 -> bf16 yp. WF: the weights'
// element format (MOE_MX_W_E4M3 or MOE_MX_W_E2M1). tmA / tmB: the operands
// (128-byte swizzle); tmSA / tmSB: their chunked scales viewed as
// [chunks * 4, 128] bytes; tmO: the output.
template <int MODE, int WF>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
ffn_mx_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const __grid_constant__ CUtensorMap tmB2,
              const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB,
              const __grid_constant__ CUtensorMap tmO, MxArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sf_base = base + kMxStages * kMxStageBytes;          // the scale ring
    uint8_t* epi_base = sf_base + kMxStages * kMxSfStage;
    MxSmem* S = reinterpret_cast<MxSmem*>(epi_base + kEpiBytes);
    int32_t* s_off = reinterpret_cast<int32_t*>(S + 1);
    int32_t* p_off = s_off + (a.E + 1);
    volatile int* abort_flag = &S->abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = ptx::cluster_ctarank();
    const bool even = rank == 0;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kMxStages; ++s) { ptx::mbar_init(&S->full[s], 1); ptx::mbar_init(&S->empty[s], 1); }
        for (int q = 0; q < kMxBufs; ++q) { ptx::mbar_init(&S->hfull[q], 1); ptx::mbar_init(&S->hempty[q], 8); }
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
        // pair offsets: p_off[e] = sum over e' < e of ceil(blocks of e' / 2)
        int carry = 0;
        if (lane == 0) p_off[0] = 0;
        for (int b = 0; b < a.E; b += 32) {
            const int i = b + lane;
            const int v = i < a.E ? (s_off[i + 1] - s_off[i] + 1) >> 1 : 0;
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
        ptx::prefetch_tmap(&tmB2);
        ptx::prefetch_tmap(&tmSA);
        ptx::prefetch_tmap(&tmSB);
        ptx::prefetch_tmap(&tmO);
    }
    __syncthreads();
    ptx::cluster_sync();   // the peer's barriers exist before any remote arrive, store or copy
    if (warp == 1) { ptx::tmem_alloc_pair(&S->tmem_base, kMxTmemCols); ptx::tmem_relinquish_pair(); }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = S->tmem_base;
    const int n_items = p_off[a.E] * a.n_tiles;
    // stages per item: the last one holds a single slab when K / 128 is odd (its
    // copies still bring two, the second beyond K or unused, and no MMA reads it)
    const int n_slabs = a.Kdim / kMxBK;
    const int kb_count = (n_slabs + kMxSlabs - 1) / kMxSlabs;

    auto slot_of = [](int k) { return k % kItemSlots; };
    auto parity_of = [](int k) { return (uint32_t)((k / kItemSlots) & 1); };
    auto take_item = [&](int k, int4& item) -> bool {
        const bool ok = even ? role_wait(&S->item_full[slot_of(k)], parity_of(k), a.spin, abort_flag, a.header)
                             : role_wait_cluster(&S->item_full[slot_of(k)], parity_of(k), a.spin, abort_flag, a.header);
        if (!ok) return false;
        item = S->items[slot_of(k)];
        return true;
    };
    auto release_item = [&](int k) { ptx::mbar_arrive(even ? &S->item_empty[slot_of(k)] : &S->fwd_empty[slot_of(k)]); };

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
                int4 item = make_int4(-1, 0, -1, -1);
                uint32_t valid = 0;
                if (lane == 0 && ok && next >= 0) {
                    int e, b0, b1, j;
                    decode_item(next, a.n_tiles, s_off, p_off, a.E, a.sched, e, b0, b1, j);
                    item = make_int4(e, j, a.blocks[kBlockInts * b0 + 1], b1 >= 0 ? a.blocks[kBlockInts * b1 + 1] : -1);
                    valid = (uint32_t)a.blocks[kBlockInts * b0 + 2] |
                            (b1 >= 0 ? (uint32_t)a.blocks[kBlockInts * b1 + 2] << 16 : 0u);
                }
                __syncwarp();
                if (lane == 0) {
                    S->items[slot_of(k)] = item;
                    S->valid[slot_of(k)] = valid;
                    ptx::st_cluster_v4(ptx::map_to_rank(ptx::smem_addr(&S->items[slot_of(k)]), 1), item);
                    ptx::st_cluster_u32(ptx::map_to_rank(ptx::smem_addr(&S->valid[slot_of(k)]), 1), valid);
                    ptx::mbar_arrive(&S->item_full[slot_of(k)]);
                    ptx::mbar_arrive_cluster(ptx::map_to_rank(ptx::smem_addr(&S->item_full[slot_of(k)]), 1));
                }
                item.x = __shfl_sync(0xffffffffu, item.x, 0);
                if (item.x < 0) break;
                if (lane == 0) next = fetch_item(a.queue, g, split, n_items);
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
            // forwarder (odd CTA): once this CTA's consumers have released a slot,
            // release it to the even CTA's scheduler at cluster scope
            for (int k = 0;; ++k) {
                int4 item;
                if (!take_item(k, item)) break;
                if (!role_wait(&S->fwd_empty[slot_of(k)], parity_of(k), a.spin, abort_flag, a.header)) break;
                ptx::mbar_arrive_cluster(ptx::map_to_rank(ptx::smem_addr(&S->item_empty[slot_of(k)]), 0));
                if (item.x < 0) break;
            }
        }
    } else if (warp == 0) {
        // ------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            long long fills = 0;
            bool ok = true;
            const int kc = a.Kdim / 128;   // scale chunks per 128-row group
            for (int k = 0; ok; ++k) {
                int4 item;
                if (!take_item(k, item)) { ok = false; break; }
                release_item(k);
                if (item.x < 0) break;
                const int e = item.x, j = item.y;
                const int row0 = even ? item.z : (item.w >= 0 ? item.w : item.z);
                const int wrow = e * a.b_rows + j * kMxItemN;        // the item's first weight row
                // half-buffers 2k mod 3 and 2k+1 mod 3 are adjacent unless the first is the last:
                // then one N = 256 MMA reads 128 contiguous rows per CTA (CTA c: rows 128c ..),
                // brought by one 128-row copy; else two N = 128 MMAs read 64 rows of each half per
                // CTA (CTA c: rows 64c ..), brought by two 64-row copies
                const bool wide = (2 * k) % kMxBufs != kMxBufs - 1;
                const int b_lo = wrow + (wide ? (even ? 0 : kMxHalf) : (even ? 0 : kMxHalfRows));
                const int b_hi = b_lo + kMxHalf;
                const int a_chunk0 = (row0 / 128) * kc;
                const int b_chunk0 = (wrow / 128) * kc, b_chunk1 = (wrow / 128 + 1) * kc;
                for (int kb = 0; kb < kb_count; ++kb) {
                    if (!role_wait(&S->empty[stage], phase ^ 1, a.spin, abort_flag, a.header)) { ok = false; break; }
                    const uint32_t bar = ptx::map_to_rank(ptx::smem_addr(&S->full[stage]), 0);
                    uint8_t* st = base + stage * kMxStageBytes;
                    uint8_t* sf = sf_base + stage * kMxSfStage;
                    const int ks0 = kb * kMxSlabs;   // the stage's first K slab
                    // E2M1 weights count their packed bytes (half a byte per element)
                    if (even)
                        ptx::mbar_arrive_expect_tx(&S->full[stage],
                                                   2 * (kMxABytes + (WF == MOE_MX_W_E2M1 ? kMxBBytes / 2 : kMxBBytes) +
                                                        kMxSfStage));
                    ptx::tma_load_3d_pair(st, &tmA, 0, row0, ks0, bar);
                    if (wide) {
                        ptx::tma_load_3d_pair(st + kMxABytes, &tmB2, 0, b_lo, ks0, bar);
                    } else {
                        ptx::tma_load_3d_pair(st + kMxABytes, &tmB, 0, b_lo, ks0, bar);
                        ptx::tma_load_3d_pair(st + kMxABytes + kMxBBytes / 2, &tmB, 0, b_hi, ks0, bar);
                    }
                    ptx::tma_load_2d_pair(sf, &tmSA, 0, (a_chunk0 + ks0) * 4, bar);
                    ptx::tma_load_2d_pair(sf + kMxSfOp, &tmSB, 0, (b_chunk0 + ks0) * 4, bar);
                    ptx::tma_load_2d_pair(sf + 2 * kMxSfOp, &tmSB, 0, (b_chunk1 + ks0) * 4, bar);
                    ++fills;
                    if (++stage == kMxStages) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok && even) {
                // let the copies still in flight land before the CTA exits
                const long long first = fills > kMxStages ? fills - kMxStages : 0;
                for (long long f = first; f < fills; ++f)
                    ptx::mbar_wait(&S->full[f % kMxStages], (uint32_t)((f / kMxStages) & 1), kDrainBudget);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (even CTA)
        if (lane == 0 && even) {
            // B format field of the instruction descriptor (bits 10-12): E4M3 0, E2M1 5
            constexpr uint32_t kBFormat = WF == MOE_MX_W_E2M1 ? (5u << 10) : 0u;
            int stage = 0;
            uint32_t phase = 0, sf_set = 0;
            bool ok = true, issued = false;
            for (int k = 0; ok; ++k) {
                int4 item;
                if (!take_item(k, item)) { ok = false; break; }
                release_item(k);
                if (item.x < 0) break;
                // this item's half-buffers and how often each was used before
                const int s0 = 2 * k, s1 = 2 * k + 1;
                const int b0 = s0 % kMxBufs, b1 = s1 % kMxBufs;
                const uint32_t p0 = (uint32_t)((s0 / kMxBufs) & 1), p1 = (uint32_t)((s1 / kMxBufs) & 1);
                if (!role_wait_cluster(&S->hempty[b0], p0 ^ 1, a.spin, abort_flag, a.header) ||
                    !role_wait_cluster(&S->hempty[b1], p1 ^ 1, a.spin, abort_flag, a.header)) { ok = false; break; }
                ptx::tc_fence_after();
                const uint32_t d0 = tmem + (uint32_t)(b0 * kMxHalf), d1 = tmem + (uint32_t)(b1 * kMxHalf);
                const bool wide = b1 == b0 + 1;   // adjacent half-buffers: one N = 256 MMA per K slice
                for (int kb = 0; kb < kb_count; ++kb) {
                    if (!role_wait(&S->full[stage], phase, a.spin, abort_flag, a.header)) { ok = false; break; }
                    ptx::tc_fence_after();
                    const uint32_t a_stage = ptx::smem_addr(base + stage * kMxStageBytes);
                    const uint32_t b_stage = a_stage + kMxABytes;
                    const uint32_t sf_stage = ptx::smem_addr(sf_base + stage * kMxSfStage);
#pragma unroll
                    for (int sl = 0; sl < kMxSlabs; ++sl) {
                        if (kb * kMxSlabs + sl >= n_slabs) break;
                        // slab sl: activation rows at sl * 16 KB; weight rows: wide, 128 rows at
                        // sl * 16 KB; else the low half's 64 rows at sl * 8 KB and the high half's at
                        // kMxBBytes / 2 + sl * 8 KB; each scale operand's chunk at sl * 512 B
                        const uint32_t a_addr = a_stage + sl * kMxSlabA;
                        const uint32_t b_addr = wide ? b_stage + sl * kMxSlabB : b_stage + sl * (kMxSlabB / 2);
                        const uint32_t b_hi_addr = b_stage + kMxBBytes / 2 + sl * (kMxSlabB / 2);
                        const uint32_t sf_addr = sf_stage + sl * kMxSfBytes;
                        const uint32_t sfa_t = tmem + kMxSfCol + 12u * sf_set;
                        ptx::tmem_cp_sf_pair(sfa_t, ptx::sdesc_sf(sf_addr));
                        ptx::tmem_cp_sf_pair(sfa_t + 4u, ptx::sdesc_sf(sf_addr + kMxSfOp));
                        ptx::tmem_cp_sf_pair(sfa_t + 8u, ptx::sdesc_sf(sf_addr + 2 * kMxSfOp));
                        const int kk = kb * kMxSlabs + sl;   // K slab index: the first one starts the accumulation
                        if (wide) {
                            // one N = 256 MMA per K slice over both half-buffers (d1 = d0 + 128); its
                            // B scales are the 8 columns from sfa_t + 4 (rows 0-127, then 128-255)
#pragma unroll
                            for (uint32_t ks = 0; ks < kMxBK / 32; ++ks)
                                ptx::mma_mx_pair(d0, ptx::sdesc_k_sw128(a_addr + ks * 32),
                                                 ptx::sdesc_k_sw128(b_addr + ks * 32),
                                                 ptx::idesc_mx_e4m3(2 * kBM, kMxItemN, ks, ks) | kBFormat,
                                                 sfa_t | (ks << 30), (sfa_t + 4u) | (ks << 30),
                                                 (kk | (int)ks) != 0 ? 1u : 0u);
                        } else {
#pragma unroll
                            for (uint32_t ks = 0; ks < kMxBK / 32; ++ks) {
                                const uint32_t idesc = ptx::idesc_mx_e4m3(2 * kBM, kMxHalf, ks, ks) | kBFormat;
                                const uint32_t acc = (kk | (int)ks) != 0 ? 1u : 0u;
                                const uint64_t adesc = ptx::sdesc_k_sw128(a_addr + ks * 32);
                                ptx::mma_mx_pair(d0, adesc, ptx::sdesc_k_sw128(b_addr + ks * 32), idesc,
                                                 sfa_t | (ks << 30), (sfa_t + 4u) | (ks << 30), acc);
                                ptx::mma_mx_pair(d1, adesc, ptx::sdesc_k_sw128(b_hi_addr + ks * 32), idesc,
                                                 sfa_t | (ks << 30), (sfa_t + 8u) | (ks << 30), acc);
                            }
                        }
                        sf_set ^= 1u;
                    }
                    issued = true;
                    const uint32_t empty_addr = ptx::smem_addr(&S->empty[stage]);
                    ptx::mma_commit_pair(empty_addr);
                    ptx::mma_commit_pair(ptx::map_to_rank(empty_addr, 1));
                    if (++stage == kMxStages) { stage = 0; phase ^= 1; }
                }
                if (ok) {
                    const uint32_t f0 = ptx::smem_addr(&S->hfull[b0]), f1 = ptx::smem_addr(&S->hfull[b1]);
                    ptx::mma_commit_pair(f0);
                    ptx::mma_commit_pair(ptx::map_to_rank(f0, 1));
                    ptx::mma_commit_pair(f1);
                    ptx::mma_commit_pair(ptx::map_to_rank(f1, 1));
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
            __syncwarp();
            if (lane == 0) release_item(k);
            if (item.x < 0) break;
            const int j = item.y;
            const bool pad = m >= (int)(even ? (vv & 0xffffu) : (vv >> 16));
            const int row0 = even ? item.z : item.w;   // -1: this CTA's half of the pair is empty
            bool ok = true;
            for (int half = 0; half < 2 && ok; ++half) {
                const int sl = 2 * k + half;
                const int b = sl % kMxBufs;
                const uint32_t par = (uint32_t)((sl / kMxBufs) & 1);
                if (!role_wait(&S->hfull[b], par, a.spin, abort_flag, a.header)) { ok = false; break; }
                ptx::tc_fence_after();
                const uint32_t t_half = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(b * kMxHalf);
                const int col0 = MODE == 0 ? j * 2 * kMxHalfRows + half * kMxHalfRows : j * kMxItemN + half * kMxHalf;
                if (row0 >= 0) mx_epilogue_half<MODE>(t_half, lane, quad, stg, buf, &tmO, a, col0, row0, pad);
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (even) ptx::mbar_arrive(&S->hempty[b]);
                    else ptx::mbar_arrive_cluster(ptx::map_to_rank(ptx::smem_addr(&S->hempty[b]), 0));
                }
            }
            if (!ok) break;
        }
        if (lane == 0) ptx::bulk_wait_group<0>();   // the stores are done before the CTA exits
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();   // no CTA leaves while its peer may still signal it
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc_pair(tmem, kMxTmemCols);
    }
}

// A 2D byte matrix [rows, inner] with a box of [box_rows, box_inner] bytes.
bool make_tmap_u8(CUtensorMap* tm, const void* ptr, uint64_t inner, uint64_t rows, uint32_t box_inner,
                  uint32_t box_rows, bool swizzle128) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    swizzle128 ? CU_TENSOR_MAP_L2_PROMOTION_L2_256B : CU_TENSOR_MAP_L2_PROMOTION_NONE,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// An E4M3 code matrix [rows, K] as 3-D (128, row, K/128 slab), box (128,
// box_rows, kMxSlabs): kMxSlabs 128-byte K slabs of box_rows rows, slab
// after slab, 128-byte swizzle.
bool make_tmap_slabs_u8(CUtensorMap* tm, const void* ptr, uint64_t K, uint64_t rows, uint32_t box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)kMxBK, rows, K / kMxBK};
    cuuint64_t strides[2] = {K, (cuuint64_t)kMxBK};
    cuuint32_t box[3] = {(cuuint32_t)kMxBK, box_rows, (cuuint32_t)kMxSlabs};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Packed E2M1 codes [rows, K elements] (K / 2 bytes per row) as 3-D (128,
// row, K/128 slab), box (128, box_rows, kMxSlabs) elements, unpacked to one
// byte each in shared memory, 128-byte swizzle.
bool make_tmap_e2m1(CUtensorMap* tm, const void* ptr, uint64_t K, uint64_t rows, uint32_t box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)kMxBK, rows, K / kMxBK};
    cuuint64_t strides[2] = {K / 2, (cuuint64_t)kMxBK / 2};
    cuuint32_t box[3] = {(cuuint32_t)kMxBK, box_rows, (cuuint32_t)kMxSlabs};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int MODE, int WF>
cudaError_t launch_one(const CUtensorMap& tA, const CUtensorMap& tB, const CUtensorMap& tB2, const CUtensorMap& tSA,
                       const CUtensorMap& tSB, const CUtensorMap& tO, const MxArgs& a, int grid, cudaStream_t st) {
    cudaError_t err = cudaFuncSetAttribute(ffn_mx_kernel<MODE, WF>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)kMxSmemBytes);
    if (err != cudaSuccess) return err;
    ffn_mx_kernel<MODE, WF><<<grid, kThreads, kMxSmemBytes, st>>>(tA, tB, tB2, tSA, tSB, tO, a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ffn_mx(const Shape& s, int which, const uint8_t* a_q, const uint8_t* a_sc, const uint8_t* w_q,
                          const uint8_t* w_sc, int wfmt, void* out, uint8_t* out_sc, const WsPtrs& ws,
                          cudaStream_t st, long long spin_budget) {
    if (s.d % 256 != 0 || s.F % 128 != 0) return cudaErrorInvalidValue;
    if (wfmt != MOE_MX_W_E4M3 && wfmt != MOE_MX_W_E2M1) return cudaErrorInvalidValue;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    sms &= ~1;   // whole CTA pairs
    const bool fc1 = which == 1;
    MxArgs a;
    a.Kdim = fc1 ? s.d : s.F;
    a.n_tiles = fc1 ? s.F / (2 * kMxHalfRows) : s.d / kMxItemN;
    a.b_rows = fc1 ? 2 * s.F : s.d;
    a.E = s.E;
    a.out_K = s.F;
    a.spin = spin_budget;
    a.blocks = ws.blocks;
    a.sched = ws.sched;
    a.sched_off = ws.sched_off;
    a.header = ws.header;
    a.queue = ws.gemm_q;
    a.out_sc = out_sc;
    const uint64_t rows_a = (uint64_t)s.rows_cap;
    const uint64_t rows_b = (uint64_t)s.E * a.b_rows;
    const uint64_t chunks_a = (uint64_t)((s.rows_cap + 127) / 128) * (a.Kdim / 128);
    const uint64_t chunks_b = rows_b / 128 * (a.Kdim / 128);
    CUtensorMap tA, tB, tB2, tSA, tSB, tO;
    const bool e2m1 = wfmt == MOE_MX_W_E2M1;
    const bool b_ok = e2m1 ? make_tmap_e2m1(&tB, w_q, (uint64_t)a.Kdim, rows_b, kMxHalfRows) &&
                                 make_tmap_e2m1(&tB2, w_q, (uint64_t)a.Kdim, rows_b, kMxHalf)
                           : make_tmap_slabs_u8(&tB, w_q, (uint64_t)a.Kdim, rows_b, kMxHalfRows) &&
                                 make_tmap_slabs_u8(&tB2, w_q, (uint64_t)a.Kdim, rows_b, kMxHalf);
    // scales: a stage's kMxSlabs consecutive 512-byte chunks of each operand in one copy
    if (!make_tmap_slabs_u8(&tA, a_q, (uint64_t)a.Kdim, rows_a, kBM) || !b_ok ||
        !make_tmap_u8(&tSA, a_sc, 128, chunks_a * 4, 128, 4 * kMxSlabs, false) ||
        !make_tmap_u8(&tSB, w_sc, 128, chunks_b * 4, 128, 4 * kMxSlabs, false))
        return cudaErrorInvalidValue;
    const bool out_ok = fc1 ? make_tmap_u8(&tO, out, (uint64_t)s.F, rows_a, 32, 32, false)
                            : make_tmap_out(&tO, out, (uint64_t)s.d, rows_a);
    if (!out_ok) return cudaErrorInvalidValue;
    if (wfmt == MOE_MX_W_E2M1)
        return fc1 ? launch_one<0, MOE_MX_W_E2M1>(tA, tB, tB2, tSA, tSB, tO, a, sms, st)
                   : launch_one<1, MOE_MX_W_E2M1>(tA, tB, tB2, tSA, tSB, tO, a, sms, st);
    return fc1 ? launch_one<0, MOE_MX_W_E4M3>(tA, tB, tB2, tSA, tSB, tO, a, sms, st)
               : launch_one<1, MOE_MX_W_E4M3>(tA, tB, tB2, tSA, tSB, tO, a, sms, st);
}

}  // namespace moe
