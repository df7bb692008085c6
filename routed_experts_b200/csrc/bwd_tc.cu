// bwd_tc.cu - the backward grouped GEMMs of the expert FFN on the tcgen05
// tensor cores.
//
// [MegaFlux] "MegaFlux: Skew-Resilient MoE Megakernels via Pipelined Expert
// Replication", §3.2 'Backward': DGrad runs through W2 and then W1 over the
// routed token blocks, and WGrad forms each expert's weight gradients from
// its blocks; the partial gradients of an expert's replicas are reduced into
// one. On one GPU the replicas of an expert are row ranges of the same padded
// buffers, so WGrad walks all of an expert's blocks (owner and replica pieces
// alike, in schedule order) inside one accumulation: the reduction of the
// replica partials happens in TMEM, in a fixed order.
//
// MODE 0  DGrad through W2 and the SwiGLU derivative: dH = dY . W2_e, then
//         dA = dH * g * silu'(a), dG = dH * silu(a) -> dAG = [dA | dG]
// MODE 1  DGrad through W1: dXp = dAG . W1_e (W1_e = [W_gate; W_up], [2F, d])
// MODE 2  WGrad of W2: dW2_e = dY_e^T . h_e        [d, F], fp32
// MODE 3  WGrad of W1: dW1_e = dAG_e^T . xp_e      [2F, d], fp32
//
// The kernel is the forward GEMM's design (ffn_tc.cu: CTA pairs running
// 256 x 256 tcgen05.mma.cta_group::2 tiles, a 6-stage TMA ring, a scheduler
// warp with die-split dynamic queues, two TMEM accumulators, TMA-stored
// epilogue tiles, bounded waits) with operands that are not K-major: the
// weights in DGrad (W2_e read as [K = d, N = F], W1_e as [K = 2F, N = d]) and
// both activations in WGrad (K = token rows) are read in place as MN-major
// tiles (64-element, 128-byte slabs along M or N, 64 K rows each), so no
// operand is transposed in memory. DGrad items are (expert, block pair,
// 256-column tile) as in the forward; WGrad items are (expert, 256-row M
// tile, 256-column N tile) whose K loop runs over the expert's blocks, two
// 64-row k-steps per block.
#include <math.h>

#include "common.cuh"
#include "ptx.cuh"
#include "tc_common.cuh"

namespace moe {
namespace {

using namespace tc;

constexpr int kSlabBytes = 64 * kBK * 2;   // 64 elements along M or N x 64 K rows: 8 KB

struct BwdArgs {
    int E;
    int F;
    int Kdim;         // DGrad: the contraction length (d for MODE 0, 2F for MODE 1)
    int n_tiles;      // 256-column tiles of the output
    int m_pairs;      // WGrad: 256-row tiles of the output per expert
    int b_rows;       // DGrad: rows of one expert in the 2D weight view (d or 2F)
    int out_rows;     // WGrad: rows of one expert in the 2D gradient view (d or 2F)
    long long spin;
    const int32_t* blocks;
    const int32_t* sched;
    const int32_t* sched_off;
    uint32_t* header;
    int32_t* queue;
    const __nv_bfloat16* ag;   // MODE 0: the pre-activations [gate | up], [rows_cap, 2F]
};

__device__ __forceinline__ float sigmoidf_fast(float a) { return __fdividef(1.f, 1.f + __expf(-a)); }

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
bwd_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const __grid_constant__ CUtensorMap tmO, BwdArgs a) {
    constexpr bool kWgrad = MODE >= 2;
    constexpr bool kAmn = kWgrad;   // A stored M-contiguous
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
    if (warp == 0 && !kWgrad) {
        // pair offsets: p_off[e] = sum over e' < e of ceil(blocks(e') / 2)
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
    if (warp == 0 && lane == 0) { ptx::prefetch_tmap(&tmA); ptx::prefetch_tmap(&tmB); ptx::prefetch_tmap(&tmO); }
    __syncthreads();
    ptx::cluster_sync();   // the peer's barriers exist before any remote arrive, store or copy
    if (warp == 1) { ptx::tmem_alloc_pair(&S->tmem_base, kTmemCols); ptx::tmem_relinquish_pair(); }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = S->tmem_base;
    const int per_expert = a.m_pairs * a.n_tiles;
    const int n_items = kWgrad ? a.E * per_expert : p_off[a.E] * a.n_tiles;

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
    // k-steps of an item: DGrad a fixed contraction, WGrad two per block of the expert
    auto ksteps = [&](const int4& item) { return kWgrad ? 2 * item.w : a.Kdim / kBK; };

    if (warp == kSchedWarp) {
        // ------------------------------------------------ scheduler (even CTA) / forwarder (odd CTA)
        if (even) {
            const int g = ptx::smid() >= (ptx::nsmid() >> 1) ? 1 : 0;
            // split the expert-major list where half of the work (block pairs, or
            // blocks for WGrad) lies before
            int lo = 0, hi = a.E;
            const int* cum = kWgrad ? s_off : p_off;
            const int half = cum[a.E] / 2;
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (cum[mid] < half) lo = mid + 1; else hi = mid;
            }
            const int split = kWgrad ? lo * per_expert : p_off[lo] * a.n_tiles;
            int next = lane == 0 ? fetch_item(a.queue, g, split, n_items) : 0;
            for (int k = 0;; ++k) {
                const bool ok = role_wait_cluster(&S->item_empty[slot_of(k)], parity_of(k) ^ 1, a.spin, abort_flag, a.header);
                int4 item = make_int4(-1, 0, -1, -1);
                uint32_t valid = 0;
                if (lane == 0 && ok && next >= 0) {
                    if (kWgrad) {
                        // (expert, N tile, M tile, blocks of the expert)
                        const int e = next / per_expert, r = next % per_expert;
                        item = make_int4(e, r % a.n_tiles, r / a.n_tiles, s_off[e + 1] - s_off[e]);
                    } else {
                        int e, b0, b1, j;
                        decode_item(next, a.n_tiles, s_off, p_off, a.E, a.sched, e, b0, b1, j);
                        item = make_int4(e, j, a.blocks[kBlockInts * b0 + 1], b1 >= 0 ? a.blocks[kBlockInts * b1 + 1] : -1);
                        valid = (uint32_t)a.blocks[kBlockInts * b0 + 2] |
                                (b1 >= 0 ? (uint32_t)a.blocks[kBlockInts * b1 + 2] << 16 : 0u);
                    }
                }
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
            __syncwarp();
            if (lane == 0) release_item(k);
            if (item.x < 0) break;
            const int e = item.x, j = item.y;
            const int kb_count = ksteps(item);
            // B columns (N) this CTA holds: its 128 of the item's 256
            const int ncol = j * kN + (int)rank * kHalfN;
            int a_row = 0, b_row = 0, mcol = 0;
            int my_r0 = 0;   // WGrad: first row of block (32*chunk + lane) of the expert
            if (!kWgrad) {
                a_row = even ? item.z : (item.w >= 0 ? item.w : item.z);
                b_row = e * a.b_rows;
            } else {
                mcol = item.z * kN + (int)rank * kBM;
            }
            for (int kb = 0; kb < kb_count; ++kb) {
                int krow;   // WGrad: the token row this k-step starts at
                if (kWgrad) {
                    const int bi = kb >> 1;
                    if ((bi & 31) == 0 && (kb & 1) == 0) {
                        const int b = bi + lane;
                        my_r0 = b < item.w ? __ldg(a.blocks + kBlockInts * __ldg(a.sched + s_off[e] + b) + 1) : 0;
                    }
                    krow = __shfl_sync(0xffffffffu, my_r0, bi & 31) + (kb & 1) * kBK;
                }
                if (!role_wait(&S->empty[stage], phase ^ 1, a.spin, abort_flag, a.header)) { ok = false; break; }
                const uint32_t bar = ptx::map_to_rank(ptx::smem_addr(&S->full[stage]), 0);
                uint8_t* st = base + stage * kStageBytes;
                if (lane == 0) {
                    if (even) ptx::mbar_arrive_expect_tx(&S->full[stage], 2 * kStageBytes);
                    if (kWgrad) {
                        ptx::tma_load_2d_pair(st, &tmA, mcol, krow, bar);
                        ptx::tma_load_2d_pair(st + kSlabBytes, &tmA, mcol + 64, krow, bar);
                        ptx::tma_load_2d_pair(st + kABytes, &tmB, ncol, krow, bar);
                        ptx::tma_load_2d_pair(st + kABytes + kSlabBytes, &tmB, ncol + 64, krow, bar);
                    } else {
                        ptx::tma_load_2d_pair(st, &tmA, kb * kBK, a_row, bar);
                        ptx::tma_load_2d_pair(st + kABytes, &tmB, ncol, b_row + kb * kBK, bar);
                        ptx::tma_load_2d_pair(st + kABytes + kSlabBytes, &tmB, ncol + 64, b_row + kb * kBK, bar);
                    }
                }
                ++fills;
                if (++stage == kStages) { stage = 0; phase ^= 1; }
            }
        }
        if (!ok && even && lane == 0) {
            const long long first = fills > kStages ? fills - kStages : 0;
            for (long long f = first; f < fills; ++f)
                ptx::mbar_wait(&S->full[f % kStages], (uint32_t)((f / kStages) & 1), kDrainBudget);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (even CTA)
        if (lane == 0 && even) {
            const uint32_t idesc = ptx::idesc_bf16_f32_major(2 * kBM, kN, kAmn, true);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true, issued = false;
            for (int k = 0; ok; ++k) {
                int4 item;
                if (!take_item(k, item)) { ok = false; break; }
                release_item(k);
                if (item.x < 0) break;
                const int kb_count = ksteps(item);
                const int acc = k & 1;
                const uint32_t acc_phase = (uint32_t)((k >> 1) & 1);
                if (!role_wait_cluster(&S->acc_empty[acc], acc_phase ^ 1, a.spin, abort_flag, a.header)) { ok = false; break; }
                ptx::tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(acc * kN);
                for (int kb = 0; kb < kb_count; ++kb) {
                    if (!role_wait(&S->full[stage], phase, a.spin, abort_flag, a.header)) { ok = false; break; }
                    ptx::tc_fence_after();
                    const uint32_t a_addr = ptx::smem_addr(base + stage * kStageBytes);
                    const uint32_t b_addr = a_addr + kABytes;
#pragma unroll
                    for (int ks = 0; ks < kBK / 16; ++ks) {
                        const uint64_t da = kAmn ? ptx::sdesc_mn_sw128(a_addr + ks * 2048, kSlabBytes)
                                                 : ptx::sdesc_k_sw128(a_addr + ks * 32);
                        const uint64_t db = ptx::sdesc_mn_sw128(b_addr + ks * 2048, kSlabBytes);
                        ptx::mma_bf16_pair(d_tmem, da, db, idesc, (kb | ks) != 0 ? 1u : 0u);
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
                ptx::mma_commit_pair(ptx::smem_addr(&S->drain));
                ptx::mbar_wait(&S->drain, 0, kDrainBudget);
            }
        }
    } else {
        // ------------------------------------------------ epilogue, warps 2..5 of both CTAs
        const int quad = warp & 3;
        const int m = quad * 32 + lane;
        uint8_t* stg = epi_base + quad * 2 * kEpiBuf;
        int buf = 0;
        for (int k = 0;; ++k) {
            int4 item;
            if (!take_item(k, item)) break;
            const uint32_t vv = S->valid[slot_of(k)];
            __syncwarp();
            if (lane == 0) release_item(k);
            if (item.x < 0) break;
            const int acc = k & 1;
            const uint32_t acc_phase = (uint32_t)((k >> 1) & 1);
            const int j = item.y;
            // MODE 0: this row's pre-activations (gate at column f, up at F + f) are loaded a
            // chunk ahead of their use, the first chunk before the accumulator is ready
            uint4 av[4], gv[4];
            const __nv_bfloat16* ag_row = nullptr;
            if (MODE == 0) {
                const int row0 = even ? item.z : item.w;
                if (row0 >= 0) {
                    ag_row = a.ag + (int64_t)(row0 + m) * 2 * a.F + j * kN;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        av[q] = __ldg(reinterpret_cast<const uint4*>(ag_row) + q);
                        gv[q] = __ldg(reinterpret_cast<const uint4*>(ag_row + a.F) + q);
                    }
                }
            }
            if (!role_wait(&S->acc_full[acc], acc_phase, a.spin, abort_flag, a.header)) break;
            ptx::tc_fence_after();
            const uint32_t t_row = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * kN);
            if (kWgrad) {
                // fp32 gradient rows: expert e's row block of this CTA, 16-column stores
                const bool empty = item.w == 0;   // no rows routed to the expert: zero gradient
                const int orow = item.x * a.out_rows + item.z * kN + (int)rank * kBM + quad * 32;
#pragma unroll 1
                for (int c = 0; c < kN; c += 32) {
                    uint32_t v[32];
                    if (!empty) {
                        ptx::tmem_ld32(t_row + c, v);
                        ptx::tmem_ld_wait();
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] = 0u;
                    }
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if (lane == 0) ptx::bulk_wait_group_read<1>();
                        __syncwarp();
                        uint8_t* tile = stg + buf * kEpiBuf;
                        uint4* srow = reinterpret_cast<uint4*>(tile + lane * 64);   // 16 fp32
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            srow[q] = make_uint4(v[16 * h + 4 * q], v[16 * h + 4 * q + 1], v[16 * h + 4 * q + 2],
                                                 v[16 * h + 4 * q + 3]);
                        ptx::fence_proxy_async_shared();
                        __syncwarp();
                        if (lane == 0) {
                            ptx::tma_store_2d(&tmO, tile, j * kN + c + 16 * h, orow);
                            ptx::bulk_commit_group();
                        }
                        buf ^= 1;
                    }
                }
            } else {
                const int row0 = even ? item.z : item.w;   // -1: this CTA's half of the pair is empty
                const bool pad = m >= (int)(even ? (vv & 0xffffu) : (vv >> 16));
                if (row0 >= 0) {
#pragma unroll 1
                    for (int c = 0; c < kN; c += 32) {
                        uint32_t v[32];
                        ptx::tmem_ld32(t_row + c, v);
                        ptx::tmem_ld_wait();
                        if (MODE == 0) {
                            // SwiGLU derivative with this row's pre-activations a (gate) and g (up)
                            const int f0 = j * kN + c;
                            uint4 an[4], gn[4];
                            if (c + 32 < kN) {
#pragma unroll
                                for (int q = 0; q < 4; ++q) {
                                    an[q] = __ldg(reinterpret_cast<const uint4*>(ag_row + c + 32) + q);
                                    gn[q] = __ldg(reinterpret_cast<const uint4*>(ag_row + a.F + c + 32) + q);
                                }
                            }
                            const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(av);
                            const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(gv);
                            uint32_t pa[16], pg[16];
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                const float2 af = __bfloat1622float2(a2[i]);
                                const float2 gf = __bfloat1622float2(g2[i]);
                                const float d0 = __uint_as_float(v[2 * i]), d1 = __uint_as_float(v[2 * i + 1]);
                                const float s0 = sigmoidf_fast(af.x), s1 = sigmoidf_fast(af.y);
                                const float da0 = d0 * gf.x * (s0 * (1.f + af.x * (1.f - s0)));
                                const float da1 = d1 * gf.y * (s1 * (1.f + af.y * (1.f - s1)));
                                pa[i] = pad ? 0u : pack_bf16(da0, da1);
                                pg[i] = pad ? 0u : pack_bf16(d0 * (af.x * s0), d1 * (af.y * s1));
                            }
                            if (lane == 0) ptx::bulk_wait_group_read<0>();
                            __syncwarp();
                            uint4* sa = reinterpret_cast<uint4*>(stg + lane * 64);
                            uint4* sg = reinterpret_cast<uint4*>(stg + kEpiBuf + lane * 64);
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                sa[q] = make_uint4(pa[4 * q], pa[4 * q + 1], pa[4 * q + 2], pa[4 * q + 3]);
                                sg[q] = make_uint4(pg[4 * q], pg[4 * q + 1], pg[4 * q + 2], pg[4 * q + 3]);
                            }
                            ptx::fence_proxy_async_shared();
                            __syncwarp();
                            if (lane == 0) {
                                ptx::tma_store_2d(&tmO, stg, f0, row0 + quad * 32);
                                ptx::tma_store_2d(&tmO, stg + kEpiBuf, a.F + f0, row0 + quad * 32);
                                ptx::bulk_commit_group();
                            }
#pragma unroll
                            for (int q = 0; q < 4; ++q) { av[q] = an[q]; gv[q] = gn[q]; }
                        } else {
                            uint32_t pk[16];
#pragma unroll
                            for (int i = 0; i < 16; ++i)
                                pk[i] = pad ? 0u : pack_bf16(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
                            if (lane == 0) ptx::bulk_wait_group_read<1>();
                            __syncwarp();
                            uint8_t* tile = stg + buf * kEpiBuf;
                            uint4* srow = reinterpret_cast<uint4*>(tile + lane * 64);
#pragma unroll
                            for (int q = 0; q < 4; ++q) srow[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
                            ptx::fence_proxy_async_shared();
                            __syncwarp();
                            if (lane == 0) {
                                ptx::tma_store_2d(&tmO, tile, j * kN + c, row0 + quad * 32);
                                ptx::bulk_commit_group();
                            }
                            buf ^= 1;
                        }
                    }
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (even) ptx::mbar_arrive(&S->acc_empty[acc]);
                else ptx::mbar_arrive_cluster(ptx::map_to_rank(ptx::smem_addr(&S->acc_empty[acc]), 0));
            }
        }
        if (lane == 0) ptx::bulk_wait_group<0>();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc_pair(tmem, kTmemCols);
    }
}

template <int MODE>
cudaError_t launch_bwd_mode(const CUtensorMap& tA, const CUtensorMap& tB, const CUtensorMap& tO, const BwdArgs& a,
                            int grid, cudaStream_t st) {
    cudaError_t err = cudaFuncSetAttribute(bwd_tc_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)kSmemBytes);
    if (err != cudaSuccess) return err;
    bwd_tc_kernel<MODE><<<grid, kThreads, kSmemBytes, st>>>(tA, tB, tO, a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_tc(const Shape& s, int mode, const void* a_mat, const void* b_mat, void* out,
                          const void* ag, const WsPtrs& ws, cudaStream_t st, long long spin_budget) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    sms &= ~1;
    BwdArgs a{};
    a.E = s.E;
    a.F = s.F;
    a.spin = spin_budget;
    a.blocks = ws.blocks;
    a.sched = ws.sched;
    a.sched_off = ws.sched_off;
    a.header = ws.header;
    a.queue = ws.gemm_q;
    a.ag = static_cast<const __nv_bfloat16*>(ag);
    a.m_pairs = 1;
    CUtensorMap tA, tB, tO;
    const uint64_t rows = (uint64_t)s.rows_cap;
    switch (mode) {
        case 0:   // dY [rows, d] (K-major) x W2 [E*d (K), F (N)] -> dAG [rows, 2F]
            if (!make_tmap(&tA, a_mat, (uint64_t)s.d, rows, kBM) ||
                !make_tmap(&tB, b_mat, (uint64_t)s.F, (uint64_t)s.E * s.d, 64) ||
                !make_tmap_out(&tO, out, (uint64_t)2 * s.F, rows))
                return cudaErrorInvalidValue;
            a.Kdim = s.d;
            a.n_tiles = s.F / kN;
            a.b_rows = s.d;
            return launch_bwd_mode<0>(tA, tB, tO, a, sms, st);
        case 1:   // dAG [rows, 2F] (K-major) x W1 [E*2F (K), d (N)] -> dXp [rows, d]
            if (!make_tmap(&tA, a_mat, (uint64_t)2 * s.F, rows, kBM) ||
                !make_tmap(&tB, b_mat, (uint64_t)s.d, (uint64_t)s.E * 2 * s.F, 64) ||
                !make_tmap_out(&tO, out, (uint64_t)s.d, rows))
                return cudaErrorInvalidValue;
            a.Kdim = 2 * s.F;
            a.n_tiles = s.d / kN;
            a.b_rows = 2 * s.F;
            return launch_bwd_mode<1>(tA, tB, tO, a, sms, st);
        case 2:   // dY [rows (K), d (M)] x h [rows (K), F (N)] -> dW2 [E*d, F]
            if (!make_tmap(&tA, a_mat, (uint64_t)s.d, rows, 64) ||
                !make_tmap(&tB, b_mat, (uint64_t)s.F, rows, 64) ||
                !make_tmap_out_f32(&tO, out, (uint64_t)s.F, (uint64_t)s.E * s.d))
                return cudaErrorInvalidValue;
            a.m_pairs = s.d / kN;
            a.n_tiles = s.F / kN;
            a.out_rows = s.d;
            return launch_bwd_mode<2>(tA, tB, tO, a, sms, st);
        case 3:   // dAG [rows (K), 2F (M)] x xp [rows (K), d (N)] -> dW1 [E*2F, d]
            if (!make_tmap(&tA, a_mat, (uint64_t)2 * s.F, rows, 64) ||
                !make_tmap(&tB, b_mat, (uint64_t)s.d, rows, 64) ||
                !make_tmap_out_f32(&tO, out, (uint64_t)s.d, (uint64_t)s.E * 2 * s.F))
                return cudaErrorInvalidValue;
            a.m_pairs = 2 * s.F / kN;
            a.n_tiles = s.d / kN;
            a.out_rows = 2 * s.F;
            return launch_bwd_mode<3>(tA, tB, tO, a, sms, st);
        default:
            return cudaErrorInvalidValue;
    }
}

}  // namespace moe
