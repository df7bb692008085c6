// tc_common.cuh - what the tcgen05 grouped GEMMs (forward and backward) share:
// tile and ring sizes, the shared-memory control block, bounded role waits,
// the work queues, the block-pair decode, the SwiGLU helpers and tensor maps.
#pragma once

#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <mutex>

#include "common.cuh"
#include "ptx.cuh"

namespace moe {
namespace tc {

constexpr int kBM = 128, kBK = 64, kStages = 6, kThreads = 224;
constexpr int kN = 256;                        // accumulator columns per item (pair MMA N)
constexpr int kHalfN = 128;                    // weight rows each CTA of the pair holds
constexpr uint32_t kTmemCols = 2 * kN;         // two accumulators
constexpr int kABytes = kBM * kBK * 2;         // 16 KB
constexpr int kBBytes = kHalfN * kBK * 2;      // 16 KB
constexpr int kStageBytes = kABytes + kBBytes; // 32 KB
constexpr long long kDrainBudget = 2000000000LL;
constexpr int kItemSlots = 4;                  // ring of fetched, decoded work items (few: a short window keeps L2 reuse)
// Releases of an item slot. Even CTA: its TMA thread, MMA thread and 4
// epilogue warps arrive locally, and the odd CTA's forwarder arrives once for
// its CTA; odd CTA: its TMA thread and 4 epilogue warps arrive locally on the
// forwarder's barrier. Only the forwarder, which holds nothing in flight,
// makes the cluster-scope release: that release waits for the releasing
// thread's outstanding copies and MMAs, which costs the TMA and MMA threads
// about a microsecond per item when they make it themselves.
constexpr uint32_t kItemConsumers = 7;
constexpr uint32_t kOddConsumers = 5;
constexpr int kSchedWarp = 6;                  // scheduler (even CTA), forwarder (odd CTA)


struct Smem {
    uint64_t full[kStages], empty[kStages], acc_full[2], acc_empty[2], drain;
    uint64_t item_full[kItemSlots], item_empty[kItemSlots], fwd_empty[kItemSlots];
    int4 items[kItemSlots];   // expert (-1: no more work), column tile, first row of each CTA's block (-1: none)
    uint32_t valid[kItemSlots];   // valid rows of the even CTA's block (low 16 bits) and the odd CTA's (high)
    int32_t pair_idx[kItemSlots];  // fused FFN: the item's block pair, counting over all experts
    int32_t rows[kItemSlots][kBM];   // gathered FC1: token of each row of this CTA's block
    uint32_t tmem_base;
    int abort_flag;
};

// epilogue staging: two 32 x 32 bf16 tiles (2 KB) per epilogue warp, each
// written to global memory by one TMA store
constexpr int kEpiBuf = 32 * 32 * 2;
constexpr int kEpiBytes = 4 * 2 * kEpiBuf;
constexpr size_t kSmemBytes = 1024 /*align slack*/ + kStages * kStageBytes + kEpiBytes + sizeof(Smem) +
                              2 * sizeof(int32_t) * (kMaxE + 1);
static_assert(kSmemBytes <= 232448, "shared memory per CTA");

__device__ __forceinline__ bool role_wait(uint64_t* bar, uint32_t parity, long long budget,
                                          volatile int* abort_flag, uint32_t* header) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    for (;;) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > budget) {
            *abort_flag = 1;
            atomicOr(header + H_STATUS, (uint32_t)MOE_DEV_TIMEOUT);
            return false;
        }
    }
}

// As role_wait, acquiring at cluster scope (the item ring of the odd CTA is
// written by the even CTA).
__device__ __forceinline__ bool role_wait_cluster(uint64_t* bar, uint32_t parity, long long budget,
                                                  volatile int* abort_flag, uint32_t* header) {
    if (ptx::mbar_try_wait_cluster(bar, parity)) return true;
    const long long t0 = clock64();
    for (;;) {
        if (ptx::mbar_try_wait_cluster(bar, parity)) return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > budget) {
            *abort_flag = 1;
            atomicOr(header + H_STATUS, (uint32_t)MOE_DEV_TIMEOUT);
            return false;
        }
    }
}

// Next work item for a cluster of group g (0 or 1), or -1 when none is left:
// its own half of the list first, then the other half.
__device__ __forceinline__ int fetch_item(int32_t* queue, int g, int split, int n_items) {
    const int lo = g ? split : 0, hi = g ? n_items : split;
    const int i = atomicAdd(&queue[g], 1);
    if (lo + i < hi) return lo + i;
    const int lo2 = g ? 0 : split, hi2 = g ? split : n_items;
    const int i2 = atomicAdd(&queue[1 - g], 1);
    if (lo2 + i2 < hi2) return lo2 + i2;
    return -1;
}

// Work item -> (expert, its two blocks, column tile). Expert e owns items
// [n_tiles*p_off[e], n_tiles*p_off[e+1]), column tile major, then its block
// pairs in schedule order; b1 = -1 when the pair has one block.
__device__ __forceinline__ void decode_item(long long it, int n_tiles, const int32_t* s_off, const int32_t* p_off,
                                            int E, const int32_t* sched, int& e, int& b0, int& b1, int& j,
                                            int* pair = nullptr) {
    int lo = 0, hi = E;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if ((long long)n_tiles * p_off[mid] <= it) lo = mid; else hi = mid;
    }
    const int np = p_off[lo + 1] - p_off[lo];
    const int nb = s_off[lo + 1] - s_off[lo];
    const long long local = it - (long long)n_tiles * p_off[lo];
    j = (int)(local / np);
    const int q = (int)(local % np);
    e = lo;
    b0 = sched[s_off[lo] + 2 * q];
    b1 = 2 * q + 1 < nb ? sched[s_off[lo] + 2 * q + 1] : -1;
    if (pair) *pair = p_off[lo] + q;
}

// silu(a) = a / (1 + e^-a) with the fast reciprocal-based divide (the IEEE
// divide's range checks made the FC1 epilogue slower than the main loop it
// must hide behind); the result is rounded to bf16 right after.
__device__ __forceinline__ float silu(float a) { return __fdividef(a, 1.f + __expf(-a)); }

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// ---------------------------------------------------------------- tensor maps (host)

inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2D bf16 tensor map of a row-major [rows, inner] matrix, box [box_rows, 64].
inline bool make_tmap(CUtensorMap* tm, const void* ptr, uint64_t inner, uint64_t rows, uint32_t box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner * 2};
    cuuint32_t box[2] = {(cuuint32_t)kBK, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// The output (h or yp) as 32 x 32 tiles, unswizzled, for the epilogue's stores.
inline bool make_tmap_out(CUtensorMap* tm, void* ptr, uint64_t cols, uint64_t rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ptr, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// An fp32 output as 32-row x 16-column tiles, unswizzled, for the weight
// gradients' epilogue stores.
inline bool make_tmap_out_f32(CUtensorMap* tm, void* ptr, uint64_t cols, uint64_t rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 4};
    cuuint32_t box[2] = {16, 32};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, ptr, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace tc
}  // namespace moe
