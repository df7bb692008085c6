// ffn_tc.cu - the grouped SwiGLU expert FFN on the 5th-generation tensor cores
// (steps A7, A8 for bf16 layers): a persistent, warp-specialised tcgen05 GEMM
// over the planned token blocks, fed by TMA, accumulating in TMEM.
//
// [MegaFlux] "MegaFlux: Skew-Resilient MoE Megakernels via Pipelined Expert
// Replication", §2.1 'Persistent MoE execution': persistent CTAs with
// warp-specialised workers (token movement, MMA, epilogue), tcgen05 MMA with
// fp32 accumulation in TMEM, operands staged by TMA; §3.1 'Problem
// formulation': the token blocks of the plan match the FC1/FC2 token tile
// (128 rows here); §3.2 'Forward': FC1 needs W1 and an input block, FC2 needs
// W2 and the finished activation block.
//
// Work item = (planned block of one expert, column tile). FC1 tiles are 128
// gate columns plus the matching 128 up columns, computed as one 128x256 MMA
// tile so the SwiGLU epilogue has both halves in one TMEM accumulator
// (gate+up fused in one pass over the A tile); FC2 tiles are 256 columns of
// d. Items are ordered expert-major (then column tile, then block), so the
// CTAs running at one time share a few experts' weight tiles in L2, and a
// block's activation rows are reused across its expert's column tiles.
//
// CTA = 6 warps: warp 0 issues TMA loads into a 4-stage ring (A 128x64 and
// B 256x64 bf16 per stage, 128-byte swizzle); warp 1 allocates 512 TMEM
// columns and one thread issues tcgen05.mma (M=128, N=256, K=16) into one of
// two accumulators; warps 2-5 drain the other accumulator (tcgen05.ld), apply
// the epilogue and store bf16 rows, so epilogue and MMA overlap. Every wait is
// bounded: a wait that runs out sets MOE_DEV_TIMEOUT, raises a CTA-wide abort
// flag, lets in-flight copies and MMAs finish, frees TMEM and returns.
#include <cudaTypedefs.h>
#include <math.h>

#include <mutex>

#include "common.cuh"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr int kBM = 128, kBK = 64, kStages = 4, kThreads = 192;
constexpr int kN = 256;                       // accumulator columns per item
constexpr uint32_t kTmemCols = 2 * kN;        // two accumulators
constexpr int kABytes = kBM * kBK * 2;        // 16 KB
constexpr int kBBytes = kN * kBK * 2;         // 32 KB
constexpr long long kDrainBudget = 2000000000LL;

struct TcArgs {
    __nv_bfloat16* out;       // h (FC1) or yp (FC2)
    int out_ld;               // F or d
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
};

struct Smem {
    uint64_t full[kStages], empty[kStages], acc_full[2], acc_empty[2], drain;
    uint32_t tmem_base;
    int abort_flag;
};

constexpr size_t kSmemBytes = 1024 /*align slack*/ + kStages * (kABytes + kBBytes) + sizeof(Smem) +
                              sizeof(int32_t) * (kMaxE + 1);

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

// Work item -> (expert, first row, column tile). Items run expert-major:
// expert e owns items [n_tiles*off[e], n_tiles*off[e+1]), column tile major,
// then its blocks in schedule order.
__device__ __forceinline__ void decode_item(long long it, int n_tiles, const int32_t* s_off, int E,
                                            const int32_t* sched, const int32_t* blocks, int& expert,
                                            int& row0, int& j) {
    int lo = 0, hi = E;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if ((long long)n_tiles * s_off[mid] <= it) lo = mid; else hi = mid;
    }
    const int nb = s_off[lo + 1] - s_off[lo];
    const long long local = it - (long long)n_tiles * s_off[lo];
    j = (int)(local / nb);
    const int b = sched[s_off[lo] + (int)(local % nb)];
    expert = blocks[kBlockInts * b];
    row0 = blocks[kBlockInts * b + 1];
}

__device__ __forceinline__ float silu(float a) { return a / (1.f + __expf(-a)); }

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// MODE 0: FC1 + SwiGLU -> h; MODE 1: FC2 -> yp.
template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
ffn_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, TcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = base;
    uint8_t* sB = base + kStages * kABytes;
    Smem* S = reinterpret_cast<Smem*>(sB + kStages * kBBytes);
    int32_t* s_off = reinterpret_cast<int32_t*>(S + 1);
    volatile int* abort_flag = &S->abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) { ptx::mbar_init(&S->full[s], 1); ptx::mbar_init(&S->empty[s], 1); }
        for (int q = 0; q < 2; ++q) { ptx::mbar_init(&S->acc_full[q], 1); ptx::mbar_init(&S->acc_empty[q], 128); }
        ptx::mbar_init(&S->drain, 1);
        S->abort_flag = 0;
        ptx::fence_barrier_init();
    }
    for (int i = threadIdx.x; i <= a.E; i += kThreads) s_off[i] = a.sched_off[i];
    if (warp == 0 && lane == 0) { ptx::prefetch_tmap(&tmA); ptx::prefetch_tmap(&tmB); }
    if (warp == 1) { ptx::tmem_alloc(&S->tmem_base, kTmemCols); ptx::tmem_relinquish(); }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = S->tmem_base;
    const long long n_items = (long long)a.header[H_NBLOCKS] * a.n_tiles;
    const int kb_count = a.Kdim / kBK;
    constexpr int kColTile = MODE == 0 ? 128 : 256;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            long long fills = 0;
            bool ok = true;
            for (long long it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
                int e, row0, j;
                decode_item(it, a.n_tiles, s_off, a.E, a.sched, a.blocks, e, row0, j);
                const int brow = e * a.b_rows + j * kColTile;
                for (int kb = 0; kb < kb_count; ++kb) {
                    if (!role_wait(&S->empty[stage], phase ^ 1, a.spin, abort_flag, a.header)) { ok = false; break; }
                    ptx::mbar_arrive_expect_tx(&S->full[stage], kABytes + kBBytes);
                    ptx::tma_load_2d(sA + stage * kABytes, &tmA, kb * kBK, row0, &S->full[stage]);
                    if (MODE == 0) {
                        ptx::tma_load_2d(sB + stage * kBBytes, &tmB, kb * kBK, brow, &S->full[stage]);
                        ptx::tma_load_2d(sB + stage * kBBytes + kBBytes / 2, &tmB, kb * kBK, brow + a.F,
                                         &S->full[stage]);
                    } else {
                        ptx::tma_load_2d(sB + stage * kBBytes, &tmB, kb * kBK, brow, &S->full[stage]);
                    }
                    ++fills;
                    if (++stage == kStages) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok) {
                // let every copy still in flight land before the CTA exits
                const long long first = fills > kStages ? fills - kStages : 0;
                for (long long f = first; f < fills; ++f)
                    ptx::mbar_wait(&S->full[f % kStages], (uint32_t)((f / kStages) & 1), kDrainBudget);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = ptx::idesc_bf16_f32(kBM, kN);
            int stage = 0;
            uint32_t phase = 0;
            int local = 0;
            bool ok = true, issued = false;
            for (long long it = blockIdx.x; it < n_items && ok; it += gridDim.x, ++local) {
                const int acc = local & 1;
                const uint32_t acc_phase = (uint32_t)((local >> 1) & 1);
                if (!role_wait(&S->acc_empty[acc], acc_phase ^ 1, a.spin, abort_flag, a.header)) { ok = false; break; }
                ptx::tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(acc * kN);
                for (int kb = 0; kb < kb_count; ++kb) {
                    if (!role_wait(&S->full[stage], phase, a.spin, abort_flag, a.header)) { ok = false; break; }
                    ptx::tc_fence_after();
                    const uint32_t a_addr = ptx::smem_addr(sA + stage * kABytes);
                    const uint32_t b_addr = ptx::smem_addr(sB + stage * kBBytes);
#pragma unroll
                    for (int ks = 0; ks < kBK / 16; ++ks) {
                        ptx::mma_bf16(d_tmem, ptx::sdesc_k_sw128(a_addr + ks * 32), ptx::sdesc_k_sw128(b_addr + ks * 32),
                                      idesc, (kb | ks) != 0 ? 1u : 0u);
                    }
                    issued = true;
                    ptx::mma_commit(&S->empty[stage]);
                    if (++stage == kStages) { stage = 0; phase ^= 1; }
                }
                if (ok) ptx::mma_commit(&S->acc_full[acc]);
            }
            if (!ok && issued) {
                // wait for every MMA issued so far before TMEM is freed
                ptx::mma_commit(&S->drain);
                ptx::mbar_wait(&S->drain, 0, kDrainBudget);
            }
        }
    } else {
        // ------------------------------------------------ epilogue, warps 2..5
        const int quad = warp & 3;                 // TMEM lanes 32*quad .. 32*quad+31
        const int m = quad * 32 + lane;            // row inside the tile
        int local = 0;
        for (long long it = blockIdx.x; it < n_items; it += gridDim.x, ++local) {
            int e, row0, j;
            decode_item(it, a.n_tiles, s_off, a.E, a.sched, a.blocks, e, row0, j);
            const int acc = local & 1;
            const uint32_t acc_phase = (uint32_t)((local >> 1) & 1);
            if (!role_wait(&S->acc_full[acc], acc_phase, a.spin, abort_flag, a.header)) break;
            ptx::tc_fence_after();
            const uint32_t t_row = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * kN);
            uint4* orow = reinterpret_cast<uint4*>(a.out + (int64_t)(row0 + m) * a.out_ld + (int64_t)j * kColTile);
            if (MODE == 0) {
#pragma unroll 1
                for (int c = 0; c < 128; c += 32) {
                    uint32_t g[32], u[32];
                    ptx::tmem_ld32(t_row + c, g);
                    ptx::tmem_ld32(t_row + 128 + c, u);
                    ptx::tmem_ld_wait();
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float h0 = silu(__uint_as_float(g[2 * i])) * __uint_as_float(u[2 * i]);
                        const float h1 = silu(__uint_as_float(g[2 * i + 1])) * __uint_as_float(u[2 * i + 1]);
                        pk[i] = pack_bf16(h0, h1);
                    }
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        orow[c / 8 + v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
                }
            } else {
#pragma unroll 1
                for (int c = 0; c < 256; c += 32) {
                    uint32_t y[32];
                    ptx::tmem_ld32(t_row + c, y);
                    ptx::tmem_ld_wait();
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) pk[i] = pack_bf16(__uint_as_float(y[2 * i]), __uint_as_float(y[2 * i + 1]));
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        orow[c / 8 + v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
                }
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(&S->acc_empty[acc]);
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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
bool make_tmap(CUtensorMap* tm, const void* ptr, uint64_t inner, uint64_t rows, uint32_t box_rows) {
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

template <int MODE>
cudaError_t launch_mode(const CUtensorMap& tA, const CUtensorMap& tB, const TcArgs& a, int grid,
                        cudaStream_t st) {
    cudaError_t err = cudaFuncSetAttribute(ffn_tc_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)kSmemBytes);
    if (err != cudaSuccess) return err;
    ffn_tc_kernel<MODE><<<grid, kThreads, kSmemBytes, st>>>(tA, tB, a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ffn_tc(const Shape& s, int which, const void* a_mat, const void* w, void* out,
                          const WsPtrs& ws, cudaStream_t st, long long spin_budget) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    TcArgs a;
    a.E = s.E;
    a.spin = spin_budget;
    a.blocks = ws.blocks;
    a.sched = ws.sched;
    a.sched_off = ws.sched_off;
    a.header = ws.header;
    a.out = static_cast<__nv_bfloat16*>(out);
    CUtensorMap tA, tB;
    if (which == 1) {
        // FC1 + SwiGLU: xp [rows_cap, d] x w_gate_up [E*2F, d] -> h [rows_cap, F]
        if (!make_tmap(&tA, a_mat, (uint64_t)s.d, (uint64_t)s.rows_cap, kBM) ||
            !make_tmap(&tB, w, (uint64_t)s.d, (uint64_t)s.E * 2 * s.F, 128))
            return cudaErrorInvalidValue;
        a.out_ld = s.F;
        a.Kdim = s.d;
        a.n_tiles = s.F / 128;
        a.F = s.F;
        a.b_rows = 2 * s.F;
        return launch_mode<0>(tA, tB, a, sms, st);
    }
    // FC2: h [rows_cap, F] x w_down [E*d, F] -> yp [rows_cap, d]
    if (!make_tmap(&tA, a_mat, (uint64_t)s.F, (uint64_t)s.rows_cap, kBM) ||
        !make_tmap(&tB, w, (uint64_t)s.F, (uint64_t)s.E * s.d, 256))
        return cudaErrorInvalidValue;
    a.out_ld = s.d;
    a.Kdim = s.F;
    a.n_tiles = s.d / 256;
    a.F = 0;
    a.b_rows = s.d;
    return launch_mode<1>(tA, tB, a, sms, st);
}

}  // namespace moe
