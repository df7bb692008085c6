// topk_hist.cu - router top-k, gating weights and the per-chunk expert-load
// histogram (steps A1-A3).
//
// [MegaFlux] "MegaFlux: Skew-Resilient MoE Megakernels via Pipelined Expert
// Replication", §1: a learned router selects a few experts per token whose
// outputs are combined by routing weights; §4.1 "Routing workload
// construction": k distinct experts per token; §3.1: the planner starts from
// the routing profile (per-expert load).
//
// One warp per token (a CTA per 32-token chunk). Lane l holds logits of experts l, l+32, l+64, ...
// (coalesced 128-byte rows). K rounds of a warp arg-max pick the experts in
// descending logit order, ties to the lower expert id: each round is two
// warp reductions (redux.sync), the largest order-preserving key of the
// lanes' best logits, then the lowest expert among the lanes that hold it. Gating: softmax over
// the chosen logits (equal to the full softmax renormalised over them), or
// their sigmoids normalised over them. Every CTA covers kTokPerChunk tokens
// and counts its chunk's entries per expert in shared memory; the planner
// turns the per-chunk counts into totals and per-chunk offsets, so no global
// atomics and no zeroing pass are needed.
#include <math.h>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kWarps = kTokPerChunk;   // one warp per token

__device__ __forceinline__ bool better(float va, int ea, float vb, int eb) {
    return va > vb || (va == vb && ea < eb);
}

// An unsigned key in the order of the float (finite or -inf, -0 already
// folded into +0, so equal values have equal keys), and back.
__device__ __forceinline__ uint32_t order_key(float x) {
    const uint32_t b = __float_as_uint(x);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Two CTAs per SM where the logits of a lane fit in few registers.
template <int EPT>
__global__ void __launch_bounds__(kWarps * 32, EPT <= 4 ? 2 : 1)
topk_hist_kernel(const float* __restrict__ logits, int32_t* __restrict__ idx,
                 float* __restrict__ wout, int T, int E, int K, int gating,
                 int32_t* __restrict__ chunk_counts, uint32_t* __restrict__ chunk_flags) {
    pdl_wait();
    pdl_trigger();
    extern __shared__ int32_t hist[];   // [E]
    __shared__ uint32_t flag;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int chunk = blockIdx.x;
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
    if (threadIdx.x == 0) flag = 0;
    __syncthreads();

    uint32_t bad = 0;
    for (int i = warp; i < kTokPerChunk; i += kWarps) {
        const int t = chunk * kTokPerChunk + i;
        if (t >= T) break;
        const float* row = logits + (int64_t)t * E;
        float v[EPT];
#pragma unroll
        for (int j = 0; j < EPT; ++j) {
            const int e = j * 32 + lane;
            float x = e < E ? __ldg(row + e) : -INFINITY;
            if (e < E && !isfinite(x)) bad = 1;
            if (x != x) x = -INFINITY;
            if (x == 0.f) x = 0.f;   // -0 and +0 compare equal: one key for both
            v[j] = x;
        }
        // lane k < K owns entry k
        uint32_t taken = 0;
        float my_v = 0.f, top = 0.f;
        int my_e = 0;
        for (int k = 0; k < K; ++k) {
            float bv = -INFINITY;
            int be = 0x7fffffff;
#pragma unroll
            for (int j = 0; j < EPT; ++j) {
                const int e = j * 32 + lane;
                if (!(taken >> j & 1u) && e < E && better(v[j], e, bv, be)) { bv = v[j]; be = e; }
            }
            const uint32_t key = order_key(bv);
            const uint32_t kmax = __reduce_max_sync(0xffffffffu, key);
            be = (int)__reduce_min_sync(0xffffffffu, key == kmax ? (uint32_t)be : 0xffffffffu);
            bv = key_value(kmax);
            if ((be & 31) == lane) taken |= 1u << (be >> 5);
            if (k == 0) top = bv;
            if (k == lane) { my_v = bv; my_e = be; }
        }
        float g = 0.f;
        if (lane < K) {
            g = gating == MOE_GATE_SOFTMAX_TOPK ? expf(my_v - top) : 1.f / (1.f + expf(-my_v));
        }
        float sum = g;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        if (lane < K) {
            idx[(int64_t)t * K + lane] = my_e;
            wout[(int64_t)t * K + lane] = g / sum;
            atomicAdd(&hist[my_e], 1);
        }
    }
    if (bad) atomicOr(&flag, (uint32_t)MOE_DEV_BAD_INDEX);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        chunk_counts[(int64_t)chunk * E + e] = hist[e];
    if (threadIdx.x == 0) chunk_flags[chunk] = flag;
}

template <int EPT>
cudaError_t launch_ept(const Shape& s, const float* logits, int32_t* idx, float* w,
                       const WsPtrs& ws, cudaStream_t st) {
    const size_t smem = sizeof(int32_t) * s.E;
    return launch_pdl(topk_hist_kernel<EPT>, dim3(s.n_chunks), dim3(kWarps * 32), smem, st, logits, idx, w, s.T,
                      s.E, s.K, s.gating, ws.chunk_counts, ws.chunk_flags);
}

}  // namespace

cudaError_t launch_topk_hist(const Shape& s, const float* logits, int32_t* idx, float* w,
                             const WsPtrs& ws, cudaStream_t st) {
    const int need = (s.E + 31) / 32;
    if (need <= 1) return launch_ept<1>(s, logits, idx, w, ws, st);
    if (need <= 2) return launch_ept<2>(s, logits, idx, w, ws, st);
    if (need <= 4) return launch_ept<4>(s, logits, idx, w, ws, st);
    if (need <= 8) return launch_ept<8>(s, logits, idx, w, ws, st);
    if (need <= 16) return launch_ept<16>(s, logits, idx, w, ws, st);
    return launch_ept<32>(s, logits, idx, w, ws, st);
}

}  // namespace moe
