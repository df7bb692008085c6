// combine.cu - the weighted top-k sum (step A9).
//
// [MegaFlux] "MegaFlux: Skew-Resilient MoE Megakernels via Pipelined Expert
// Replication", §1: expert outputs are combined according to the routing
// weights; §2.1: the final top-k sum is its own launch.
//
// out[t] = sum over k = 0..K-1, in that order, of w[t,k] * yp[row_of(t,k)],
// accumulated in fp32 and rounded once to the output type. One warp per token;
// each lane owns 16-byte column vectors and keeps the K row loads in flight.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kCWarps = 8;

// KMAX: a compile-time bound on K (K <= KMAX) so the K rows a lane reads stay in
// registers without reserving room for the largest K.
template <bool BF16, int KMAX>
__global__ void __launch_bounds__(kCWarps * 32)
combine_kernel(const uint4* __restrict__ yp, const float* __restrict__ w, uint4* __restrict__ out,
               int T, int K, int nvec, int64_t rows_cap, WsPtrs ws) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t bad = 0;
    for (int t = blockIdx.x * kCWarps + warp; t < T; t += gridDim.x * kCWarps) {
        int my_row = 0;
        float my_w = 0.f;
        if (lane < K) {
            my_row = ws.row_of[(int64_t)t * K + lane];
            my_w = w ? w[(int64_t)t * K + lane] : 1.f;   // no weights: a plain sum (the backward's dx)
            if (my_row < 0 || my_row >= rows_cap) { bad = 1; my_row = 0; my_w = 0.f; }
        }
        int rows[KMAX];
        float ws_[KMAX];
#pragma unroll
        for (int k = 0; k < KMAX; ++k) {
            rows[k] = __shfl_sync(0xffffffffu, my_row, k);
            ws_[k] = __shfl_sync(0xffffffffu, my_w, k);
        }
        for (int v = lane; v < nvec; v += 32) {
            uint4 val[KMAX];
#pragma unroll
            for (int k = 0; k < KMAX; ++k)
                if (k < K) val[k] = __ldg(yp + (int64_t)rows[k] * nvec + v);
            if (BF16) {
                float acc[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[j] = 0.f;
#pragma unroll
                for (int k = 0; k < KMAX; ++k) {
                    if (k >= K) break;
                    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&val[k]);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float2 f = __bfloat1622float2(p[j]);
                        acc[2 * j] = fmaf(ws_[k], f.x, acc[2 * j]);
                        acc[2 * j + 1] = fmaf(ws_[k], f.y, acc[2 * j + 1]);
                    }
                }
                uint4 o;
                __nv_bfloat162* q = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
                for (int j = 0; j < 4; ++j) q[j] = __floats2bfloat162_rn(acc[2 * j], acc[2 * j + 1]);
                out[(int64_t)t * nvec + v] = o;
            } else {
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int k = 0; k < KMAX; ++k) {
                    if (k >= K) break;
                    const float* f = reinterpret_cast<const float*>(&val[k]);
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[j] = fmaf(ws_[k], f[j], acc[j]);
                }
                out[(int64_t)t * nvec + v] = make_uint4(__float_as_uint(acc[0]), __float_as_uint(acc[1]),
                                                        __float_as_uint(acc[2]), __float_as_uint(acc[3]));
            }
        }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) set_status(ws.header, MOE_DEV_BAD_INDEX);
}

}  // namespace

cudaError_t launch_combine(const Shape& s, const void* yp, const float* w, void* out,
                           const WsPtrs& ws, cudaStream_t st) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int nvec = (int)((int64_t)s.d * s.eb / 16);
    int64_t want = (s.T + kCWarps - 1) / kCWarps;
    int64_t cap = (int64_t)sms * 16;
    const int grid = (int)(want < cap ? want : cap);
    const uint4* y4 = static_cast<const uint4*>(yp);
    uint4* o4 = static_cast<uint4*>(out);
#define MOE_COMBINE(B, KM) \
    return launch_pdl(combine_kernel<B, KM>, dim3(grid), dim3(kCWarps * 32), 0, st, y4, w, o4, s.T, s.K, nvec, \
                      s.rows_cap, ws)
    const bool bf = s.dtype == MOE_BF16;
    if (s.K <= 2) { if (bf) MOE_COMBINE(true, 2); else MOE_COMBINE(false, 2); }
    else if (s.K <= 4) { if (bf) MOE_COMBINE(true, 4); else MOE_COMBINE(false, 4); }
    else if (s.K <= 8) { if (bf) MOE_COMBINE(true, 8); else MOE_COMBINE(false, 8); }
    else { if (bf) MOE_COMBINE(true, 16); else MOE_COMBINE(false, 16); }
#undef MOE_COMBINE
}

}  // namespace moe
