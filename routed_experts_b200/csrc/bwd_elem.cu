// bwd_elem.cu - the memory-bound steps of the layer's backward.
//
// [MegaFlux] "MegaFlux: Skew-Resilient MoE Megakernels via Pipelined Expert
// Replication", §3.2 'Backward'. Around the grouped GEMMs of bwd_tc.cu:
//   - the combine's backward: every routed entry (t, k) gets the row
//     dY = bf16(w[t,k] * dOut[t]) (the product formed in fp32), and the
//     routing weight's gradient dw[t,k] = dOut[t] . yp[row(t,k)];
//   - padding rows of xp and dY set to zero, so that WGrad, whose contraction
//     runs over whole blocks, reads zeros there (dispatch leaves xp's padding
//     rows unwritten);
//   - the gating's backward: dlogits[t, idx[t,m]] = w_m (dw_m - sum_k w_k dw_k),
//     times (1 - sigmoid(l)) for sigmoid gating; zero off the top-k. The
//     weights sum to one, so the inner term is formed as sum_k w_k (dw_m - dw_k),
//     which keeps its precision when one weight is close to one.
// dx = sum over k of dXp[row(t,k)] is the combine kernel with unit weights.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kWarps = 8;

template <int KMAX>
__global__ void __launch_bounds__(kWarps * 32)
bwd_scatter_kernel(const uint4* __restrict__ d_out, const uint4* __restrict__ yp, const float* __restrict__ w,
                   uint4* __restrict__ dy, float* __restrict__ dw, int T, int K, int nvec, int64_t rows_cap,
                   WsPtrs ws) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t bad = 0;
    for (int t = blockIdx.x * kWarps + warp; t < T; t += gridDim.x * kWarps) {
        int my_row = 0;
        float my_w = 0.f;
        if (lane < K) {
            my_row = ws.row_of[(int64_t)t * K + lane];
            my_w = w[(int64_t)t * K + lane];
            if (my_row < 0 || my_row >= rows_cap) { bad = 1; my_row = -1; }
        }
        int rows[KMAX];
        float wk[KMAX], part[KMAX];
#pragma unroll
        for (int k = 0; k < KMAX; ++k) {
            rows[k] = __shfl_sync(0xffffffffu, my_row, k);
            wk[k] = __shfl_sync(0xffffffffu, my_w, k);
            part[k] = 0.f;
        }
        for (int v = lane; v < nvec; v += 32) {
            const uint4 go = __ldg(d_out + (int64_t)t * nvec + v);
            // the K rows' vectors are all requested before any is used
            uint4 yv[KMAX];
#pragma unroll
            for (int k = 0; k < KMAX; ++k)
                if (k < K && rows[k] >= 0) yv[k] = __ldg(yp + (int64_t)rows[k] * nvec + v);
            const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&go);
            float gf[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(g2[i]);
                gf[2 * i] = f.x;
                gf[2 * i + 1] = f.y;
            }
#pragma unroll
            for (int k = 0; k < KMAX; ++k) {
                if (k >= K || rows[k] < 0) continue;
                const __nv_bfloat162* y2 = reinterpret_cast<const __nv_bfloat162*>(&yv[k]);
                uint4 o;
                __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 yf = __bfloat1622float2(y2[i]);
                    part[k] = fmaf(gf[2 * i], yf.x, part[k]);
                    part[k] = fmaf(gf[2 * i + 1], yf.y, part[k]);
                    o2[i] = __floats2bfloat162_rn(__fmul_rn(wk[k], gf[2 * i]), __fmul_rn(wk[k], gf[2 * i + 1]));
                }
                dy[(int64_t)rows[k] * nvec + v] = o;
            }
        }
#pragma unroll
        for (int k = 0; k < KMAX; ++k) {
            if (k >= K) break;
            float s = part[k];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
            if (lane == 0) dw[(int64_t)t * K + k] = s;
        }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) set_status(ws.header, MOE_DEV_BAD_INDEX);
}

// Zero the padding rows (src_of = -1) of up to two [rows, nvec x 16 B] buffers.
__global__ void __launch_bounds__(kWarps * 32)
zero_padding_kernel(uint4* __restrict__ a, uint4* __restrict__ b, int nvec, WsPtrs ws) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int total = (int)ws.header[H_TOTAL_ROWS];
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int row = blockIdx.x * kWarps + warp; row < total; row += gridDim.x * kWarps) {
        if (ws.src_of[row] >= 0) continue;
        for (int v = lane; v < nvec; v += 32) {
            a[(int64_t)row * nvec + v] = z;
            if (b) b[(int64_t)row * nvec + v] = z;
        }
    }
}

__global__ void __launch_bounds__(kWarps * 32)
dlogits_kernel(const float* __restrict__ logits, const int32_t* __restrict__ idx, const float* __restrict__ w,
               const float* __restrict__ dw, float* __restrict__ dl, int T, int E, int K, int sigmoid_gating) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int t = blockIdx.x * kWarps + warp; t < T; t += gridDim.x * kWarps) {
        float wk = 0.f, dwk = 0.f;
        int e = -1;
        if (lane < K) {
            wk = w[(int64_t)t * K + lane];
            dwk = dw[(int64_t)t * K + lane];
            e = idx[(int64_t)t * K + lane];
        }
        float inner = 0.f;
        for (int k = 0; k < K; ++k) {
            const float w_k = __shfl_sync(0xffffffffu, wk, k), dw_k = __shfl_sync(0xffffffffu, dwk, k);
            inner = fmaf(w_k, dwk - dw_k, inner);
        }
        float* row = dl + (int64_t)t * E;
        for (int c = lane; c < E; c += 32) row[c] = 0.f;
        __syncwarp();
        if (lane < K && e >= 0 && e < E) {
            float v = wk * inner;
            if (sigmoid_gating) v *= 1.f - 1.f / (1.f + expf(-logits[(int64_t)t * E + e]));
            row[e] = v;
        }
    }
}

int grid_for(int64_t work_warps) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (work_warps + kWarps - 1) / kWarps;
    const int64_t cap = (int64_t)sms * 8;
    return (int)(want < 1 ? 1 : (want < cap ? want : cap));
}

}  // namespace

cudaError_t launch_bwd_scatter(const Shape& s, const void* d_out, const void* yp, const float* w, void* dy,
                               float* dw, const WsPtrs& ws, cudaStream_t st) {
    const int nvec = (int)((int64_t)s.d * s.eb / 16);
    const int grid = grid_for(s.T);
    auto d4 = static_cast<const uint4*>(d_out);
    auto y4 = static_cast<const uint4*>(yp);
    auto o4 = static_cast<uint4*>(dy);
    if (s.K <= 8)
        bwd_scatter_kernel<8><<<grid, kWarps * 32, 0, st>>>(d4, y4, w, o4, dw, s.T, s.K, nvec, s.rows_cap, ws);
    else
        bwd_scatter_kernel<16><<<grid, kWarps * 32, 0, st>>>(d4, y4, w, o4, dw, s.T, s.K, nvec, s.rows_cap, ws);
    return cudaGetLastError();
}

cudaError_t launch_zero_padding(const Shape& s, void* a, void* b, int64_t row_bytes, const WsPtrs& ws,
                                cudaStream_t st) {
    const int grid = grid_for(s.rows_cap);
    zero_padding_kernel<<<grid, kWarps * 32, 0, st>>>(static_cast<uint4*>(a), static_cast<uint4*>(b),
                                                      (int)(row_bytes / 16), ws);
    return cudaGetLastError();
}

cudaError_t launch_dlogits(const Shape& s, const float* logits, const int32_t* idx, const float* w, const float* dw,
                           float* dl, cudaStream_t st) {
    const int grid = grid_for(s.T);
    dlogits_kernel<<<grid, kWarps * 32, 0, st>>>(logits, idx, w, dw, dl, s.T, s.E, s.K,
                                                 s.gating == MOE_GATE_SIGMOID_TOPK ? 1 : 0);
    return cudaGetLastError();
}

}  // namespace moe
