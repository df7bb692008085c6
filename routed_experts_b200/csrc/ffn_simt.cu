// ffn_simt.cu - the grouped SwiGLU expert FFN in fp32 on the CUDA cores
// (steps A7, A8 for fp32 layers).
//
// [MegaFlux] "MegaFlux: Skew-Resilient MoE Megakernels via Pipelined Expert
// Replication", §2.1 and §3.2 'Forward': FC1 (gate and up projections) then
// FC2 (down projection) per planned token block; §4.1: SwiGLU experts.
// fp32 layers need fp32 products and sums (the tensor cores' tf32 mode keeps
// 10 mantissa bits), so they run here: each CTA takes (block, column tile)
// work items of the planned block table, stages a BK-deep slice of the block's
// rows and of the expert's weight rows in shared memory, and accumulates in
// registers. h = silu(gate) * up with silu(a) = a / (1 + exp(-a)). Rows of
// a block past its valid ones (padding) are stored as zero.
#include <math.h>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kBN = 64, kBK = 32, kThr = 256;

// MODE 0: FC1 + SwiGLU (out = h, n over F); MODE 1: FC2 (out = yp, n over d).
template <int MODE, int BM>
__global__ void __launch_bounds__(kThr)
ffn_simt_kernel(const float* __restrict__ a_mat, const float* __restrict__ w, float* __restrict__ out,
                int Kdim, int Nout, int F, int64_t w_expert_rows, WsPtrs ws) {
    constexpr int MR = BM / 4;
    __shared__ float As[kBK][BM];
    __shared__ float Bg[kBK][kBN + 1];
    __shared__ float Bu[MODE == 0 ? kBK : 1][kBN + 1];
    const int tid = threadIdx.x, tx = tid % kBN, ty = tid / kBN;
    const int n_blocks = (int)ws.header[H_NBLOCKS];
    const int n_tiles = Nout / kBN;
    const int64_t n_items = (int64_t)n_blocks * n_tiles;
    for (int64_t it = blockIdx.x; it < n_items; it += gridDim.x) {
        const int b = (int)(it / n_tiles), j = (int)(it % n_tiles);
        const int32_t* B = ws.blocks + (int64_t)kBlockInts * b;
        const int e = B[0], row0 = B[1], valid = B[2];
        const int n0 = j * kBN;
        float acc_g[MR], acc_u[MR];
#pragma unroll
        for (int i = 0; i < MR; ++i) { acc_g[i] = 0.f; acc_u[i] = 0.f; }
        const float* wg = w + ((int64_t)e * w_expert_rows + n0) * Kdim;
        const float* wu = wg + (int64_t)F * Kdim;
        for (int k0 = 0; k0 < Kdim; k0 += kBK) {
            for (int q = tid; q < BM * kBK; q += kThr) {
                const int m = q / kBK, kk = q % kBK;
                As[kk][m] = a_mat[(int64_t)(row0 + m) * Kdim + k0 + kk];
            }
            for (int q = tid; q < kBN * kBK; q += kThr) {
                const int n = q / kBK, kk = q % kBK;
                Bg[kk][n] = wg[(int64_t)n * Kdim + k0 + kk];
                if (MODE == 0) Bu[kk][n] = wu[(int64_t)n * Kdim + k0 + kk];
            }
            __syncthreads();
#pragma unroll 4
            for (int kk = 0; kk < kBK; ++kk) {
                const float bg = Bg[kk][tx];
                const float bu = MODE == 0 ? Bu[kk][tx] : 0.f;
#pragma unroll
                for (int i = 0; i < MR; ++i) {
                    const float av = As[kk][ty + 4 * i];
                    acc_g[i] = fmaf(av, bg, acc_g[i]);
                    if (MODE == 0) acc_u[i] = fmaf(av, bu, acc_u[i]);
                }
            }
            __syncthreads();
        }
#pragma unroll
        for (int i = 0; i < MR; ++i) {
            const int m = ty + 4 * i;
            float v;
            if (MODE == 0) v = acc_g[i] / (1.f + expf(-acc_g[i])) * acc_u[i];
            else v = acc_g[i];
            out[(int64_t)(row0 + m) * Nout + n0 + tx] = m < valid ? v : 0.f;   // padding rows: zero
        }
    }
}

template <int BM>
cudaError_t launch_bm(const Shape& s, int which, const void* a_mat, const void* w, void* out, const WsPtrs& ws,
                      cudaStream_t st, int grid) {
    if (which == 1)
        ffn_simt_kernel<0, BM><<<grid, kThr, 0, st>>>(static_cast<const float*>(a_mat), static_cast<const float*>(w),
                                                     static_cast<float*>(out), s.d, s.F, s.F, 2 * (int64_t)s.F, ws);
    else
        ffn_simt_kernel<1, BM><<<grid, kThr, 0, st>>>(static_cast<const float*>(a_mat), static_cast<const float*>(w),
                                                     static_cast<float*>(out), s.F, s.d, s.F, (int64_t)s.d, ws);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ffn_simt(const Shape& s, int which, const void* a_mat, const void* w, void* out,
                            const WsPtrs& ws, cudaStream_t st) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = sms * 4;
    switch (s.tile) {
        case 16: return launch_bm<16>(s, which, a_mat, w, out, ws, st, grid);
        case 32: return launch_bm<32>(s, which, a_mat, w, out, ws, st, grid);
        case 64: return launch_bm<64>(s, which, a_mat, w, out, ws, st, grid);
        case 128: return launch_bm<128>(s, which, a_mat, w, out, ws, st, grid);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe
