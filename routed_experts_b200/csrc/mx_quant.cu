// mx_quant.cu - MXFP8 quantization on the GPU: the expert weights (once,
// ahead of the layer) and the token rows inside the dispatch.
//
// [MegaFlux] "MegaFlux: Skew-Resilient MoE Megakernels via Pipelined Expert
// Replication", §2.1 'Persistent MoE execution' (block-scaled MXFP8 / MXFP4
// tensor-core MMA) and §4.1 'Setup' (MX operands in the forward, fp32
// accumulation, bf16 outputs); [MoonEP] "A bandwidth-only model" (one scale
// per 32 elements). The formats are the OCP Microscaling ones: per 32
// consecutive elements along the contraction a scale 2^(s - 127) kept as its
// exponent s (E8M0), s = floor(log2 max|v|) - 8 + 127 clamped to [0, 254]
// (0 for an all-zero block), and each element v / 2^(s - 127) rounded to
// E4M3 (nearest, ties to even, saturating at 448). For an fp32 block maximum,
// floor(log2 max|v|) + 127 is its exponent field, so s = max(field - 8, 0);
// 2^(127 - s) is built from its exponent field 254 - s and multiplying by it
// is exact.
//
// A warp takes 256 elements of a row per step, 8 per lane (one 16-byte
// load); four neighbouring lanes hold one 32-element block, whose maximum is
// two xor-shuffles away. Each lane converts its 8 values and stores 8 bytes;
// the block's first lane stores the scale byte at its place in the chunked
// scale layout (mx_scale_offset).
//
// Weights may also be quantized to MXFP4 ([MegaFlux] §4.1: MXFP4 weights):
// E2M1 elements (0, 0.5, 1, 1.5, 2, 3, 4, 6; nearest, ties to even,
// saturating at 6) with s = floor(log2 max|v|) - 2 + 127 (2 = the exponent
// of E2M1's largest normal, 6 = 1.5 * 2^2), two codes per byte, element 2i
// in the low nibble of byte i.
#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kQWarps = 8;

// The scale exponent of a block with fp32 maximum amax; EMAX is the exponent
// of the element format's largest normal (8 for E4M3, 2 for E2M1).
template <uint32_t EMAX = 8>
__device__ __forceinline__ uint32_t mx_scale_of(float amax) {
    const uint32_t field = (__float_as_uint(amax) >> 23) & 0xFFu;
    return field > EMAX ? field - EMAX : 0u;
}

__device__ __forceinline__ float mx_inv_scale(uint32_t s) { return __uint_as_float((254u - s) << 23); }

__device__ __forceinline__ float amax8(const uint4& v) {
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(p[i]);
        m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
    return m;
}

// The block scale of the 32 elements held by this lane's group of four.
template <uint32_t EMAX = 8>
__device__ __forceinline__ uint32_t group_scale(float m) {
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
    return mx_scale_of<EMAX>(m);
}

// 8 bf16 values times inv, rounded to E4M3, element 0 in the lowest byte.
__device__ __forceinline__ uint2 e4m3x8(const uint4& v, float inv) {
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 f = __bfloat1622float2(p[i]);
        f.x *= inv;
        f.y *= inv;
        const uint32_t two = (uint32_t)__nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3);
        w[i >> 1] |= two << (16 * (i & 1));
    }
    return make_uint2(w[0], w[1]);
}

// 8 bf16 values times inv, rounded to E2M1, two per byte, element 0 in the
// lowest nibble.
__device__ __forceinline__ uint32_t e2m1x8(const uint4& v, float inv) {
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
    uint32_t w = 0u;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 f = __bfloat1622float2(p[i]);
        f.x *= inv;
        f.y *= inv;
        w |= (uint32_t)__nv_cvt_float2_to_fp4x2(f, __NV_E2M1, cudaRoundNearest) << (8 * i);
    }
    return w;
}

// Row r of the quantized matrix reads input row src_row(r).
__device__ __forceinline__ int64_t src_row(int64_t r, int interleave_F) {
    if (interleave_F <= 0) return r;
    const int64_t per = 2LL * interleave_F;
    const int64_t e = r / per, rr = r % per, jt = rr / 128, t = rr % 128;
    return e * per + (t < 64 ? jt * 64 + t : interleave_F + jt * 64 + (t - 64));
}

template <int FMT>   // MOE_MX_W_E4M3 or MOE_MX_W_E2M1
__global__ void __launch_bounds__(kQWarps * 32)
mx_quantize_kernel(const uint4* __restrict__ x, int64_t rows, int K, int interleave_F, uint8_t* __restrict__ q,
                   uint8_t* __restrict__ sc) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int segs = (K + 255) / 256;   // K % 128 == 0: the last step of a row may be half full
    const int64_t units = rows * segs;
    for (int64_t u = (int64_t)blockIdx.x * kQWarps + warp; u < units; u += (int64_t)gridDim.x * kQWarps) {
        const int64_t r = u / segs;
        const int seg = (int)(u % segs);
        const int64_t col = (int64_t)seg * 256 + lane * 8;
        const bool in = col < K;   // whole groups of four lanes (32-blocks) are in or out together
        const uint4 v = in ? __ldg(x + (src_row(r, interleave_F) * K + col) / 8) : make_uint4(0, 0, 0, 0);
        const uint32_t s = group_scale<FMT == MOE_MX_W_E2M1 ? 2u : 8u>(amax8(v));
        if (in) {
            if (FMT == MOE_MX_W_E2M1)
                *reinterpret_cast<uint32_t*>(q + (r * K + col) / 2) = e2m1x8(v, mx_inv_scale(s));
            else
                *reinterpret_cast<uint2*>(q + r * K + col) = e4m3x8(v, mx_inv_scale(s));
            if ((lane & 3) == 0) sc[mx_scale_offset(r, col / 32, K)] = (uint8_t)s;
        }
    }
}

// One warp per token: quantize its row once, store codes and scales to the K
// rows the row map names. Padding rows are not written (the MX FFN writes
// zero rows of h and yp there whatever they hold).
__global__ void __launch_bounds__(kQWarps * 32)
dispatch_mx_kernel(const uint4* __restrict__ x, uint8_t* __restrict__ xq, uint8_t* __restrict__ xs, int T, int K,
                   int d, int64_t rows_cap, WsPtrs ws) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t bad = 0;
    for (int t = blockIdx.x * kQWarps + warp; t < T; t += gridDim.x * kQWarps) {
        int my_row = -1;
        if (lane < K) {
            my_row = ws.row_of[(int64_t)t * K + lane];
            if (my_row < 0 || my_row >= rows_cap) { bad = 1; my_row = -1; }
        }
        for (int seg = 0; seg < d / 256; ++seg) {
            const int64_t col = (int64_t)seg * 256 + lane * 8;
            const uint4 v = __ldg(x + ((int64_t)t * d + col) / 8);
            const uint32_t s = group_scale<8u>(amax8(v));
            const uint2 c = e4m3x8(v, mx_inv_scale(s));
            for (int k = 0; k < K; ++k) {
                const int row = __shfl_sync(0xffffffffu, my_row, k);
                if (row < 0) continue;
                *reinterpret_cast<uint2*>(xq + (int64_t)row * d + col) = c;
                if ((lane & 3) == 0) xs[mx_scale_offset(row, col / 32, d)] = (uint8_t)s;
            }
        }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) set_status(ws.header, MOE_DEV_BAD_INDEX);
}

int grid_for(int64_t warps) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (warps + kQWarps - 1) / kQWarps, cap = (int64_t)sms * 8;
    return (int)(want < 1 ? 1 : (want < cap ? want : cap));
}

}  // namespace

cudaError_t launch_mx_quantize(const void* x, int64_t rows, int K, int interleave_F, int fmt, uint8_t* q,
                               uint8_t* sc, cudaStream_t st) {
    if (K % 128 != 0 || rows <= 0) return cudaErrorInvalidValue;
    const int grid = grid_for(rows * ((K + 255) / 256));
    const uint4* x4 = static_cast<const uint4*>(x);
    if (fmt == MOE_MX_W_E2M1)
        mx_quantize_kernel<MOE_MX_W_E2M1><<<grid, kQWarps * 32, 0, st>>>(x4, rows, K, interleave_F, q, sc);
    else if (fmt == MOE_MX_W_E4M3)
        mx_quantize_kernel<MOE_MX_W_E4M3><<<grid, kQWarps * 32, 0, st>>>(x4, rows, K, interleave_F, q, sc);
    else
        return cudaErrorInvalidValue;
    return cudaGetLastError();
}

cudaError_t launch_dispatch_mx(const Shape& s, const void* x, uint8_t* xq, uint8_t* xs, const WsPtrs& ws,
                               cudaStream_t st) {
    if (s.d % 256 != 0 || s.K > 32) return cudaErrorInvalidValue;
    dispatch_mx_kernel<<<grid_for(s.T), kQWarps * 32, 0, st>>>(static_cast<const uint4*>(x), xq, xs, s.T, s.K, s.d,
                                                               s.rows_cap, ws);
    return cudaGetLastError();
}

}  // namespace moe
