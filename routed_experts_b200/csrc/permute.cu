// permute.cu - row maps (step A5) and the dispatch gather into the expert-major,
// tile-padded buffer (step A6).
//
// [MegaFlux] "MegaFlux: Skew-Resilient MoE Megakernels via Pipelined Expert
// Replication", App. A.2 'Mapping blocks to routed assignments': within each
// expert, routed assignments are ordered by source rank and then local
// (token, top-k position) and cut into the planned blocks. With source rank
// t / S this is plain (t, k) order, so pos(t,k) is the number of earlier
// entries that chose the same expert, and the entry lands in the piece of its
// expert whose [start, start+len) holds pos.
//
// Ranking is order-preserving and deterministic: one warp walks its
// 32-token chunk in (t, k) order, 32 entries at a time; __match_any_sync
// groups lanes that chose the same expert, a lane's rank inside its group is
// the popcount of the group's lanes below it, and the group leader advances
// the warp's per-expert counter, which starts at the chunk's exclusive offset
// from the planner. No slot is claimed with atomics.
//
// [MegaFlux] §1: routed activations travel to the ranks computing their
// experts. On one GPU that is a copy of token rows, done as a scatter: one
// warp per token reads its row of x once (16-byte vectors) and stores it to
// the K rows the row map names, so x is read from memory once even when it
// does not fit in L2. Padding rows of xp are not written: each output
// element of the expert FFN depends on its own token row alone, so nothing
// they hold reaches a valid row of h or yp.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kRmWarps = 4;

__global__ void __launch_bounds__(kRmWarps * 32)
row_maps_kernel(const int32_t* __restrict__ idx, int T, int K, int E, int n_chunks, int max_pieces, WsPtrs ws) {
    pdl_wait();
    pdl_trigger();
    extern __shared__ int32_t sm_rm[];
    int32_t* s_poff = sm_rm;                       // [E+1] first piece of each expert (start order)
    int4* s_piece = reinterpret_cast<int4*>(s_poff + ((E + 1 + 3) & ~3));   // [n_pieces]: start, len, row0
    int32_t* base_all = reinterpret_cast<int32_t*>(s_piece + max_pieces);  // [kRmWarps][E]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // the piece tables, in expert/start order, staged once per CTA
    const int n_pieces = (int)ws.header[H_NPIECES];
    for (int e = threadIdx.x; e <= E; e += blockDim.x) s_poff[e] = ws.exp_piece_off[e];
    for (int p = threadIdx.x; p < n_pieces; p += blockDim.x) {
        const int32_t* P = ws.pieces + (int64_t)kPieceInts * ws.exp_piece_idx[p];
        s_piece[p] = make_int4(P[2], P[3], P[4], 0);
    }
    __syncthreads();
    const int chunk = blockIdx.x * kRmWarps + warp;
    if (chunk >= n_chunks) return;           // whole warp leaves; no CTA-wide barrier below
    int32_t* base = base_all + warp * E;
    for (int e = lane; e < E; e += 32) base[e] = ws.chunk_base[(int64_t)chunk * E + e];
    __syncwarp();
    const int64_t i0 = (int64_t)chunk * kTokPerChunk * K;
    const int64_t t1 = min((int64_t)T, (int64_t)(chunk + 1) * kTokPerChunk);
    const int64_t i1 = t1 * K;
    uint32_t bad = 0;
    // the chunk's expert ids, loaded up front (a full chunk is K rounds of 32)
    int ev[kMaxK];
#pragma unroll
    for (int r = 0; r < kMaxK; ++r) {
        const int64_t i = i0 + (int64_t)r * 32 + lane;
        ev[r] = (r < K && i < i1) ? __ldg(idx + i) : -1;
    }
#pragma unroll
    for (int r = 0; r < kMaxK; ++r) {
        if (r >= K) break;
        const int64_t i = i0 + (int64_t)r * 32 + lane;
        const bool valid = i < i1;
        int e = valid ? ev[r] : -1;
        if (valid && (e < 0 || e >= E)) { bad = 1; e = -2; }
        const bool ok = valid && e >= 0;
        const unsigned m = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(m & ((1u << lane) - 1u));
        const int pos = ok ? base[e] + rank : 0;
        __syncwarp();
        if (ok && lane == __ffs(m) - 1) base[e] += __popc(m);
        __syncwarp();
        if (ok) {
            int row = -1;
            const int p1 = s_poff[e + 1];
            for (int p = s_poff[e]; p < p1; ++p) {
                const int4 P = s_piece[p];
                if (pos < P.x + P.y) { row = P.z + pos - P.x; break; }
            }
            if (row < 0) {
                bad = 1;
            } else {
                ws.row_of[i] = row;
                ws.src_of[row] = (int32_t)(i / K);
            }
        }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) set_status(ws.header, MOE_DEV_BAD_INDEX);
}

constexpr int kGWarps = 8;
constexpr int kUnroll = 8;

__global__ void __launch_bounds__(kGWarps * 32)
dispatch_kernel(const uint4* __restrict__ x, uint4* __restrict__ xp, int T, int K, int nvec, int64_t rows_cap,
                WsPtrs ws) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t bad = 0;
    for (int t = blockIdx.x * kGWarps + warp; t < T; t += gridDim.x * kGWarps) {
        int my_row = -1;
        if (lane < K) {
            my_row = ws.row_of[(int64_t)t * K + lane];
            if (my_row < 0 || my_row >= rows_cap) { bad = 1; my_row = -1; }
        }
        const uint4* src = x + (int64_t)t * nvec;
        for (int v0 = 0; v0 < nvec; v0 += 32 * kUnroll) {
            uint4 buf[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int v = v0 + u * 32 + lane;
                if (v < nvec) buf[u] = __ldg(src + v);
            }
            for (int k = 0; k < K; ++k) {
                const int row = __shfl_sync(0xffffffffu, my_row, k);
                if (row < 0) continue;
                uint4* dst = xp + (int64_t)row * nvec;
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) {
                    const int v = v0 + u * 32 + lane;
                    if (v < nvec) dst[v] = buf[u];
                }
            }
        }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) set_status(ws.header, MOE_DEV_BAD_INDEX);
}

}  // namespace

cudaError_t launch_row_maps(const Shape& s, const int32_t* idx, const WsPtrs& ws, cudaStream_t st) {
    const int grid = (s.n_chunks + kRmWarps - 1) / kRmWarps;
    const size_t smem = sizeof(int32_t) * (((s.E + 1 + 3) & ~3) + kRmWarps * s.E) + sizeof(int4) * s.max_pieces;
    if (smem > 48 * 1024) {
        cudaError_t err = cudaFuncSetAttribute(row_maps_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
    }
    return launch_pdl(row_maps_kernel, dim3(grid), dim3(kRmWarps * 32), smem, st, idx, s.T, s.K, s.E, s.n_chunks,
                      (int)s.max_pieces, ws);
}

cudaError_t launch_gather(const Shape& s, const void* x, void* xp, const WsPtrs& ws,
                          cudaStream_t st) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int nvec = (int)((int64_t)s.d * s.eb / 16);
    int64_t want = (s.T + kGWarps - 1) / kGWarps;
    int64_t cap = (int64_t)sms * 8;
    const int grid = (int)(want < cap ? want : cap);
    if (grid == 0) return cudaSuccess;
    return launch_pdl(dispatch_kernel, dim3(grid), dim3(kGWarps * 32), 0, st, static_cast<const uint4*>(x),
                      static_cast<uint4*>(xp), s.T, s.K, nvec, s.rows_cap, ws);
}

}  // namespace moe
