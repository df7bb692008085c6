// plan.cu - the on-device greedy replication planner and tile layout (step A4),
// one CTA of 1024 threads.
//
// [MoonEP] "MoonEP routing flow - live", 'Per-expert breakdown': every rank's
// capacity is S*K entries. 'The greedy balance, step by step': each move
// refills the currently hungriest rank in one shot from the currently biggest
// donor; the donor may overshoot into deficit and is refilled by a later move;
// a move slices off the donor's biggest experts; each foreign slice is one
// weight copy.
// [MegaFlux] "MegaFlux: Skew-Resilient MoE Megakernels via Pipelined Expert
// Replication", §3.1 and App. A.1: planning starts from the no-replica
// assignment under a per-GPU replica budget; §3.1 'Problem formulation':
// token blocks of at most beta rows; §3.1 'On-device planning and route
// construction' and App. A.2: a stable per-expert order maps every routed
// assignment to its block.
//
// Readings (shared with the CPU oracle, which is written independently):
// owner(e) = e / (E/R); every tie goes to the lowest index; a slice is the
// tail of the rows the donor still holds of that expert; a receiver that has
// used its budget takes nothing more, and when the hungriest rank can take
// nothing the plan is flagged inexact; pieces are laid out in (rank, expert)
// order, each padded to whole tiles at a tile-aligned row.
//
// Phases: (A) per-expert totals and per-chunk exclusive offsets from the
// top-k kernel's chunk histograms (all threads); (B) the greedy moves (warp
// 0, warp-shuffle arg-min/arg-max); (C) per-rank piece lists and block table
// (one thread per rank, block scans for offsets); (D) per-expert piece index
// in start order and the expert-major block schedule the GEMM walks.
#include <limits.h>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kThreads = 1024;

// Exclusive scan of one int per thread over the whole CTA (1024 threads).
// Returns the exclusive prefix; *total receives the sum. tmp: 32 ints.
__device__ int block_excl_scan(int v, int* tmp, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
    }
    if (lane == 31) tmp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = tmp[lane];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, off);
            if (lane >= off) w += y;
        }
        tmp[lane] = w;   // inclusive warp totals
    }
    __syncthreads();
    const int base = warp > 0 ? tmp[warp - 1] : 0;
    const int tot = tmp[31];
    __syncthreads();
    if (total) *total = tot;
    return base + x - v;
}

struct PlanArgs {
    int E, R, per, tile, budget, n_chunks, G;
    int C;
    int max_rep;
    int plan_mode;
    int max_pairs;   // length of the fused FFN's readiness counters
    int sort_off;    // byte offset in dynamic shared memory of the partial-block sort scratch
    int packed;      // loads fit the greedy's packed (value, index) keys
};

// ---------------------------------------------------------------- warp helpers
// Minimum of (v, i) over the warp, lowest i on ties.
__device__ __forceinline__ void warp_min_vi(int& v, int& i) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const int ov = __shfl_xor_sync(0xffffffffu, v, off);
        const int oi = __shfl_xor_sync(0xffffffffu, i, off);
        if (ov < v || (ov == v && oi < i)) { v = ov; i = oi; }
    }
}

// Maximum of v over the warp, lowest i on ties.
__device__ __forceinline__ void warp_max_vi(int& v, int& i) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const int ov = __shfl_xor_sync(0xffffffffu, v, off);
        const int oi = __shfl_xor_sync(0xffffffffu, i, off);
        if (ov > v || (ov == v && oi < i)) { v = ov; i = oi; }
    }
}

// One greedy candidate of the block-granular planner ([MegaFlux] §3.1
// 'Bounded greedy search', App. A.1), run by one warp on its own copy of the
// assignment q[e*R + r] (blocks of expert e on rank r). prio 0: donors by
// decreasing overload; prio 1: by largest remaining home-expert blocks.
// fan 0: at most one new copy per expert per round; fan 1: any number.
__device__ void block_candidate(int prio, int fan, const int32_t* b, int E, int R, int per, int budget, int tau,
                                int16_t* q, int32_t* load, int32_t* nrep, uint8_t* newcopy, int32_t* dkey,
                                int32_t* ekey, int32_t* moves_out) {
    const int lane = threadIdx.x & 31;
    for (int i = lane; i < E * R; i += 32) q[i] = 0;
    __syncwarp();
    for (int e = lane; e < E; e += 32) q[e * R + e / per] = (int16_t)b[e];
    for (int r = lane; r < R; r += 32) {
        int sum = 0;
        for (int e = r * per; e < (r + 1) * per; ++e) sum += b[e];
        load[r] = sum;
        nrep[r] = 0;
    }
    __syncwarp();
    int moves = 0;
    for (int round = 0; round < budget + 2; ++round) {
        int moved = 0;
        for (int e = lane; e < E; e += 32) newcopy[e] = 0;
        for (int r = lane; r < R; r += 32) {
            int key = -1;
            if (load[r] > tau) {
                if (prio == 0) key = load[r] - tau;
                else {
                    key = 0;
                    for (int e = r * per; e < (r + 1) * per; ++e) key = max(key, (int)q[e * R + r]);
                }
            }
            dkey[r] = key;
        }
        __syncwarp();
        for (;;) {
            // next donor of this round: largest key, lowest rank on ties
            int bk = -1, br = INT_MAX;
            for (int r = lane; r < R; r += 32) if (dkey[r] > bk) { bk = dkey[r]; br = r; }
            warp_max_vi(bk, br);
            if (bk < 0) break;
            const int d = br;
            __syncwarp();
            if (lane == 0) dkey[d] = -1;
            for (int i = lane; i < per; i += 32) ekey[i] = q[(d * per + i) * R + d];
            __syncwarp();
            for (;;) {
                if (load[d] <= tau) break;
                // the donor's next home expert: most remaining blocks, lowest id on ties
                int bv = -1, bi = INT_MAX;
                for (int i = lane; i < per; i += 32) if (ekey[i] > bv) { bv = ekey[i]; bi = i; }
                warp_max_vi(bv, bi);
                if (bv < 0) break;
                __syncwarp();
                if (lane == 0) ekey[bi] = -1;
                __syncwarp();
                const int e = d * per + bi;
                while (load[d] > tau && q[e * R + d] > 0) {
                    // an existing copy below tau, least loaded first
                    int lv = INT_MAX, lr = INT_MAX;
                    for (int r = lane; r < R; r += 32)
                        if (r != d && q[e * R + r] > 0 && load[r] < tau && load[r] < lv) { lv = load[r]; lr = r; }
                    warp_min_vi(lv, lr);
                    if (lv == INT_MAX) {
                        if (fan == 0 && newcopy[e]) break;
                        for (int r = lane; r < R; r += 32)
                            if (r != d && q[e * R + r] == 0 && load[r] < tau && nrep[r] < budget && load[r] < lv) {
                                lv = load[r];
                                lr = r;
                            }
                        warp_min_vi(lv, lr);
                        if (lv == INT_MAX) break;
                        __syncwarp();
                        if (lane == 0) { nrep[lr] += 1; newcopy[e] = 1; }
                    }
                    const int rcv = lr;
                    int x = q[e * R + d];
                    x = min(x, load[d] - tau);
                    x = min(x, tau - load[rcv]);
                    __syncwarp();
                    if (lane == 0) {
                        q[e * R + d] = (int16_t)(q[e * R + d] - x);
                        q[e * R + rcv] = (int16_t)(q[e * R + rcv] + x);
                        load[d] -= x;
                        load[rcv] += x;
                    }
                    __syncwarp();
                    moved += x;
                    moves += 1;
                }
            }
        }
        if (moved == 0) break;
    }
    if (lane == 0) *moves_out = moves;
}

__global__ void __launch_bounds__(kThreads, 1)
plan_kernel(PlanArgs a, int32_t* __restrict__ counts_out, WsPtrs ws) {
    pdl_wait();
    pdl_trigger();
    extern __shared__ int32_t sm[];
    const int E = a.E, R = a.R;
    int32_t* part = sm;                              // [G*E]
    int32_t* cnt = part + a.G * E;                   // [E]
    int32_t* rem = cnt + E;                          // [E]
    int32_t* own_pid = rem + E;                      // [E]
    int32_t* L = own_pid + E;                        // [R]
    int32_t* used = L + R;                           // [R]
    int32_t* rep = used + R;                         // [max_rep][5]: rank, expert, start, len, pid
    int32_t* pfb = rep + 5 * a.max_rep;              // [max_pieces+1]: first block of each piece
    int32_t* pq = pfb + (E + a.max_rep + 1);         // [max_pieces][4]: expert, rank, len, row0
    int32_t* tmp = pq + 4 * (E + a.max_rep);         // [32]
    // block-granular planner (plan_mode 1) state
    int32_t* bl = tmp + 32;                           // [E] blocks per expert
    int32_t* cload = bl + E;                          // [4][R]
    int32_t* cnrep = cload + 4 * R;                   // [4][R]
    int32_t* cdkey = cnrep + 4 * R;                   // [4][R]
    int32_t* cekey = cdkey + 4 * R;                   // [4][per]
    int32_t* cmoves = cekey + 4 * a.per;              // [4]
    int32_t* plist = cmoves + 4;                      // [max_rep][2]: (e*R + r, blocks at pass entry)
    uint8_t* cnew = reinterpret_cast<uint8_t*>(plist + 2 * a.max_rep);        // [4][E]
    int16_t* cq = reinterpret_cast<int16_t*>(cnew + ((4 * E + 15) & ~15));   // [4][E*R]
    __shared__ uint32_t s_status;
    __shared__ int s_moves, s_nrep;
    __shared__ int s_tot_blocks, s_tau, s_best;   // block-granular planner
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // ---------------- (A) totals and per-chunk offsets
    if (tid == 0) s_status = 0;
    __syncthreads();
    {
        uint32_t f = 0;
        for (int c = tid; c < a.n_chunks; c += kThreads) f |= ws.chunk_flags[c];
        if (f) atomicOr(&s_status, f);
    }
    auto chunk_count = [&](int c, int e) -> int { return __ldg(ws.chunk_counts + (int64_t)c * E + e); };
    const int g = tid / E, e0 = tid % E;
    if (g < a.G) {
        const int c0 = (int)((int64_t)g * a.n_chunks / a.G), c1 = (int)((int64_t)(g + 1) * a.n_chunks / a.G);
        int s = 0;
#pragma unroll 8
        for (int c = c0; c < c1; ++c) s += chunk_count(c, e0);
        part[g * E + e0] = s;
    }
    __syncthreads();
    if (tid < E) {
        int run = 0;
        for (int gg = 0; gg < a.G; ++gg) {
            const int t = part[gg * E + tid];
            part[gg * E + tid] = run;
            run += t;
        }
        cnt[tid] = run;
        rem[tid] = run;
        own_pid[tid] = -1;
        counts_out[tid] = run;
    }
    __syncthreads();
    if (g < a.G) {
        const int c0 = (int)((int64_t)g * a.n_chunks / a.G), c1 = (int)((int64_t)(g + 1) * a.n_chunks / a.G);
        int run = part[g * E + e0];
#pragma unroll 8
        for (int c = c0; c < c1; ++c) {
            ws.chunk_base[(int64_t)c * E + e0] = run;
            run += chunk_count(c, e0);
        }
    }
    if (tid < R) {
        int s = 0;
        for (int e = tid * a.per; e < (tid + 1) * a.per; ++e) s += cnt[e];
        L[tid] = s;
        used[tid] = 0;
    }
    __syncthreads();

    // ---------------- (B) greedy moves, warp 0
    if (a.plan_mode == MOE_PLAN_EXACT && warp == 0) {
        const int C = a.C;
        const int cap = R * R + E;
        int moves = 0, nrep = 0;
        uint32_t st = 0;
        for (;;) {
            // hungriest rank: lowest load, lowest index on ties; biggest donor: highest
            // load, lowest index on ties. With loads below 2^23 both are one warp
            // reduction of a packed key (load above the rank's 8 bits).
            int mv = INT_MAX, mr = INT_MAX;
            int xv = INT_MIN, xr = INT_MAX;
            if (a.packed) {
                uint32_t kmin = 0xffffffffu, kmax = 0u;
                for (int r = lane; r < R; r += 32) {
                    const uint32_t l = (uint32_t)L[r];
                    kmin = min(kmin, (l << 8) | (uint32_t)r);
                    kmax = max(kmax, (l << 8) | (uint32_t)(255 - r));
                }
                kmin = __reduce_min_sync(0xffffffffu, kmin);
                kmax = __reduce_max_sync(0xffffffffu, kmax);
                mv = (int)(kmin >> 8); mr = (int)(kmin & 255u);
                xv = (int)(kmax >> 8); xr = 255 - (int)(kmax & 255u);
            } else {
            for (int r = lane; r < R; r += 32) {
                const int l = L[r];
                if (l < mv) { mv = l; mr = r; }
                if (l > xv) { xv = l; xr = r; }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const int ov = __shfl_xor_sync(0xffffffffu, mv, off);
                const int orr = __shfl_xor_sync(0xffffffffu, mr, off);
                if (ov < mv || (ov == mv && orr < mr)) { mv = ov; mr = orr; }
                const int pv = __shfl_xor_sync(0xffffffffu, xv, off);
                const int pr = __shfl_xor_sync(0xffffffffu, xr, off);
                if (pv > xv || (pv == xv && pr < xr)) { xv = pv; xr = pr; }
            }
            }
            const int recv = mr, donor = xr;
            if (mv >= C) break;
            if (moves == cap) { st |= MOE_DEV_PLAN_INEXACT; break; }
            int need = C - mv;
            int gave = 0;
            while (need > 0) {
                // donor's biggest remaining expert, lowest id on ties
                int bv = 0, be = INT_MAX;
                if (a.packed) {
                    // remaining entries above the expert's 10-bit position among the donor's
                    uint32_t kb = 0u;
                    for (int e = donor * a.per + lane; e < (donor + 1) * a.per; e += 32) {
                        const int r_ = rem[e];
                        if (r_ > 0) kb = max(kb, ((uint32_t)r_ << 10) | (uint32_t)(1023 - (e - donor * a.per)));
                    }
                    kb = __reduce_max_sync(0xffffffffu, kb);
                    bv = (int)(kb >> 10);
                    be = donor * a.per + 1023 - (int)(kb & 1023u);
                } else {
                for (int e = donor * a.per + lane; e < (donor + 1) * a.per; e += 32) {
                    const int r_ = rem[e];
                    if (r_ > bv) { bv = r_; be = e; }
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    const int ov = __shfl_xor_sync(0xffffffffu, bv, off);
                    const int oe = __shfl_xor_sync(0xffffffffu, be, off);
                    if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; }
                }
                }
                if (bv <= 0) break;                       // donor holds nothing
                if (used[recv] >= a.budget) break;        // no replica slot left
                if (nrep >= a.max_rep) { st |= MOE_DEV_PLAN_INEXACT; break; }
                const int x = bv < need ? bv : need;
                if (lane == 0) {
                    int32_t* q = rep + 5 * nrep;
                    q[0] = recv; q[1] = be; q[2] = bv - x; q[3] = x; q[4] = -1;
                    used[recv] += 1;
                    rem[be] -= x;
                    L[donor] -= x;
                    L[recv] += x;
                }
                __syncwarp();
                ++nrep;
                need -= x;
                gave += x;
            }
            if (gave == 0) { st |= MOE_DEV_PLAN_INEXACT; break; }
            ++moves;
        }
        if (lane == 0) {
            s_moves = moves;
            s_nrep = nrep;
            if (st) atomicOr(&s_status, st);
        }
    }
    if (a.plan_mode == MOE_PLAN_BLOCKS) {
        // ---------------- (B') block-granular planner ([MegaFlux] §3.1, App. A.1, A.2)
        int tot_blocks = 0;
        for (int e = tid; e < E; e += kThreads) bl[e] = (cnt[e] + a.tile - 1) / a.tile;
        __syncthreads();
        if (warp == 0) {
            int sum = 0;
            for (int e = lane; e < E; e += 32) sum += bl[e];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
            if (lane == 0) s_tot_blocks = sum;
        }
        __syncthreads();
        tot_blocks = s_tot_blocks;
        const int tau = (tot_blocks + R - 1) / R;
        if (warp < 4) {
            block_candidate(warp / 2, warp % 2, bl, E, R, a.per, a.budget, tau, cq + (size_t)warp * E * R,
                            cload + warp * R, cnrep + warp * R, cnew + warp * E, cdkey + warp * R,
                            cekey + warp * a.per, cmoves + warp);
        }
        __syncthreads();
        if (warp == 0) {
            // the winner: smallest maximum load, then fewest replicas, then candidate order
            int best = 0, best_max = INT_MAX, best_reps = INT_MAX;
            for (int c = 0; c < 4; ++c) {
                int mx = 0, reps = 0;
                for (int r = lane; r < R; r += 32) { mx = max(mx, cload[c * R + r]); reps += cnrep[c * R + r]; }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, off));
                    reps += __shfl_xor_sync(0xffffffffu, reps, off);
                }
                if (mx < best_max || (mx == best_max && reps < best_reps)) { best = c; best_max = mx; best_reps = reps; }
            }
            int16_t* q = cq + (size_t)best * E * R;
            int32_t* load = cload + best * R;
            int32_t* nr = cnrep + best * R;
            int moves = cmoves[best];
            // pruning: replicas in increasing blocks at pass entry (then e, r)
            int np = 0;
            for (int base = 0; base < E * R; base += 32) {
                const int i = base + lane;
                const bool is_rep = i < E * R && (i % R) != (i / R) / a.per && q[i] > 0;
                const unsigned m = __ballot_sync(0xffffffffu, is_rep);
                if (is_rep) {
                    const int at = np + __popc(m & ((1u << lane) - 1u));
                    plist[2 * at] = i;
                    plist[2 * at + 1] = q[i];
                }
                np += __popc(m);
            }
            __syncwarp();
            for (int k = 0; k < np; ++k) {
                // next replica: smallest (blocks at entry, e*R + r) among the unvisited
                int kv = INT_MAX, ki = INT_MAX;
                for (int j = lane; j < np; j += 32) {
                    const int v = plist[2 * j + 1], id = plist[2 * j];
                    if (v >= 0 && (v < kv || (v == kv && id < ki))) { kv = v; ki = id; }
                }
                warp_min_vi(kv, ki);
                for (int j = lane; j < np; j += 32) if (plist[2 * j] == ki) plist[2 * j + 1] = -1;
                __syncwarp();
                const int e = ki / R, r = ki % R, o = e / a.per;
                const int x = q[ki];
                if (x == 0) continue;
                int tgt = -1;
                if (load[o] + x <= best_max) {
                    tgt = o;
                } else {
                    int lv = INT_MAX, lr = INT_MAX;
                    for (int c2 = lane; c2 < R; c2 += 32)
                        if (c2 != r && c2 != o && q[e * R + c2] > 0 && load[c2] + x <= best_max && load[c2] < lv) {
                            lv = load[c2];
                            lr = c2;
                        }
                    warp_min_vi(lv, lr);
                    if (lv != INT_MAX) tgt = lr;
                }
                if (tgt < 0) continue;
                __syncwarp();
                if (lane == 0) {
                    q[ki] = 0;
                    q[e * R + tgt] = (int16_t)(q[e * R + tgt] + x);
                    load[r] -= x;
                    load[tgt] += x;
                    nr[r] -= 1;
                }
                __syncwarp();
                moves += 1;
            }
            // refinement: single blocks from the most- to the least-loaded rank
            for (int it = 0; it < tot_blocks; ++it) {
                int hv = INT_MIN, hr = INT_MAX, lv = INT_MAX, lr = INT_MAX;
                for (int r = lane; r < R; r += 32) {
                    if (load[r] > hv) { hv = load[r]; hr = r; }
                    if (load[r] < lv) { lv = load[r]; lr = r; }
                }
                warp_max_vi(hv, hr);
                warp_min_vi(lv, lr);
                if (hv - lv <= 1) break;
                int es = INT_MAX;
                for (int e = lane; e < E; e += 32)
                    if (q[e * R + hr] > 0 && (e / a.per == lr || q[e * R + lr] > 0)) { es = e; break; }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) es = min(es, __shfl_xor_sync(0xffffffffu, es, off));
                if (es == INT_MAX) break;
                __syncwarp();
                if (lane == 0) {
                    q[es * R + hr] = (int16_t)(q[es * R + hr] - 1);
                    q[es * R + lr] = (int16_t)(q[es * R + lr] + 1);
                    load[hr] -= 1;
                    load[lr] += 1;
                }
                __syncwarp();
                moves += 1;
            }
            if (lane == 0) {
                s_moves = moves;
                s_best = best;
                s_tau = tau;
            }
        }
        __syncthreads();
        const int best = s_best;
        const int16_t* q = cq + (size_t)best * E * R;
        // materialise: the owner takes the first blocks of each expert's list,
        // then the other ranks in increasing index; replica slices are listed
        // per expert in decreasing start (the order the layout phase expects)
        int nrep_e = 0;
        if (tid < E) for (int r = 0; r < R; ++r) nrep_e += (r != tid / a.per && q[tid * R + r] > 0);
        int tot_rep;
        const int rep_off = block_excl_scan(tid < E ? nrep_e : 0, tmp, &tot_rep);
        if (tid < R) used[tid] = 0;
        __syncthreads();
        if (tid < E) {
            const int e = tid, o = e / a.per, ce = cnt[e];
            const int owner_blocks = q[e * R + o];
            rem[e] = min(owner_blocks * a.tile, ce);
            int off = owner_blocks;
            int k = rep_off + nrep_e;   // fill from the end: decreasing start
            for (int r = 0; r < R; ++r) {
                if (r == o || q[e * R + r] == 0) continue;
                const int n = q[e * R + r];
                const int start = off * a.tile;
                const int end = min((off + n) * a.tile, ce);
                int32_t* Q = rep + 5 * (--k);
                Q[0] = r; Q[1] = e; Q[2] = start; Q[3] = end - start; Q[4] = -1;
                atomicAdd(&used[r], 1);
                off += n;
            }
        }
        if (tid == 0) s_nrep = tot_rep;
    }
    __syncthreads();
    const int nrep = s_nrep;

    // ---------------- (C) per-rank pieces and blocks
    // pass 1: counts per rank (thread r); replica slices of r sorted by expert
    int my_rep[kMaxBudget];
    int nr = 0, np_r = 0, nb_r = 0, rows_r = 0;
    if (tid < R) {
        for (int i = 0; i < nrep; ++i) {
            if (rep[5 * i] != tid) continue;
            int j = nr++;
            while (j > 0 && rep[5 * my_rep[j - 1] + 1] > rep[5 * i + 1]) { my_rep[j] = my_rep[j - 1]; --j; }
            my_rep[j] = i;
        }
        for (int k = 0; k < nr; ++k) {
            const int len = rep[5 * my_rep[k] + 3];
            const int nt = (len + a.tile - 1) / a.tile;
            np_r += 1; nb_r += nt; rows_r += nt * a.tile;
        }
        for (int e = tid * a.per; e < (tid + 1) * a.per; ++e) {
            if (rem[e] > 0) {
                const int nt = (rem[e] + a.tile - 1) / a.tile;
                np_r += 1; nb_r += nt; rows_r += nt * a.tile;
            }
        }
    }
    int tot_p, tot_b, tot_rows;
    const int p_off = block_excl_scan(tid < R ? np_r : 0, tmp, &tot_p);
    const int b_off = block_excl_scan(tid < R ? nb_r : 0, tmp, &tot_b);
    const int r_off = block_excl_scan(tid < R ? rows_r : 0, tmp, &tot_rows);
    if (tid < R) {
        // pass 2: merge owned experts (ascending) with replica slices (ascending)
        int pid = p_off, bid = b_off, row = r_off, load = 0;
        int k = 0;
        int e = tid * a.per;
        const int e_end = (tid + 1) * a.per;
        for (;;) {
            // next piece in expert order
            int pe = INT_MAX, pstart = 0, plen = 0, rep_i = -1;
            while (e < e_end && rem[e] <= 0) ++e;
            if (e < e_end) { pe = e; pstart = 0; plen = rem[e]; }
            if (k < nr && rep[5 * my_rep[k] + 1] < pe) {
                rep_i = my_rep[k];
                pe = rep[5 * rep_i + 1]; pstart = rep[5 * rep_i + 2]; plen = rep[5 * rep_i + 3];
            }
            if (pe == INT_MAX) break;
            if (rep_i >= 0) { rep[5 * rep_i + 4] = pid; ++k; }
            else { own_pid[e] = pid; ++e; }
            int32_t* P = ws.pieces + (int64_t)kPieceInts * pid;
            P[0] = pe; P[1] = tid; P[2] = pstart; P[3] = plen; P[4] = row;
            pfb[pid] = bid;
            pq[4 * pid] = pe; pq[4 * pid + 1] = tid; pq[4 * pid + 2] = plen; pq[4 * pid + 3] = row;
            const int nt = (plen + a.tile - 1) / a.tile;
            bid += nt;
            row += nt * a.tile;
            load += plen;
            ++pid;
        }
        ws.rank_load[tid] = load;
        ws.rank_replicas[tid] = used[tid];
        ws.rank_row0[tid] = r_off;
        if (tid == R - 1) ws.rank_row0[R] = row;
    }
    if (tid == 0) pfb[tot_p] = tot_b;
    __syncthreads();
    // blocks of every piece, written by the whole CTA: block b belongs to the
    // last piece whose first block is <= b
    for (int b = tid; b < tot_b; b += kThreads) {
        int lo = 0, hi = tot_p - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (pfb[mid] <= b) lo = mid; else hi = mid - 1;
        }
        const int i = b - pfb[lo];
        const int v = pq[4 * lo + 2] - i * a.tile;
        int32_t* B = ws.blocks + (int64_t)kBlockInts * b;
        B[0] = pq[4 * lo]; B[1] = pq[4 * lo + 3] + i * a.tile; B[2] = v < a.tile ? v : a.tile; B[3] = pq[4 * lo + 1];
    }
    // padding rows (the tail of each piece's last tile) map to no token
    for (int p = warp; p < tot_p; p += kThreads / 32) {
        const int len = pq[4 * p + 2], row0 = pq[4 * p + 3];
        const int padded = (len + a.tile - 1) / a.tile * a.tile;
        for (int r = row0 + len + lane; r < row0 + padded; r += 32) ws.src_of[r] = -1;
    }

    // ---------------- (D) per-expert piece index (start order) and block schedule
    int np_e = 0, nb_e = 0;
    if (tid < E) {
        if (own_pid[tid] >= 0) { np_e = 1; nb_e = (rem[tid] + a.tile - 1) / a.tile; }
        for (int i = 0; i < nrep; ++i) {
            if (rep[5 * i + 1] != tid) continue;
            np_e += 1;
            nb_e += (rep[5 * i + 3] + a.tile - 1) / a.tile;
        }
    }
    int dummy;
    const int ep_off = block_excl_scan(tid < E ? np_e : 0, tmp, &dummy);
    const int eb_off = block_excl_scan(tid < E ? nb_e : 0, tmp, &dummy);
    if (tid < E) {
        ws.exp_piece_off[tid] = ep_off;
        ws.sched_off[tid] = eb_off;
        if (tid == E - 1) { ws.exp_piece_off[E] = ep_off + np_e; ws.sched_off[E] = eb_off + nb_e; }
        int pi = ep_off, bi = eb_off;
        // The expert's schedule lists its whole blocks first, then the partial
        // last block of each piece, larger first (ties in start order), so the
        // GEMM's consecutive block pairs hold blocks of about the same size.
        // Pieces in start order: the owner's prefix starts at 0; later slices
        // were cut from the tail, so reverse creation order is ascending start.
        if (own_pid[tid] >= 0) {
            const int pid = own_pid[tid];
            ws.exp_piece_idx[pi++] = pid;
            for (int i = 0; i < rem[tid] / a.tile; ++i) ws.sched[bi++] = pfb[pid] + i;
        }
        for (int i = nrep - 1; i >= 0; --i) {
            if (rep[5 * i + 1] != tid) continue;
            const int pid = rep[5 * i + 4];
            ws.exp_piece_idx[pi++] = pid;
            for (int j = 0; j < rep[5 * i + 3] / a.tile; ++j) ws.sched[bi++] = pfb[pid] + j;
        }
        // partial last blocks: insertion-sorted by their valid rows (stable) in this
        // expert's own stretch of shared scratch (one slot per piece of the expert)
        int32_t* srt = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(sm) + a.sort_off) + ep_off;
        int np_part = 0;
        auto add_partial = [&](int pid, int len) {
            const int v = len % a.tile;
            if (v == 0) return;
            int k = np_part++;
            while (k > 0 && pq[4 * srt[k - 1] + 2] % a.tile < v) {
                srt[k] = srt[k - 1];
                --k;
            }
            srt[k] = pid;
        };
        if (own_pid[tid] >= 0) add_partial(own_pid[tid], rem[tid]);
        for (int i = nrep - 1; i >= 0; --i)
            if (rep[5 * i + 1] == tid) add_partial(rep[5 * i + 4], rep[5 * i + 3]);
        for (int k = 0; k < np_part; ++k) ws.sched[bi++] = pfb[srt[k]] + pq[4 * srt[k] + 2] / a.tile;
    }
    if (tid == 0) {
        ws.header[H_STATUS] = s_status;
        ws.header[H_NPIECES] = (uint32_t)tot_p;
        ws.header[H_NBLOCKS] = (uint32_t)tot_b;
        ws.header[H_TOTAL_ROWS] = (uint32_t)tot_rows;
        ws.header[H_MOVES] = (uint32_t)s_moves;
        ws.header[H_REPLICAS] = (uint32_t)nrep;
        ws.header[H_TAU] = a.plan_mode == MOE_PLAN_BLOCKS ? (uint32_t)s_tau : 0u;
        ws.header[H_CANDIDATE] = a.plan_mode == MOE_PLAN_BLOCKS ? (uint32_t)s_best : 0u;
        for (int q = 0; q < kGemmQWords; ++q) ws.gemm_q[q] = 0;   // fresh GEMM work queues
    }
    for (int q = tid; q < a.max_pairs; q += blockDim.x) ws.pair_ready[q] = 0;   // and readiness counters
}

}  // namespace

cudaError_t launch_plan(const Shape& s, int32_t* counts_out, const WsPtrs& ws, cudaStream_t st) {
    PlanArgs a;
    a.E = s.E; a.R = s.R; a.per = s.per; a.tile = s.tile; a.budget = s.budget;
    a.n_chunks = s.n_chunks;
    int G = kThreads / s.E;
    if (G < 1) G = 1;
    if (G > s.n_chunks) G = s.n_chunks;
    a.G = G;
    a.C = (int)s.C;
    a.max_rep = s.R * s.budget;
    a.plan_mode = s.plan_mode;
    a.max_pairs = (int)max_pairs(s);
    size_t smem = sizeof(int32_t) * ((size_t)G * s.E + 3 * s.E + 2 * s.R + 5 * a.max_rep +
                                     5 * (s.E + a.max_rep) + 1 + 32);
    if (s.plan_mode == MOE_PLAN_BLOCKS)
        smem += sizeof(int32_t) * ((size_t)s.E + 12 * s.R + 4 * s.per + 4 + 2 * a.max_rep) +
                (((size_t)4 * s.E + 15) & ~(size_t)15) + sizeof(int16_t) * 4 * (size_t)s.E * s.R;
    smem = (smem + 15) & ~(size_t)15;
    a.sort_off = (int)smem;                                   // one int per piece
    smem += sizeof(int32_t) * ((size_t)s.E + a.max_rep);
    smem = (smem + 15) & ~(size_t)15;
    // packed greedy keys: a rank's load and an expert's count stay below 2^22
    a.packed = s.N < ((int64_t)1 << 22) && s.R <= 256 && s.per <= 1024 ? 1 : 0;
    cudaError_t err = cudaFuncSetAttribute(plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
    if (err != cudaSuccess) return err;
    return launch_pdl(plan_kernel, dim3(1), dim3(kThreads), smem, st, a, counts_out, ws);
}

}  // namespace moe
