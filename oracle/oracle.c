/*
 * oracle.c - plain, slow CPU oracle for the skew-resilient routed-expert MoE
 * layer: router top-k and gating, expert-load histogram, greedy replication
 * planner, tile layout, row maps, dispatch, SwiGLU expert FFN and weighted
 * combine, plus a dense compute-every-expert-then-mask reference.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the package smoke check and the
 * benchmark's CPU-baseline leg load this library. It shares no code with the
 * CUDA library and neither one calls the other.
 *
 * Sources, cited by page title and section:
 *   [MegaFlux]  "MegaFlux: Skew-Resilient MoE Megakernels via Pipelined
 *               Expert Replication"
 *   [MoonEP]    "MoonEP routing flow - live" (an explainer of MoonEP's
 *               planning kernel)
 *
 * Where the pages leave a step open, the reading taken is marked READING.
 * Single-threaded plain loops; floating point in fp64. Rounding points
 * (round_mode) mirror where the GPU path stores a narrower type:
 *   ORC_ROUND_NONE  no rounding anywhere (pure fp64),
 *   ORC_ROUND_F32   H, Yp and out stored as fp32,
 *   ORC_ROUND_BF16  H, Yp and out rounded to bf16 (nearest even).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORC_BF16 = 0, ORC_FP32 = 1 };
enum { ORC_GATE_SOFTMAX_TOPK = 0, ORC_GATE_SIGMOID_TOPK = 1 };
enum { ORC_ROUND_NONE = 0, ORC_ROUND_F32 = 1, ORC_ROUND_BF16 = 2 };
enum { ORC_PLAN_INEXACT = 1u };
enum { ORC_OK = 0, ORC_ERR_ARG = 1, ORC_ERR_INTERNAL = 2 };

typedef struct { int32_t expert, rank, start, len, row0; } orc_piece;
typedef struct { int32_t expert, row0, valid, rank; } orc_block;

/* ---------------------------------------------------------------- numbers */

static double bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Round a double to the nearest bf16 (8 significant bits), ties to even. */
static uint16_t double_to_bf16(double v)
{
    if (v == 0.0) {
        float z = (float)v; /* keeps the sign of zero */
        uint32_t u;
        memcpy(&u, &z, 4);
        return (uint16_t)(u >> 16);
    }
    int e;
    double m = frexp(v, &e);            /* |m| in [0.5, 1) */
    double r = nearbyint(ldexp(m, 8));  /* 8 significant bits, ties to even */
    float f = (float)ldexp(r, e - 8);   /* exact: r has at most 9 bits */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

static double round_as(double v, int round_mode)
{
    if (round_mode == ORC_ROUND_BF16) return bf16_to_double(double_to_bf16(v));
    if (round_mode == ORC_ROUND_F32) return (double)(float)v;
    return v;
}

static double load_elem(const void* p, int64_t i, int dtype)
{
    if (dtype == ORC_BF16) return bf16_to_double(((const uint16_t*)p)[i]);
    return (double)((const float*)p)[i];
}

static void store_elem(void* p, int64_t i, int dtype, double v)
{
    if (dtype == ORC_BF16) ((uint16_t*)p)[i] = double_to_bf16(v);
    else ((float*)p)[i] = (float)v;
}

/* ------------------------------------------------- top-k and gating (A1, A2)
 * [MegaFlux] §1: a learned router selects a small set of experts per token
 * and their outputs are combined by the routing weights; §4.1 "Routing
 * workload construction": each token has k distinct experts.
 * READING: the K largest logits, in descending order, ties to the lower
 * expert id. Gating (softmax or sigmoid, normalised over the chosen k) is
 * taken on the same logits that choose the experts.
 */
int orc_topk_gate(int64_t T, int32_t E, int32_t K, int32_t gating,
                  const float* logits, int32_t* idx, float* w)
{
    if (T < 0 || E <= 0 || K <= 0 || K > E) return ORC_ERR_ARG;
    char* taken = (char*)malloc((size_t)E);
    double* g = (double*)malloc(sizeof(double) * (size_t)K);
    if (!taken || !g) { free(taken); free(g); return ORC_ERR_INTERNAL; }
    for (int64_t t = 0; t < T; ++t) {
        const float* l = logits + t * E;
        memset(taken, 0, (size_t)E);
        for (int k = 0; k < K; ++k) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || l[e] > l[best]) best = e;   /* strict: lower id wins ties */
            }
            taken[best] = 1;
            idx[t * K + k] = best;
        }
        double sum = 0.0;
        for (int k = 0; k < K; ++k) {
            double lk = (double)l[idx[t * K + k]];
            if (gating == ORC_GATE_SOFTMAX_TOPK) {
                g[k] = exp(lk - (double)l[idx[t * K]]);     /* softmax, renormalised over top-k */
            } else {
                g[k] = 1.0 / (1.0 + exp(-lk));              /* sigmoid, normalised over top-k */
            }
            sum += g[k];
        }
        for (int k = 0; k < K; ++k) w[t * K + k] = (float)(g[k] / sum);
    }
    free(taken);
    free(g);
    return ORC_OK;
}

/* ------------------------------------------------- histogram (A3)
 * [MegaFlux] §3.1 and App. A.1: the planner's input is the routing profile,
 * the per-expert load. Here the load is counted in routed entries.
 */
int orc_histogram(int64_t n_entries, int32_t E, const int32_t* idx, int32_t* counts)
{
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t i = 0; i < n_entries; ++i) {
        if (idx[i] < 0 || idx[i] >= E) return ORC_ERR_ARG;
        counts[idx[i]] += 1;
    }
    return ORC_OK;
}

/* ------------------------------------------------- planner (A4) and layout
 * [MoonEP] "Per-expert breakdown": every rank's capacity is S*K entries and
 * its surplus is the sum of its experts' loads minus that capacity.
 * [MoonEP] "The greedy balance, step by step": each move refills the
 * currently hungriest rank in one shot from the currently biggest donor; the
 * donor may overshoot into deficit and is then refilled by a later move; a
 * move slices off the donor's biggest experts; every slice of a foreign
 * expert ships one weight copy.
 * [MegaFlux] §3.1 "Bounded greedy search" / App. A.1: the search starts from
 * the no-replica assignment (every expert on its owner); §4.1: each GPU has
 * capacity for a fixed number of extra replicas (the budget).
 * [MegaFlux] §3.1 "Problem formulation": token blocks of at most beta rows
 * match the FC1/FC2 token tile.
 *
 * READINGS:
 *  - owner(e) = e / (E/R) (contiguous expert ownership).
 *  - hungriest = lowest load, biggest donor = highest load, biggest expert =
 *    largest remaining rows; every tie goes to the lowest index.
 *  - a slice is the tail of the rows the donor still holds of that expert,
 *    so the owner keeps a prefix; pieces of one expert partition its list.
 *  - a receiver that has used its budget takes no new slice; if the
 *    hungriest rank can take nothing, planning stops and the plan is
 *    flagged inexact (still a valid partition of all entries).
 *  - cut points are per entry (every rank gets exactly S*K entries when the
 *    plan is exact); each piece is then padded to whole beta-row tiles at a
 *    beta-aligned row, pieces laid out in (rank, expert) order.
 */
/* Tile layout of a plan given as a table of pieces (rank r computes entries
 * [start, start+len) of expert e's list): pieces in (rank, expert) order,
 * each padded to whole tiles at a tile-aligned row, and one block per tile.
 * [MegaFlux] §3.1 'Problem formulation': blocks of at most beta rows match
 * the FC1/FC2 token tile. */
static void layout_pieces(int32_t E, int32_t R, int32_t tile, const int64_t* p_start,
                          const int64_t* p_len, const int32_t* used, orc_piece* pieces,
                          int32_t* n_pieces, orc_block* blocks, int32_t* n_blocks,
                          int64_t* rank_load, int32_t* rank_replicas, int64_t* rank_row0)
{
    int32_t np = 0, nb = 0;
    int64_t row = 0;
    for (int r = 0; r < R; ++r) {
        rank_row0[r] = row;
        rank_load[r] = 0;
        rank_replicas[r] = used[r];
        for (int e = 0; e < E; ++e) {
            int64_t len = p_len[(size_t)r * E + e];
            if (len == 0) continue;
            orc_piece* p = &pieces[np++];
            p->expert = e;
            p->rank = r;
            p->start = (int32_t)p_start[(size_t)r * E + e];
            p->len = (int32_t)len;
            p->row0 = (int32_t)row;
            int64_t ntiles = (len + tile - 1) / tile;
            for (int64_t i = 0; i < ntiles; ++i) {
                orc_block* b = &blocks[nb++];
                b->expert = e;
                b->row0 = (int32_t)(row + i * tile);
                b->valid = (int32_t)((len - i * tile) < tile ? (len - i * tile) : tile);
                b->rank = r;
            }
            row += ntiles * tile;
            rank_load[r] += len;
        }
    }
    rank_row0[R] = row;
    *n_pieces = np;
    *n_blocks = nb;
}

int orc_plan(int64_t T, int32_t E, int32_t K, int32_t R, int32_t tile, int32_t budget,
             const int32_t* counts,
             orc_piece* pieces, int32_t* n_pieces,
             orc_block* blocks, int32_t* n_blocks,
             int64_t* rank_load, int32_t* rank_replicas, int64_t* rank_row0,
             int32_t* moves_out, uint32_t* status)
{
    if (R <= 0 || E <= 0 || E % R != 0 || T % R != 0 || tile <= 0 || budget < 0)
        return ORC_ERR_ARG;
    const int64_t C = (T / R) * (int64_t)K;       /* per-rank capacity S*K */
    const int32_t per = E / R;                    /* experts owned per rank */

    int64_t* rem = (int64_t*)calloc((size_t)E, sizeof(int64_t));
    int64_t* L = (int64_t*)calloc((size_t)R, sizeof(int64_t));
    int32_t* used = (int32_t*)calloc((size_t)R, sizeof(int32_t));
    int64_t* p_start = (int64_t*)calloc((size_t)R * E, sizeof(int64_t));
    int64_t* p_len = (int64_t*)calloc((size_t)R * E, sizeof(int64_t));
    if (!rem || !L || !used || !p_start || !p_len) {
        free(rem); free(L); free(used); free(p_start); free(p_len);
        return ORC_ERR_INTERNAL;
    }
    int rc = ORC_OK;
    uint32_t st = 0;

    /* no-replica start: every expert's whole list is held by its owner */
    for (int e = 0; e < E; ++e) {
        rem[e] = counts[e];
        L[e / per] += counts[e];
    }

    int32_t moves = 0;
    const int32_t cap = R * R + E;               /* backstop; a move settles a rank */
    for (;;) {
        int recv = 0;
        for (int r = 1; r < R; ++r) if (L[r] < L[recv]) recv = r;
        if (L[recv] >= C) break;                 /* sum is R*C, so all equal C */
        if (moves == cap) { st |= ORC_PLAN_INEXACT; break; }
        int donor = 0;
        for (int r = 1; r < R; ++r) if (L[r] > L[donor]) donor = r;

        int64_t phi_before = 0;
        for (int r = 0; r < R; ++r) phi_before += llabs(L[r] - C);

        int64_t need = C - L[recv];
        int64_t gave = 0;
        while (need > 0) {
            int e_best = -1;
            for (int e = donor * per; e < (donor + 1) * per; ++e) {
                if (rem[e] <= 0) continue;
                if (e_best < 0 || rem[e] > rem[e_best]) e_best = e;
            }
            if (e_best < 0) break;               /* donor has nothing left */
            if (used[recv] >= budget) break;     /* a new replica is not allowed */
            if (p_len[(size_t)recv * E + e_best] != 0) { rc = ORC_ERR_INTERNAL; goto done; }
            int64_t x = rem[e_best] < need ? rem[e_best] : need;
            p_start[(size_t)recv * E + e_best] = rem[e_best] - x;
            p_len[(size_t)recv * E + e_best] = x;
            used[recv] += 1;
            rem[e_best] -= x;
            need -= x;
            L[donor] -= x;
            L[recv] += x;
            gave += x;
        }
        if (gave == 0) { st |= ORC_PLAN_INEXACT; break; }
        moves += 1;

        int64_t phi_after = 0;
        for (int r = 0; r < R; ++r) phi_after += llabs(L[r] - C);
        if (phi_after >= phi_before) { rc = ORC_ERR_INTERNAL; goto done; }
    }

    /* what the owners still hold: a prefix of each expert's list */
    for (int e = 0; e < E; ++e) {
        if (rem[e] > 0) {
            int o = e / per;
            p_start[(size_t)o * E + e] = 0;
            p_len[(size_t)o * E + e] = rem[e];
        }
    }

    layout_pieces(E, R, tile, p_start, p_len, used, pieces, n_pieces, blocks, n_blocks,
                  rank_load, rank_replicas, rank_row0);
    *moves_out = moves;
    *status = st;
done:
    free(rem); free(L); free(used); free(p_start); free(p_len);
    return rc;
}

/* ------------------------------------------------- block-granular planner
 * [MegaFlux] §3.1 'Bounded greedy search', App. A.1 'Candidate construction'
 * and 'Refinement', App. A.2 'Mapping blocks to routed assignments', §4.1
 * (s replica slots per GPU).
 *
 * Load is counted in token blocks: b_e = ceil(c_e / beta), tau =
 * ceil(sum_e b_e / R). Each of four candidates starts from the no-replica
 * assignment q[e][owner(e)] = b_e and runs at most s+2 rounds; a round with
 * no movement ends it. A round visits the over-loaded owners once, in the
 * candidate's donor priority (decreasing overload load-tau, or decreasing
 * largest remaining home-expert block count). A visit scans the donor's home
 * experts by decreasing remaining blocks and moves blocks of each to ranks
 * below tau: first to ranks already holding a copy of the expert, then by
 * opening a new copy on the least-loaded rank with a free replica slot; the
 * visit ends when the donor reaches tau or its scan finishes, an expert's
 * fan-out ends when the donor has no block of it left or no eligible
 * receiver remains. The SINGLE fan-out opens at most one new copy per expert
 * per round, MULTI any number. The candidate with the smallest maximum load
 * wins (ties: fewer replicas, then candidate order). Pruning visits the
 * replicas in increasing block count and moves a replica's whole allocation
 * to the owner, else to the least-loaded other copy, when that copy stays
 * within the winner's maximum load. A bounded pass then moves single blocks
 * from the most- to the least-loaded rank while they share an expert and
 * their loads differ by more than one.
 *
 * READINGS: ties go to the lowest index everywhere; a move carries
 * min(donor blocks of e, donor load - tau, tau - receiver load) blocks (no
 * donor drops below tau, no receiver rises above it); a rank shares an
 * expert when it owns it or holds blocks of it; materialisation cuts each
 * expert's (token, slot)-ordered list into blocks of beta and gives the
 * owner the first q blocks, then the other ranks in increasing index, so only
 * the expert's last block is partial. moves counts greedy transfers, pruning
 * relocations and refinement moves. The plan is never flagged inexact.
 * info: [0] tau, [1] winning candidate (2*priority + fan-out), [2] its
 * maximum load in blocks, [3] replicas in total after refinement.
 */
static void run_candidate(int32_t E, int32_t R, int32_t per, int32_t budget, int64_t tau,
                          const int64_t* b, int prio, int fan, int64_t* q, int64_t* load,
                          int32_t* nrep, int32_t* moves_out, char* newcopy, int32_t* order,
                          int32_t* donors)
{
    int32_t moves = 0;
    for (int e = 0; e < E; ++e)
        for (int r = 0; r < R; ++r) q[(size_t)e * R + r] = (r == e / per) ? b[e] : 0;
    for (int r = 0; r < R; ++r) { load[r] = 0; nrep[r] = 0; }
    for (int e = 0; e < E; ++e) load[e / per] += b[e];

    for (int round = 0; round < budget + 2; ++round) {
        int64_t moved = 0;
        memset(newcopy, 0, (size_t)E);
        /* donors of this round, in priority order (selection sort, stable by index) */
        int nd = 0;
        for (int r = 0; r < R; ++r) if (load[r] > tau) donors[nd++] = r;
        int64_t* key = (int64_t*)malloc(sizeof(int64_t) * (size_t)(nd ? nd : 1));
        for (int i = 0; i < nd; ++i) {
            int r = donors[i];
            if (prio == 0) key[i] = load[r] - tau;
            else {
                int64_t m = 0;
                for (int e = r * per; e < (r + 1) * per; ++e)
                    if (q[(size_t)e * R + r] > m) m = q[(size_t)e * R + r];
                key[i] = m;
            }
        }
        for (int i = 0; i < nd; ++i) {
            int best = i;
            for (int j = i + 1; j < nd; ++j)
                if (key[j] > key[best] || (key[j] == key[best] && donors[j] < donors[best])) best = j;
            int tr = donors[i]; donors[i] = donors[best]; donors[best] = tr;
            int64_t tk = key[i]; key[i] = key[best]; key[best] = tk;
        }
        free(key);
        for (int di = 0; di < nd; ++di) {
            const int d = donors[di];
            if (load[d] <= tau) continue;
            /* home experts by decreasing remaining blocks, at visit start */
            int no = 0;
            for (int e = d * per; e < (d + 1) * per; ++e) order[no++] = e;
            for (int i = 0; i < no; ++i) {
                int best = i;
                for (int j = i + 1; j < no; ++j) {
                    int64_t qj = q[(size_t)order[j] * R + d], qb = q[(size_t)order[best] * R + d];
                    if (qj > qb || (qj == qb && order[j] < order[best])) best = j;
                }
                int t = order[i]; order[i] = order[best]; order[best] = t;
            }
            for (int i = 0; i < no && load[d] > tau; ++i) {
                const int e = order[i];
                while (load[d] > tau && q[(size_t)e * R + d] > 0) {
                    int rcv = -1;
                    for (int r = 0; r < R; ++r) {           /* an existing copy first */
                        if (r == d || q[(size_t)e * R + r] == 0 || load[r] >= tau) continue;
                        if (rcv < 0 || load[r] < load[rcv]) rcv = r;
                    }
                    if (rcv < 0) {
                        if (fan == 0 && newcopy[e]) break;
                        for (int r = 0; r < R; ++r) {       /* a new copy */
                            if (r == d || q[(size_t)e * R + r] > 0 || load[r] >= tau || nrep[r] >= budget)
                                continue;
                            if (rcv < 0 || load[r] < load[rcv]) rcv = r;
                        }
                        if (rcv < 0) break;
                        nrep[rcv] += 1;
                        newcopy[e] = 1;
                    }
                    int64_t x = q[(size_t)e * R + d];
                    if (load[d] - tau < x) x = load[d] - tau;
                    if (tau - load[rcv] < x) x = tau - load[rcv];
                    q[(size_t)e * R + d] -= x;
                    q[(size_t)e * R + rcv] += x;
                    load[d] -= x;
                    load[rcv] += x;
                    moved += x;
                    moves += 1;
                }
            }
        }
        if (moved == 0) break;
    }
    *moves_out = moves;
}

int orc_plan_blocks(int64_t T, int32_t E, int32_t K, int32_t R, int32_t tile, int32_t budget,
                    const int32_t* counts,
                    orc_piece* pieces, int32_t* n_pieces,
                    orc_block* blocks, int32_t* n_blocks,
                    int64_t* rank_load, int32_t* rank_replicas, int64_t* rank_row0,
                    int32_t* moves_out, uint32_t* status, int32_t* info)
{
    if (R <= 0 || E <= 0 || E % R != 0 || T % R != 0 || tile <= 0 || budget < 0)
        return ORC_ERR_ARG;
    (void)K;
    const int32_t per = E / R;
    int64_t* b = (int64_t*)malloc(sizeof(int64_t) * (size_t)E);
    int64_t* qbest = (int64_t*)malloc(sizeof(int64_t) * (size_t)E * R);
    int64_t* q = (int64_t*)malloc(sizeof(int64_t) * (size_t)E * R);
    int64_t* load = (int64_t*)malloc(sizeof(int64_t) * (size_t)R);
    int64_t* lbest = (int64_t*)malloc(sizeof(int64_t) * (size_t)R);
    int32_t* nrep = (int32_t*)malloc(sizeof(int32_t) * (size_t)R);
    int32_t* nbest = (int32_t*)malloc(sizeof(int32_t) * (size_t)R);
    char* newcopy = (char*)malloc((size_t)E);
    int32_t* order = (int32_t*)malloc(sizeof(int32_t) * (size_t)(per + E * R + 1));
    int32_t* donors = (int32_t*)malloc(sizeof(int32_t) * (size_t)R);
    int64_t* p_start = (int64_t*)calloc((size_t)R * E, sizeof(int64_t));
    int64_t* p_len = (int64_t*)calloc((size_t)R * E, sizeof(int64_t));
    if (!b || !qbest || !q || !load || !lbest || !nrep || !nbest || !newcopy || !order || !donors ||
        !p_start || !p_len) {
        free(b); free(qbest); free(q); free(load); free(lbest); free(nrep); free(nbest); free(newcopy);
        free(order); free(donors); free(p_start); free(p_len);
        return ORC_ERR_INTERNAL;
    }
    int64_t total = 0;
    for (int e = 0; e < E; ++e) { b[e] = (counts[e] + tile - 1) / tile; total += b[e]; }
    const int64_t tau = (total + R - 1) / R;

    /* four candidates: (donor priority, fan-out) = (0,0), (0,1), (1,0), (1,1) */
    int best_c = -1, moves = 0;
    int64_t best_max = 0, best_reps = 0;
    for (int c = 0; c < 4; ++c) {
        int32_t mv = 0;
        run_candidate(E, R, per, budget, tau, b, c / 2, c % 2, q, load, nrep, &mv, newcopy, order, donors);
        int64_t mx = 0, reps = 0;
        for (int r = 0; r < R; ++r) { if (load[r] > mx) mx = load[r]; reps += nrep[r]; }
        if (best_c < 0 || mx < best_max || (mx == best_max && reps < best_reps)) {
            best_c = c; best_max = mx; best_reps = reps; moves = mv;
            memcpy(qbest, q, sizeof(int64_t) * (size_t)E * R);
            memcpy(lbest, load, sizeof(int64_t) * (size_t)R);
            memcpy(nbest, nrep, sizeof(int32_t) * (size_t)R);
        }
    }
    q = (int64_t*)memcpy(q, qbest, sizeof(int64_t) * (size_t)E * R);
    memcpy(load, lbest, sizeof(int64_t) * (size_t)R);
    memcpy(nrep, nbest, sizeof(int32_t) * (size_t)R);

    /* pruning: replicas in increasing allocation size (at pass entry) */
    {
        int nr = 0;
        int32_t* rl = order;   /* pairs (e, r) packed as e*R + r */
        for (int e = 0; e < E; ++e)
            for (int r = 0; r < R; ++r)
                if (r != e / per && q[(size_t)e * R + r] > 0) rl[nr++] = e * R + r;
        for (int i = 0; i < nr; ++i) {   /* stable selection sort by (blocks, e, r) */
            int best = i;
            for (int j = i + 1; j < nr; ++j) {
                int64_t qj = q[rl[j]], qb = q[rl[best]];
                if (qj < qb || (qj == qb && rl[j] < rl[best])) best = j;
            }
            int t = rl[i]; rl[i] = rl[best]; rl[best] = t;
        }
        for (int i = 0; i < nr; ++i) {
            const int e = rl[i] / R, r = rl[i] % R, o = e / per;
            const int64_t x = q[(size_t)e * R + r];
            if (x == 0) continue;
            int tgt = -1;
            if (load[o] + x <= best_max) tgt = o;
            else {
                for (int c2 = 0; c2 < R; ++c2) {
                    if (c2 == r || c2 == o || q[(size_t)e * R + c2] == 0 || load[c2] + x > best_max) continue;
                    if (tgt < 0 || load[c2] < load[tgt]) tgt = c2;
                }
            }
            if (tgt < 0) continue;
            q[(size_t)e * R + r] = 0;
            q[(size_t)e * R + tgt] += x;
            load[r] -= x;
            load[tgt] += x;
            nrep[r] -= 1;
            moves += 1;
        }
    }
    /* refinement: single blocks from the most- to the least-loaded rank */
    for (int64_t it = 0; it < total; ++it) {
        int hi = 0, lo = 0;
        for (int r = 1; r < R; ++r) {
            if (load[r] > load[hi]) hi = r;
            if (load[r] < load[lo]) lo = r;
        }
        if (load[hi] - load[lo] <= 1) break;
        int e_sh = -1;
        for (int e = 0; e < E && e_sh < 0; ++e)
            if (q[(size_t)e * R + hi] > 0 && (lo == e / per || q[(size_t)e * R + lo] > 0)) e_sh = e;
        if (e_sh < 0) break;
        q[(size_t)e_sh * R + hi] -= 1;
        q[(size_t)e_sh * R + lo] += 1;
        load[hi] -= 1;
        load[lo] += 1;
        moves += 1;
    }
    /* materialise: owner first, then the other ranks in increasing index */
    int32_t* used = nrep;
    for (int r = 0; r < R; ++r) used[r] = 0;
    int64_t mx = 0;
    for (int r = 0; r < R; ++r) if (load[r] > mx) mx = load[r];
    for (int e = 0; e < E; ++e) {
        const int o = e / per;
        int64_t off = 0;
        for (int k = -1; k < R; ++k) {
            const int r = k < 0 ? o : k;
            if (k >= 0 && r == o) continue;
            const int64_t n = q[(size_t)e * R + r];
            if (n == 0) continue;
            const int64_t start = off * tile;
            int64_t end = (off + n) * tile;
            if (end > counts[e]) end = counts[e];
            p_start[(size_t)r * E + e] = start;
            p_len[(size_t)r * E + e] = end - start;
            if (r != o) used[r] += 1;
            off += n;
        }
    }
    layout_pieces(E, R, tile, p_start, p_len, used, pieces, n_pieces, blocks, n_blocks, rank_load,
                  rank_replicas, rank_row0);
    int64_t reps = 0;
    for (int r = 0; r < R; ++r) reps += used[r];
    *moves_out = moves;
    *status = 0;
    info[0] = (int32_t)tau;
    info[1] = best_c;
    info[2] = (int32_t)mx;
    info[3] = (int32_t)reps;
    free(b); free(qbest); free(q); free(load); free(lbest); free(nrep); free(nbest); free(newcopy);
    free(order); free(donors); free(p_start); free(p_len);
    return ORC_OK;
}

/* ------------------------------------------------- row maps (A5)
 * [MegaFlux] App. A.2 "Mapping blocks to routed assignments": within each
 * expert, routed assignments are ordered by source GPU and then local
 * (token, top-k position), and cut into the planned blocks. READING: the
 * source rank of token t is t / S, so the order is plain (t, k) order.
 * pos(t,k) = number of earlier entries with the same expert; the entry goes
 * to the piece of its expert whose [start, start+len) holds pos.
 */
int orc_row_maps(int64_t T, int32_t K, int32_t E, const int32_t* idx,
                 const orc_piece* pieces, int32_t n_pieces,
                 int64_t rows_cap, int32_t* row_of, int32_t* src_of)
{
    int64_t* seen = (int64_t*)calloc((size_t)E, sizeof(int64_t));
    if (!seen) return ORC_ERR_INTERNAL;
    for (int64_t r = 0; r < rows_cap; ++r) src_of[r] = -1;
    for (int64_t t = 0; t < T; ++t) {
        for (int k = 0; k < K; ++k) {
            int e = idx[t * K + k];
            int64_t pos = seen[e]++;
            int found = -1;
            for (int p = 0; p < n_pieces; ++p) {
                if (pieces[p].expert == e && pieces[p].start <= pos &&
                    pos < (int64_t)pieces[p].start + pieces[p].len) { found = p; break; }
            }
            if (found < 0) { free(seen); return ORC_ERR_ARG; }
            int64_t row = pieces[found].row0 + (pos - pieces[found].start);
            if (row >= rows_cap) { free(seen); return ORC_ERR_ARG; }
            row_of[t * K + k] = (int32_t)row;
            src_of[row] = (int32_t)t;
        }
    }
    free(seen);
    return ORC_OK;
}

/* ------------------------------------------------- dispatch (A6)
 * [MegaFlux] §1: routed activations are sent to the GPUs hosting the
 * selected experts. On one GPU the send is a copy of token rows into the
 * expert-major buffer; padding rows are zero.
 */
int orc_dispatch(int64_t rows, int32_t d, int32_t dtype, const void* x,
                 const int32_t* src_of, void* xp)
{
    const size_t eb = dtype == ORC_BF16 ? 2 : 4;   /* a copy of the element's bytes */
    for (int64_t r = 0; r < rows; ++r) {
        for (int32_t i = 0; i < d; ++i) {
            char* dst = (char*)xp + ((size_t)r * d + i) * eb;
            if (src_of[r] >= 0)
                memcpy(dst, (const char*)x + ((size_t)src_of[r] * d + i) * eb, eb);
            else
                memset(dst, 0, eb);
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------- expert FFN (A7, A8)
 * [MegaFlux] §4.1: SwiGLU experts; §2.1 and §3.2 "Forward": FC1 (input
 * projection, W1) then FC2 (output projection, W2) per token block.
 * READING: W1 = [gate; up] stacked as w_gate_up[e] of shape [2F, d], rows
 * 0..F-1 gate and F..2F-1 up; W2 = w_down[e] of shape [d, F];
 * h = silu(x.gate) * (x.up), silu(a) = a / (1 + exp(-a)); y = h . W2.
 * One row of the expert FFN in fp64; h and y are rounded per round_mode.
 */
static void ffn_row(int32_t d, int32_t F, int32_t dtype, int32_t round_mode,
                    const void* xrow_src, int64_t xrow_off,
                    const void* w_gu, const void* w_down, int32_t e,
                    double* h /*[F]*/, double* y /*[d]*/)
{
    const int64_t gu_base = (int64_t)e * 2 * F * d;
    const int64_t dn_base = (int64_t)e * d * F;
    for (int32_t j = 0; j < F; ++j) {
        double a = 0.0, g = 0.0;
        for (int32_t i = 0; i < d; ++i) {
            double xv = load_elem(xrow_src, xrow_off + i, dtype);
            a += xv * load_elem(w_gu, gu_base + (int64_t)j * d + i, dtype);
            g += xv * load_elem(w_gu, gu_base + (int64_t)(F + j) * d + i, dtype);
        }
        double silu = a / (1.0 + exp(-a));
        h[j] = round_as(silu * g, round_mode);
    }
    for (int32_t i = 0; i < d; ++i) {
        double s = 0.0;
        for (int32_t j = 0; j < F; ++j)
            s += h[j] * load_elem(w_down, dn_base + (int64_t)i * F + j, dtype);
        y[i] = round_as(s, round_mode);
    }
}

/* H and Yp for every row of every planned block; padding rows are zero. */
int orc_expert_ffn(int32_t d, int32_t F, int32_t dtype, int32_t round_mode, int32_t tile,
                   const orc_block* blocks, int32_t n_blocks,
                   const void* xp, const void* w_gu, const void* w_down,
                   void* h_out, void* yp_out)
{
    double* h = (double*)malloc(sizeof(double) * (size_t)F);
    double* y = (double*)malloc(sizeof(double) * (size_t)d);
    if (!h || !y) { free(h); free(y); return ORC_ERR_INTERNAL; }
    for (int32_t b = 0; b < n_blocks; ++b) {
        for (int32_t r = 0; r < tile; ++r) {
            int64_t row = (int64_t)blocks[b].row0 + r;
            if (r < blocks[b].valid) {
                ffn_row(d, F, dtype, round_mode, xp, row * d, w_gu, w_down,
                        blocks[b].expert, h, y);
            } else {
                for (int32_t j = 0; j < F; ++j) h[j] = 0.0;
                for (int32_t i = 0; i < d; ++i) y[i] = 0.0;
            }
            for (int32_t j = 0; j < F; ++j) store_elem(h_out, row * F + j, dtype, h[j]);
            for (int32_t i = 0; i < d; ++i) store_elem(yp_out, row * d + i, dtype, y[i]);
        }
    }
    free(h);
    free(y);
    return ORC_OK;
}

/* ------------------------------------------------- combine (A9)
 * [MegaFlux] §1: expert outputs are combined according to the routing
 * weights; §2.1: the final top-k sum is its own launch.
 * out[t] = sum over k, in k order, of w[t,k] * Yp[row_of(t,k)].
 */
int orc_combine(int64_t T, int32_t K, int32_t d, int32_t dtype, int32_t round_mode,
                const void* yp, const int32_t* row_of, const float* w, void* out)
{
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t i = 0; i < d; ++i) {
            double s = 0.0;
            for (int32_t k = 0; k < K; ++k)
                s += (double)w[t * K + k] * load_elem(yp, (int64_t)row_of[t * K + k] * d + i, dtype);
            store_elem(out, t * d + i, dtype, round_as(s, round_mode));
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------- one token's layer output
 * The same arithmetic as dispatch + FFN + combine for one token, taken
 * straight from x: the plan only decides which rows hold a token's copies,
 * never their values. Used to check sampled tokens of large layers.
 */
int orc_token_out(int32_t d, int32_t F, int32_t K, int32_t dtype, int32_t round_mode,
                  int64_t n_tok, const int64_t* tokens,
                  const void* x, const int32_t* idx, const float* w,
                  const void* w_gu, const void* w_down, double* out /*[n_tok, d]*/)
{
    double* h = (double*)malloc(sizeof(double) * (size_t)F);
    double* y = (double*)malloc(sizeof(double) * (size_t)d * K);
    if (!h || !y) { free(h); free(y); return ORC_ERR_INTERNAL; }
    for (int64_t n = 0; n < n_tok; ++n) {
        int64_t t = tokens[n];
        for (int32_t k = 0; k < K; ++k)
            ffn_row(d, F, dtype, round_mode, x, t * d, w_gu, w_down, idx[t * K + k], h,
                    y + (size_t)k * d);
        for (int32_t i = 0; i < d; ++i) {
            double s = 0.0;
            for (int32_t k = 0; k < K; ++k) s += (double)w[t * K + k] * y[(size_t)k * d + i];
            out[n * d + i] = round_as(s, round_mode);
        }
    }
    free(h);
    free(y);
    return ORC_OK;
}

/* ------------------------------------------------- sampled entries
 * h and y of single routed entries (token t, expert e), straight from x, in
 * the same arithmetic as the expert FFN above. Used to check sampled rows of
 * large layers.
 */
int orc_entry_ffn(int32_t d, int32_t F, int32_t dtype, int32_t round_mode, int64_t n,
                  const int64_t* tokens, const int32_t* experts, const void* x,
                  const void* w_gu, const void* w_down, double* h_out /*[n,F]*/,
                  double* y_out /*[n,d]*/)
{
    for (int64_t i = 0; i < n; ++i)
        ffn_row(d, F, dtype, round_mode, x, tokens[i] * d, w_gu, w_down, experts[i],
                h_out + (size_t)i * F, y_out + (size_t)i * d);
    return ORC_OK;
}

/* ------------------------------------------------- dense reference
 * The plain definition of the routed layer: run every expert on every
 * token in fp64 and add expert e's output with weight gate(t,e) when e is
 * among the token's top-k, else zero. Membership is decided by rank
 * counting (e is chosen when fewer than K experts beat it, a higher logit
 * or an equal logit at a lower id), and the weight is the full softmax (or
 * the sigmoid) renormalised over the chosen set. Inputs are fp64 arrays.
 */
int orc_dense_layer(int64_t T, int32_t d, int32_t E, int32_t K, int32_t F, int32_t gating,
                    const double* logits, const double* x, const double* w_gu,
                    const double* w_down, double* out)
{
    double* p = (double*)malloc(sizeof(double) * (size_t)E);
    char* chosen = (char*)malloc((size_t)E);
    double* h = (double*)malloc(sizeof(double) * (size_t)F);
    if (!p || !chosen || !h) { free(p); free(chosen); free(h); return ORC_ERR_INTERNAL; }
    for (int64_t t = 0; t < T; ++t) {
        const double* l = logits + t * E;
        double mx = l[0];
        for (int e = 1; e < E; ++e) if (l[e] > mx) mx = l[e];
        double z = 0.0;
        for (int e = 0; e < E; ++e) {
            p[e] = gating == ORC_GATE_SOFTMAX_TOPK ? exp(l[e] - mx) : 1.0 / (1.0 + exp(-l[e]));
            z += p[e];
        }
        if (gating == ORC_GATE_SOFTMAX_TOPK) for (int e = 0; e < E; ++e) p[e] /= z;
        double zsel = 0.0;
        for (int e = 0; e < E; ++e) {
            int beaten_by = 0;
            for (int j = 0; j < E; ++j)
                if (l[j] > l[e] || (l[j] == l[e] && j < e)) beaten_by++;
            chosen[e] = beaten_by < K;
            if (chosen[e]) zsel += p[e];
        }
        for (int32_t i = 0; i < d; ++i) out[t * d + i] = 0.0;
        for (int e = 0; e < E; ++e) {
            double gate = chosen[e] ? p[e] / zsel : 0.0;
            const double* wg = w_gu + (int64_t)e * 2 * F * d;
            const double* wd = w_down + (int64_t)e * d * F;
            for (int32_t j = 0; j < F; ++j) {
                double a = 0.0, g = 0.0;
                for (int32_t i = 0; i < d; ++i) {
                    a += x[t * d + i] * wg[(int64_t)j * d + i];
                    g += x[t * d + i] * wg[(int64_t)(F + j) * d + i];
                }
                h[j] = a / (1.0 + exp(-a)) * g;
            }
            for (int32_t i = 0; i < d; ++i) {
                double s = 0.0;
                for (int32_t j = 0; j < F; ++j) s += h[j] * wd[(int64_t)i * F + j];
                out[t * d + i] += gate * s;
            }
        }
    }
    free(p);
    free(chosen);
    free(h);
    return ORC_OK;
}

/* ------------------------------------------------- backward (NEXT: training)
 * [MegaFlux] §3.2 "Backward": DGrad runs through W2 then W1, WGrad forms
 * each expert's weight gradients from the routed blocks, and replica
 * partials of one expert are reduced into one gradient.
 *
 * Given dOut = dL/dout [T, d], for every routed entry (t, k) of expert e:
 *   dY      = w[t,k] * dOut[t]                           (the combine's input gradient)
 *   dw[t,k] = dOut[t] . y_(t,k)                         (the routing weight's gradient)
 *   dH      = dY . W2_e            (DGrad through W2: sum over d)
 *   dA      = dH * g * silu'(a),  dG = dH * silu(a)      (SwiGLU, silu' = s (1 + a (1 - s)), s = sigmoid(a))
 *   dXp     = dA . W_gate_e + dG . W_up_e                (DGrad through W1: sum over F)
 *   dx[t]   = sum over k, in k order, of dXp_(t,k)
 *   dW2_e      += dY^T h,  dW_gate_e += dA^T x_t,  dW_up_e += dG^T x_t   (WGrad)
 * and the router logits' gradient through the gating (zero off the top-k):
 *   softmax over the chosen: dl[t, idx[t,m]] = w_m (dw_m - sum_k w_k dw_k)
 *   sigmoid normalised:      dl[t, idx[t,m]] = w_m (1 - s_m) (dw_m - sum_k w_k dw_k), s_m = sigmoid(l).
 * READING: the weights of both gatings sum to one, so the inner term is
 * taken as sum_k w_k (dw_m - dw_k): the same value, without the cancellation
 * that the first form suffers when one weight is close to one.
 * READING (rounding points, mirroring a bf16 GPU path; ORC_ROUND_NONE keeps
 * everything in fp64): dY is the fp32 product w * dOut rounded to bf16; the
 * pre-activations a and g are recomputed and rounded to bf16, and the
 * SwiGLU derivative reads the rounded values; h and y are the forward's
 * (rounded) values; dA, dG and dXp are rounded to bf16 once each; dx is
 * rounded once after its k-ordered sum. Weight gradients, dw and the logits'
 * gradient are returned in fp64 (the GPU path stores them as fp32).
 * x, d_out, weights: arrays of `dtype`; logits and w: fp32.
 */
static double sigmoid_d(double v) { return 1.0 / (1.0 + exp(-v)); }

typedef struct {
    double *a, *g, *h, *y, *dy, *dh, *da, *dg, *dxp;
} bwd_scratch;

static int bwd_scratch_alloc(bwd_scratch* s, int32_t d, int32_t F)
{
    s->a = (double*)malloc(sizeof(double) * F);   s->g = (double*)malloc(sizeof(double) * F);
    s->h = (double*)malloc(sizeof(double) * F);   s->y = (double*)malloc(sizeof(double) * d);
    s->dy = (double*)malloc(sizeof(double) * d);  s->dh = (double*)malloc(sizeof(double) * F);
    s->da = (double*)malloc(sizeof(double) * F);  s->dg = (double*)malloc(sizeof(double) * F);
    s->dxp = (double*)malloc(sizeof(double) * d);
    return s->a && s->g && s->h && s->y && s->dy && s->dh && s->da && s->dg && s->dxp;
}

static void bwd_scratch_free(bwd_scratch* s)
{
    free(s->a); free(s->g); free(s->h); free(s->y); free(s->dy); free(s->dh);
    free(s->da); free(s->dg); free(s->dxp);
}

/* Every backward quantity of one routed entry (token t, expert e, weight wt).
 * Returns dw for the entry. */
static double bwd_entry(int32_t d, int32_t F, int32_t dtype, int32_t round_mode,
                        const void* x, int64_t t, const void* w_gu, const void* w_down, int32_t e,
                        float wt, const void* d_out, bwd_scratch* s)
{
    const int64_t gu_base = (int64_t)e * 2 * F * d;
    const int64_t dn_base = (int64_t)e * d * F;
    /* forward: pre-activations, h (from the unrounded pre-activations), y */
    for (int32_t j = 0; j < F; ++j) {
        double a = 0.0, g = 0.0;
        for (int32_t i = 0; i < d; ++i) {
            double xv = load_elem(x, t * d + i, dtype);
            a += xv * load_elem(w_gu, gu_base + (int64_t)j * d + i, dtype);
            g += xv * load_elem(w_gu, gu_base + (int64_t)(F + j) * d + i, dtype);
        }
        s->h[j] = round_as(a / (1.0 + exp(-a)) * g, round_mode);
        s->a[j] = round_as(a, round_mode);
        s->g[j] = round_as(g, round_mode);
    }
    double dw = 0.0;
    for (int32_t i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int32_t j = 0; j < F; ++j) acc += s->h[j] * load_elem(w_down, dn_base + (int64_t)i * F + j, dtype);
        s->y[i] = round_as(acc, round_mode);
        const double go = load_elem(d_out, t * d + i, dtype);
        dw += go * s->y[i];
        /* dY: the product formed in fp32 before its bf16 rounding */
        s->dy[i] = round_mode == ORC_ROUND_NONE ? (double)wt * go
                                                : round_as((double)(float)((float)wt * (float)go), round_mode);
    }
    /* DGrad through W2, then the SwiGLU derivative */
    for (int32_t j = 0; j < F; ++j) {
        double acc = 0.0;
        for (int32_t i = 0; i < d; ++i) acc += s->dy[i] * load_elem(w_down, dn_base + (int64_t)i * F + j, dtype);
        s->dh[j] = acc;
        const double a = s->a[j], sg = sigmoid_d(a);
        s->da[j] = round_as(acc * s->g[j] * (sg * (1.0 + a * (1.0 - sg))), round_mode);
        s->dg[j] = round_as(acc * (a * sg), round_mode);
    }
    /* DGrad through W1 */
    for (int32_t i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int32_t j = 0; j < F; ++j)
            acc += s->da[j] * load_elem(w_gu, gu_base + (int64_t)j * d + i, dtype) +
                   s->dg[j] * load_elem(w_gu, gu_base + (int64_t)(F + j) * d + i, dtype);
        s->dxp[i] = round_as(acc, round_mode);
    }
    return dw;
}

/* The logits' gradient of one token from its routing weights' gradients. */
static void bwd_gating(int32_t E, int32_t K, int32_t gating, const float* l, const int32_t* idx,
                       const float* w, const double* dw, double* dl /*[E]*/)
{
    for (int32_t e = 0; e < E; ++e) dl[e] = 0.0;
    for (int32_t m = 0; m < K; ++m) {
        double inner = 0.0;
        for (int32_t k = 0; k < K; ++k) inner += (double)w[k] * (dw[m] - dw[k]);
        double v = (double)w[m] * inner;
        if (gating == ORC_GATE_SIGMOID_TOPK) v *= 1.0 - sigmoid_d((double)l[idx[m]]);
        dl[idx[m]] = v;
    }
}

int orc_layer_bwd(int64_t T, int32_t d, int32_t E, int32_t K, int32_t F, int32_t gating,
                  int32_t dtype, int32_t round_mode,
                  const float* logits, const int32_t* idx, const float* w,
                  const void* x, const void* w_gu, const void* w_down, const void* d_out,
                  void* dx /*[T,d] dtype*/, double* dw_gu /*[E,2F,d]*/, double* dw_down /*[E,d,F]*/,
                  double* dw_topk /*[T,K]*/, double* dlogits /*[T,E]*/)
{
    bwd_scratch s;
    double* dxs = (double*)malloc(sizeof(double) * (size_t)d);
    if (!bwd_scratch_alloc(&s, d, F) || !dxs) { bwd_scratch_free(&s); free(dxs); return ORC_ERR_INTERNAL; }
    memset(dw_gu, 0, sizeof(double) * (size_t)E * 2 * F * d);
    memset(dw_down, 0, sizeof(double) * (size_t)E * d * F);
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t i = 0; i < d; ++i) dxs[i] = 0.0;
        for (int32_t k = 0; k < K; ++k) {
            const int32_t e = idx[t * K + k];
            dw_topk[t * K + k] = bwd_entry(d, F, dtype, round_mode, x, t, w_gu, w_down, e, w[t * K + k],
                                           d_out, &s);
            for (int32_t i = 0; i < d; ++i) dxs[i] += s.dxp[i];
            double* wd = dw_down + (int64_t)e * d * F;
            for (int32_t i = 0; i < d; ++i)
                for (int32_t j = 0; j < F; ++j) wd[(int64_t)i * F + j] += s.dy[i] * s.h[j];
            double* wg = dw_gu + (int64_t)e * 2 * F * d;
            for (int32_t j = 0; j < F; ++j)
                for (int32_t i = 0; i < d; ++i) {
                    const double xv = load_elem(x, t * d + i, dtype);
                    wg[(int64_t)j * d + i] += s.da[j] * xv;
                    wg[(int64_t)(F + j) * d + i] += s.dg[j] * xv;
                }
        }
        for (int32_t i = 0; i < d; ++i) store_elem(dx, t * d + i, dtype, round_as(dxs[i], round_mode));
        if (dlogits)
            bwd_gating(E, K, gating, logits + t * E, idx + t * K, w + t * K, dw_topk + t * K, dlogits + t * E);
    }
    bwd_scratch_free(&s);
    free(dxs);
    return ORC_OK;
}

/* dx rows, dw and the logits' gradient of selected tokens (for large layers). */
int orc_bwd_tokens(int32_t d, int32_t E, int32_t K, int32_t F, int32_t gating, int32_t dtype,
                   int32_t round_mode, int64_t n_tok, const int64_t* tokens,
                   const float* logits, const int32_t* idx, const float* w,
                   const void* x, const void* w_gu, const void* w_down, const void* d_out,
                   double* dx /*[n,d]*/, double* dw_topk /*[n,K]*/, double* dlogits /*[n,E]*/)
{
    bwd_scratch s;
    if (!bwd_scratch_alloc(&s, d, F)) { bwd_scratch_free(&s); return ORC_ERR_INTERNAL; }
    for (int64_t n = 0; n < n_tok; ++n) {
        const int64_t t = tokens[n];
        double* dxs = dx + n * d;
        for (int32_t i = 0; i < d; ++i) dxs[i] = 0.0;
        for (int32_t k = 0; k < K; ++k) {
            dw_topk[n * K + k] = bwd_entry(d, F, dtype, round_mode, x, t, w_gu, w_down, idx[t * K + k],
                                           w[t * K + k], d_out, &s);
            for (int32_t i = 0; i < d; ++i) dxs[i] += s.dxp[i];
        }
        for (int32_t i = 0; i < d; ++i) dxs[i] = round_as(dxs[i], round_mode);
        bwd_gating(E, K, gating, logits + t * E, idx + t * K, w + t * K, dw_topk + n * K, dlogits + n * E);
    }
    bwd_scratch_free(&s);
    return ORC_OK;
}

/* Single elements of the weight gradients of one expert: which = 0 for
 * dW_gate[e][r][c] and 1 for dW_up[e][r][c] (r < F, c < d), 2 for
 * dW2[e][r][c] (r < d, c < F). Sums over every entry routed to e. */
int orc_bwd_wgrad_elems(int64_t T, int32_t d, int32_t K, int32_t F, int32_t dtype, int32_t round_mode,
                        const int32_t* idx, const float* w, const void* x, const void* w_gu,
                        const void* w_down, const void* d_out, int32_t e, int64_t n,
                        const int32_t* which, const int32_t* r, const int32_t* c, double* out)
{
    bwd_scratch s;
    if (!bwd_scratch_alloc(&s, d, F)) { bwd_scratch_free(&s); return ORC_ERR_INTERNAL; }
    for (int64_t q = 0; q < n; ++q) out[q] = 0.0;
    for (int64_t t = 0; t < T; ++t)
        for (int32_t k = 0; k < K; ++k) {
            if (idx[t * K + k] != e) continue;
            bwd_entry(d, F, dtype, round_mode, x, t, w_gu, w_down, e, w[t * K + k], d_out, &s);
            for (int64_t q = 0; q < n; ++q) {
                if (which[q] == 2) out[q] += s.dy[r[q]] * s.h[c[q]];
                else out[q] += (which[q] == 0 ? s.da[r[q]] : s.dg[r[q]]) * load_elem(x, t * d + c[q], dtype);
            }
        }
    bwd_scratch_free(&s);
    return ORC_OK;
}

/* bf16 rounding exposed for pins of the rounding helper itself */
uint16_t orc_double_to_bf16(double v) { return double_to_bf16(v); }

/* ================================================= MX (block-scaled) forward
 * [MegaFlux] §2.1 'Persistent MoE execution': the Blackwell MMA is block
 * scaled (MXFP8 / MXFP4); §4.1 'Setup': the forward runs with MX operands,
 * fp32 accumulation and bf16 outputs. [MoonEP] "A bandwidth-only model": an
 * MX format stores one scale per 32 elements.
 * READING: the pages name the formats but do not define them; they are read
 * as the OCP Microscaling formats. A block is 32 consecutive elements along
 * the contraction dimension; its scale is a power of two X = 2^(s - 127)
 * stored as the 8-bit exponent s (E8M0); s = floor(log2(max |v|)) - 8 + 127
 * for MXFP8 with E4M3 elements (8 = the exponent of E4M3's largest normal,
 * 448 = 1.75 * 2^8), clamped to [0, 254], and s = 0 for an all-zero block;
 * every element is v / X rounded to E4M3, nearest with ties to even,
 * saturating at +-448. E4M3: 1 sign bit, 4 exponent bits (bias 7), 3
 * mantissa bits, subnormals at exponent field 0, code 0x7F / 0xFF is NaN
 * (never produced from finite input).
 */

/* The value of an E4M3 code (NaN codes give NaN). */
static double e4m3_value(uint8_t c)
{
    const int sign = c >> 7, ef = (c >> 3) & 15, mf = c & 7;
    double v;
    if (ef == 15 && mf == 7) return NAN;
    if (ef == 0) v = ldexp((double)mf, -9);                 /* subnormal: mf/8 * 2^-6 */
    else v = ldexp(8.0 + mf, ef - 7 - 3);                  /* (1 + mf/8) * 2^(ef-7) */
    return sign ? -v : v;
}

/* v rounded to E4M3: nearest, ties to even, saturating at 448; the sign of
 * v is kept (a negative value that rounds to zero gives -0, code 0x80). */
static uint8_t e4m3_encode(double v)
{
    const uint8_t sign = signbit(v) ? 0x80 : 0x00;
    const double a = fabs(v);
    if (a >= 448.0) return sign | 0x7E;
    if (a < ldexp(1.0, -6)) {
        /* subnormal range: multiples of 2^-9; a rounding up to 2^-6 gives code 8, the smallest normal */
        const double q = nearbyint(ldexp(a, 9));
        return sign | (uint8_t)q;
    }
    int ex;
    frexp(a, &ex);                 /* a = m * 2^ex, m in [0.5, 1) */
    int e = ex - 1;                /* floor(log2 a), in [-6, 8] */
    double r = nearbyint(ldexp(a, 3 - e));   /* 1.mmm scaled to [8, 16] */
    if (r == 16.0) { r = 8.0; ++e; }
    return sign | (uint8_t)(((e + 7) << 3) | ((int)r - 8));
}

/* The E8M0 scale exponent of a block whose largest magnitude is amax. */
static uint8_t mx_scale_code(double amax)
{
    if (amax == 0.0) return 0;
    int ex;
    frexp(amax, &ex);
    int s = (ex - 1) - 8 + 127;
    if (s < 0) s = 0;
    if (s > 254) s = 254;
    return (uint8_t)s;
}

/* MXFP4 ([MegaFlux] §4.1: MXFP4 weights in the forward; [MoonEP] "A
 * bandwidth-only model": packed 4-bit elements plus one scale per 32).
 * READING: OCP E2M1 elements: 1 sign bit, 2 exponent bits (bias 1), 1
 * mantissa bit, subnormal at exponent field 0; magnitudes 0, 0.5, 1, 1.5, 2,
 * 3, 4, 6; no NaN or infinity. The block scale uses the exponent of E2M1's
 * largest normal (6 = 1.5 * 2^2): s = floor(log2 max|v|) - 2 + 127. Here a
 * code is kept one per byte (0..15); packing two per byte is storage. */
static double e2m1_value(uint8_t c)
{
    static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    return (c & 8) ? -mag[c & 7] : mag[c & 7];
}

/* v rounded to E2M1: the nearest of the eight magnitudes, ties to the even
 * code, saturating at 6; the sign of v is kept. */
static uint8_t e2m1_encode(double v)
{
    const uint8_t sign = signbit(v) ? 8 : 0;
    const double a = fabs(v);
    uint8_t best = 0;
    double bd = INFINITY;
    for (uint8_t c = 0; c < 8; ++c) {
        const double dd = fabs(e2m1_value(c) - a);
        if (dd < bd || (dd == bd && (c & 1) == 0)) { bd = dd; best = c; }
    }
    return sign | best;
}

enum { ORC_MX_E4M3 = 0, ORC_MX_E2M1 = 1 };

static int elem_emax(int fmt) { return fmt == ORC_MX_E2M1 ? 2 : 8; }

/* The scale exponent of a block with largest magnitude amax for element format fmt. */
static uint8_t mx_scale_code_fmt(double amax, int fmt)
{
    if (amax == 0.0) return 0;
    int ex;
    frexp(amax, &ex);
    int s = (ex - 1) - elem_emax(fmt) + 127;
    if (s < 0) s = 0;
    if (s > 254) s = 254;
    return (uint8_t)s;
}

/* Quantize the rows of an fp64 matrix [rows, K] (K a multiple of 32) to an MX
 * format: codes [rows, K] and scales [rows, K/32], both row-major. */
static void mx_quantize_rows_fmt(int64_t rows, int32_t K, int fmt, const double* v, uint8_t* codes,
                                 uint8_t* scales)
{
    for (int64_t r = 0; r < rows; ++r) {
        for (int32_t b = 0; b < K / 32; ++b) {
            const double* blk = v + r * K + (int64_t)b * 32;
            double amax = 0.0;
            for (int i = 0; i < 32; ++i)
                if (fabs(blk[i]) > amax) amax = fabs(blk[i]);
            const uint8_t s = mx_scale_code_fmt(amax, fmt);
            scales[r * (K / 32) + b] = s;
            const double X = ldexp(1.0, (int)s - 127);
            for (int i = 0; i < 32; ++i)
                codes[r * K + (int64_t)b * 32 + i] = fmt == ORC_MX_E2M1 ? e2m1_encode(blk[i] / X)
                                                                         : e4m3_encode(blk[i] / X);
        }
    }
}

static void mx_quantize_rows(int64_t rows, int32_t K, const double* v, uint8_t* codes, uint8_t* scales)
{
    mx_quantize_rows_fmt(rows, K, ORC_MX_E4M3, v, codes, scales);
}

static double mx_value_fmt(const uint8_t* codes, const uint8_t* scales, int32_t K, int64_t r, int32_t k, int fmt)
{
    const uint8_t c = codes[r * K + k];
    return (fmt == ORC_MX_E2M1 ? e2m1_value(c) : e4m3_value(c)) *
           ldexp(1.0, (int)scales[r * (K / 32) + k / 32] - 127);
}

static double mx_value(const uint8_t* codes, const uint8_t* scales, int32_t K, int64_t r, int32_t k)
{
    return mx_value_fmt(codes, scales, K, r, k, ORC_MX_E4M3);
}

/* MXFP8 quantization of a bf16 or fp32 matrix [rows, K]. */
int orc_mx_quantize(int64_t rows, int32_t K, int32_t dtype, const void* x, uint8_t* codes, uint8_t* scales)
{
    if (K % 32 != 0) return ORC_ERR_ARG;
    double* row = (double*)malloc(sizeof(double) * (size_t)K);
    if (!row) return ORC_ERR_INTERNAL;
    for (int64_t r = 0; r < rows; ++r) {
        for (int32_t k = 0; k < K; ++k) row[k] = load_elem(x, r * K + k, dtype);
        mx_quantize_rows(1, K, row, codes + r * K, scales + r * (K / 32));
    }
    free(row);
    return ORC_OK;
}

/* The values an MXFP8 matrix stands for, in fp64. */
int orc_mx_dequantize(int64_t rows, int32_t K, const uint8_t* codes, const uint8_t* scales, double* out)
{
    if (K % 32 != 0) return ORC_ERR_ARG;
    for (int64_t r = 0; r < rows; ++r)
        for (int32_t k = 0; k < K; ++k) out[r * K + k] = mx_value(codes, scales, K, r, k);
    return ORC_OK;
}

/* Quantization of a bf16 or fp32 matrix [rows, K] to an MX format (fmt 0:
 * MXFP8 E4M3, 1: MXFP4 E2M1, one code per byte). */
int orc_mx_quantize_fmt(int64_t rows, int32_t K, int32_t dtype, int32_t fmt, const void* x, uint8_t* codes,
                        uint8_t* scales)
{
    if (K % 32 != 0 || (fmt != ORC_MX_E4M3 && fmt != ORC_MX_E2M1)) return ORC_ERR_ARG;
    double* row = (double*)malloc(sizeof(double) * (size_t)K);
    if (!row) return ORC_ERR_INTERNAL;
    for (int64_t r = 0; r < rows; ++r) {
        for (int32_t k = 0; k < K; ++k) row[k] = load_elem(x, r * K + k, dtype);
        mx_quantize_rows_fmt(1, K, fmt, row, codes + r * K, scales + r * (K / 32));
    }
    free(row);
    return ORC_OK;
}

int orc_mx_dequantize_fmt(int64_t rows, int32_t K, int32_t fmt, const uint8_t* codes, const uint8_t* scales,
                          double* out)
{
    if (K % 32 != 0 || (fmt != ORC_MX_E4M3 && fmt != ORC_MX_E2M1)) return ORC_ERR_ARG;
    for (int64_t r = 0; r < rows; ++r)
        for (int32_t k = 0; k < K; ++k) out[r * K + k] = mx_value_fmt(codes, scales, K, r, k, fmt);
    return ORC_OK;
}

uint8_t orc_e2m1_encode(double v) { return e2m1_encode(v); }
double orc_e2m1_value(uint8_t c) { return e2m1_value(c); }
uint8_t orc_mx_scale_code_fmt(double amax, int32_t fmt) { return mx_scale_code_fmt(amax, fmt); }

/* E4M3 codes <-> values, for the pins. */
uint8_t orc_e4m3_encode(double v) { return e4m3_encode(v); }
double orc_e4m3_value(uint8_t c) { return e4m3_value(c); }
uint8_t orc_mx_scale_code(double amax) { return mx_scale_code(amax); }

/* FC1 of one routed entry of the MX expert FFN: token row xq (MXFP8 along
 * d) through expert e's W1 = w_gate_up[e] (MXFP8 along d), in fp64 over the
 * dequantized operands, SwiGLU, h rounded to bf16 (FC1's bf16 output), then
 * h quantized to MXFP8 along F (FC2's activation operand).
 * READING: FC1 writes bf16 (§4.1: bf16 outputs) and FC2's MXFP8 operand is
 * quantized from those bf16 values. */
static void mx_fc1_row(int32_t d, int32_t F, const uint8_t* xq, const uint8_t* xs, int64_t xrow,
                       const uint8_t* w1q, const uint8_t* w1s, int32_t wfmt, int32_t e,
                       double* hb /*[F]*/, uint8_t* hq /*[F]*/, uint8_t* hs /*[F/32]*/)
{
    const int64_t g0 = (int64_t)e * 2 * F, u0 = g0 + F;
    for (int32_t j = 0; j < F; ++j) {
        double a = 0.0, g = 0.0;
        for (int32_t i = 0; i < d; ++i) {
            const double xv = mx_value(xq, xs, d, xrow, i);
            a += xv * mx_value_fmt(w1q, w1s, d, g0 + j, i, wfmt);
            g += xv * mx_value_fmt(w1q, w1s, d, u0 + j, i, wfmt);
        }
        hb[j] = round_as(a / (1.0 + exp(-a)) * g, ORC_ROUND_BF16);
    }
    mx_quantize_rows(1, F, hb, hq, hs);
}

/* FC2 of one routed entry: an MXFP8 row of h (codes hq, scales hs) through
 * expert e's W2 = w_down[e] (MXFP8 along F), fp64, y rounded to bf16. */
static void mx_fc2_row(int32_t d, int32_t F, const uint8_t* hq, const uint8_t* hs, const uint8_t* w2q,
                       const uint8_t* w2s, int32_t wfmt, int32_t e, double* y /*[d]*/)
{
    const int64_t dn0 = (int64_t)e * d;
    for (int32_t i = 0; i < d; ++i) {
        double s = 0.0;
        for (int32_t j = 0; j < F; ++j)
            s += mx_value(hq, hs, F, 0, j) * mx_value_fmt(w2q, w2s, F, dn0 + i, j, wfmt);
        y[i] = round_as(s, ORC_ROUND_BF16);
    }
}

static void mx_ffn_row(int32_t d, int32_t F, const uint8_t* xq, const uint8_t* xs, int64_t xrow,
                       const uint8_t* w1q, const uint8_t* w1s, const uint8_t* w2q, const uint8_t* w2s, int32_t wfmt,
                       int32_t e, double* hb /*[F]*/, uint8_t* hq /*[F]*/, uint8_t* hs /*[F/32]*/, double* y /*[d]*/)
{
    mx_fc1_row(d, F, xq, xs, xrow, w1q, w1s, wfmt, e, hb, hq, hs);
    mx_fc2_row(d, F, hq, hs, w2q, w2s, wfmt, e, y);
}

/* FC1 alone for n rows of an MXFP8 activation matrix (row rows[i], expert
 * experts[i]): h (bf16 values), its MXFP8 codes and scales. */
int orc_mx_fc1_rows(int32_t d, int32_t F, int64_t n, const int64_t* rows, const int32_t* experts,
                    const uint8_t* xq, const uint8_t* xs, const uint8_t* w1q, const uint8_t* w1s, int32_t wfmt,
                    double* h_out /*[n,F]*/, uint8_t* hq_out /*[n,F]*/, uint8_t* hs_out /*[n,F/32]*/)
{
    if (d % 32 != 0 || F % 32 != 0) return ORC_ERR_ARG;
    for (int64_t i = 0; i < n; ++i)
        mx_fc1_row(d, F, xq, xs, rows[i], w1q, w1s, wfmt, experts[i], h_out + (size_t)i * F,
                   hq_out + (size_t)i * F, hs_out + (size_t)i * (F / 32));
    return ORC_OK;
}

/* FC2 alone for n MXFP8 rows of h (row i through expert experts[i]): y as
 * bf16 values. */
int orc_mx_fc2_rows(int32_t d, int32_t F, int64_t n, const int32_t* experts, const uint8_t* hq,
                    const uint8_t* hs, const uint8_t* w2q, const uint8_t* w2s, int32_t wfmt, double* y_out /*[n,d]*/)
{
    if (d % 32 != 0 || F % 32 != 0) return ORC_ERR_ARG;
    for (int64_t i = 0; i < n; ++i)
        mx_fc2_row(d, F, hq + (size_t)i * F, hs + (size_t)i * (F / 32), w2q, w2s, wfmt, experts[i],
                   y_out + (size_t)i * d);
    return ORC_OK;
}

/* Sampled routed entries (token t, expert e) of the MX FFN: h (bf16 values),
 * its MXFP8 codes and scales, and y (bf16 values). */
int orc_mx_entry_ffn(int32_t d, int32_t F, int64_t n, const int64_t* tokens, const int32_t* experts,
                     const uint8_t* xq, const uint8_t* xs, const uint8_t* w1q, const uint8_t* w1s,
                     const uint8_t* w2q, const uint8_t* w2s, int32_t wfmt, double* h_out /*[n,F]*/,
                     uint8_t* hq_out /*[n,F]*/, uint8_t* hs_out /*[n,F/32]*/, double* y_out /*[n,d]*/)
{
    if (d % 32 != 0 || F % 32 != 0) return ORC_ERR_ARG;
    for (int64_t i = 0; i < n; ++i)
        mx_ffn_row(d, F, xq, xs, tokens[i], w1q, w1s, w2q, w2s, wfmt, experts[i], h_out + (size_t)i * F,
                   hq_out + (size_t)i * F, hs_out + (size_t)i * (F / 32), y_out + (size_t)i * d);
    return ORC_OK;
}

/* Sampled tokens of the MX layer: the K entries of token t as above, then
 * the weighted combine in fp64, rounded to bf16. */
int orc_mx_token_out(int32_t d, int32_t F, int32_t K, int64_t n_tok, const int64_t* tokens,
                     const uint8_t* xq, const uint8_t* xs, const int32_t* idx, const float* w,
                     const uint8_t* w1q, const uint8_t* w1s, const uint8_t* w2q, const uint8_t* w2s, int32_t wfmt,
                     double* out /*[n_tok, d]*/)
{
    if (d % 32 != 0 || F % 32 != 0) return ORC_ERR_ARG;
    double* hb = (double*)malloc(sizeof(double) * (size_t)F);
    uint8_t* hq = (uint8_t*)malloc((size_t)F);
    uint8_t* hs = (uint8_t*)malloc((size_t)F / 32);
    double* y = (double*)malloc(sizeof(double) * (size_t)d * K);
    if (!hb || !hq || !hs || !y) { free(hb); free(hq); free(hs); free(y); return ORC_ERR_INTERNAL; }
    for (int64_t n = 0; n < n_tok; ++n) {
        const int64_t t = tokens[n];
        for (int32_t k = 0; k < K; ++k)
            mx_ffn_row(d, F, xq, xs, t, w1q, w1s, w2q, w2s, wfmt, idx[t * K + k], hb, hq, hs, y + (size_t)k * d);
        for (int32_t i = 0; i < d; ++i) {
            double s = 0.0;
            for (int32_t k = 0; k < K; ++k) s += (double)w[t * K + k] * y[(size_t)k * d + i];
            out[n * d + i] = round_as(s, ORC_ROUND_BF16);
        }
    }
    free(hb); free(hq); free(hs); free(y);
    return ORC_OK;
}
