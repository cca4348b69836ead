// placement.cu -- correlated expert placement (md_place_correlated).
//
// "Expert Coupling in MoE Pretraining" (PicX summary), Correlated Placement: a
// Kernighan-Lin-style local search starts from contiguous placement and swaps
// expert pairs between GPUs to maximise the sum of W[e, e'] over pairs that
// share a GPU; each GPU holds exactly E/EP experts.  The search itself is not
// printed; this is its plainest reading: repeat the best single swap while it
// gains.  Optionally the search starts from a greedy co-location of the
// heaviest pairs instead.
//
// One CTA of 1024 threads does the whole search.  Both phases repeatedly take
// the best candidate pair (a < b) in the order (value desc, a asc, b asc) and
// keep, per expert row a, the best candidate of that row, so that a step only
// re-examines the rows a move can have changed.  In the greedy seed a row's
// candidate lives in a register of the lane that owns the row (lane j of warp
// w owns row w + 32 j); in the refinement the candidates live in shared
// memory, one thread per row updates them and the rows that need a full
// rescan are spread over all warps.  A step ends with one block-wide arg-max
// and one update.
//   Greedy seed: a pair (a, b) with W > 0 is eligible while it could still be
//   placed (both unplaced and some rank has two free slots, or one placed on
//   a rank with room and the other unplaced).  Ranks only fill up, so an
//   ineligible pair never becomes eligible again; taking the heaviest
//   eligible pair until none is left therefore places exactly the pairs that
//   the ordered scan over all pairs by weight places, and a row's candidate
//   stays its best for as long as it stays eligible.
//   Refinement: A[e][d] = sum of W[e][e'] over e' != e on rank d; swapping a
//   (rank P) with b (rank Q) gains A[a][Q] - A[a][P] + A[b][P] - A[b][Q]
//   - 2 W[a][b].  A swap between P and Q changes only columns P and Q of A,
//   so the gain of (a, b) changes only when a or b sits on P or Q: rows on P
//   or Q, and rows whose candidate sits there, are rescanned; every other row
//   compares its candidate with the pairs it forms with the 2 E/R experts of
//   P and Q.  A lives in shared memory when it fits, rows padded to R + 1
//   entries so that lanes reading consecutive rows hit different banks.
#include <climits>

#include "common.cuh"

namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr size_t kSmemA = 160 * 1024;  // largest A kept in shared memory

struct Cand {
    long long g;
    int a, b;
    int P, Q;  // ranks of a and b when the candidate was taken
};

__device__ __forceinline__ bool better(const Cand &x, const Cand &y)
{
    if (x.a < 0) return false;
    if (y.a < 0) return true;
    if (x.g != y.g) return x.g > y.g;
    if (x.a != y.a) return x.a < y.a;
    return x.b < y.b;
}

__device__ __forceinline__ Cand shfl_cand(const Cand &v, int o)
{
    Cand u;
    u.g = __shfl_xor_sync(0xffffffffu, v.g, o);
    u.a = __shfl_xor_sync(0xffffffffu, v.a, o);
    u.b = __shfl_xor_sync(0xffffffffu, v.b, o);
    u.P = __shfl_xor_sync(0xffffffffu, v.P, o);
    u.Q = __shfl_xor_sync(0xffffffffu, v.Q, o);
    return u;
}

__device__ __forceinline__ Cand warp_best(Cand v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const Cand u = shfl_cand(v, o);
        if (better(u, v)) v = u;
    }
    return v;
}

struct Smem {
    int *p;     // [E] rank of each expert (-1: not placed yet)
    int *fill;  // [R] experts on each rank
    int *mem;   // [E] experts of rank d at mem[d*cap ..]
    int *slot;  // [E] position of e in its rank's list
    int *cb;    // [E] refinement: best partner of row a (-1: no positive gain)
    int *list;  // [E] refinement: rows to rescan in this step
    long long *cg;  // [E] refinement: gain of (a, cb[a])
    long long *A;   // [E][ar]: A[e][d] at A[e * ar + d]
    int ar;         // row stride of A: R + 1, so that consecutive rows fall in different banks
};

// ------------------------------------------------------------ greedy seed
__device__ __forceinline__ bool eligible(const Smem &s, int a, int b, int cap, int maxfree)
{
    const int pa = s.p[a], pb = s.p[b];
    if (pa < 0 && pb < 0) return maxfree >= 2;
    if (pa >= 0 && pb < 0) return s.fill[pa] < cap;
    if (pa < 0 && pb >= 0) return s.fill[pb] < cap;
    return false;
}

// Best eligible partner b > a of row a: heaviest W, lowest b on ties.  The
// whole warp scans, kBatch loads per lane in flight; every lane gets (w, b),
// b = -1 when none.
constexpr int kBatch = 4;

__device__ __forceinline__ void greedy_row(const uint32_t *__restrict__ W, const Smem &s, int E,
                                           int a, int cap, int maxfree, uint32_t &w_out, int &b_out)
{
    const int lane = threadIdx.x & 31;
    uint32_t bw = 0;
    int bb = INT_MAX;
    const uint32_t *row = W + (int64_t)a * E;
    for (int b0 = a + 1; b0 < E; b0 += 32 * kBatch) {
        uint32_t wv[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int b = b0 + u * 32 + lane;
            wv[u] = b < E ? __ldg(row + b) : 0u;
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int b = b0 + u * 32 + lane;
            if (wv[u] > bw && eligible(s, a, b, cap, maxfree)) {
                bw = wv[u];
                bb = b;
            }
        }
    }
    const uint32_t wmax = __reduce_max_sync(0xffffffffu, bw);
    const unsigned bmin = __reduce_min_sync(0xffffffffu, (wmax > 0 && bw == wmax) ? (unsigned)bb
                                                                              : 0xffffffffu);
    w_out = wmax;
    b_out = wmax > 0 ? (int)bmin : -1;
}

// ------------------------------------------------------------- refinement
__device__ __forceinline__ long long gain_w(const Smem &s, int R, int a, int b, uint32_t wab)
{
    const int P = s.p[a], Q = s.p[b];
    const long long *Aa = s.A + (int64_t)a * s.ar, *Ab = s.A + (int64_t)b * s.ar;
    return Aa[Q] - Aa[P] + Ab[P] - Ab[Q] - 2ll * (long long)wab;
}

// Best positive-gain partner b > a (p[b] != p[a]) of row a, lowest b on ties.
__device__ __forceinline__ void refine_row(const uint32_t *__restrict__ W, const Smem &s, int E,
                                           int R, int a, long long &g_out, int &b_out)
{
    const int lane = threadIdx.x & 31;
    const int P = s.p[a];
    const uint32_t *row = W + (int64_t)a * E;
    long long bg = 0;
    int bb = -1;
    for (int b0 = a + 1; b0 < E; b0 += 32 * kBatch) {
        uint32_t wv[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int b = b0 + u * 32 + lane;
            wv[u] = b < E ? __ldg(row + b) : 0u;
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int b = b0 + u * 32 + lane;
            if (b >= E || s.p[b] == P) continue;
            const long long g = gain_w(s, R, a, b, wv[u]);
            if (g > bg) {
                bg = g;
                bb = b;
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const long long g2 = __shfl_xor_sync(0xffffffffu, bg, o);
        const int b2 = __shfl_xor_sync(0xffffffffu, bb, o);
        if (b2 >= 0 && (bb < 0 || g2 > bg || (g2 == bg && b2 < bb))) {
            bg = g2;
            bb = b2;
        }
    }
    g_out = bg;
    b_out = bb;
}

__global__ void __launch_bounds__(kThreads, 1)
    k_place(const uint32_t *__restrict__ W, int E, int R, int seed_mode, int refine,
            int32_t *__restrict__ p_out, long long *__restrict__ A_global, int a_in_smem)
{
    extern __shared__ __align__(16) unsigned char sm_raw[];
    __shared__ Cand s_red[kWarps];
    __shared__ int s_maxfree, s_roomiest, s_nlist;
    const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
    const int cap = E / R;

    Smem s;
    s.A = a_in_smem ? reinterpret_cast<long long *>(sm_raw) : A_global;
    s.ar = R + 1;
    s.cg = reinterpret_cast<long long *>(sm_raw + (a_in_smem ? (size_t)E * (R + 1) * 8 : 0));
    int *ip = reinterpret_cast<int *>(s.cg + E);
    s.p = ip;
    s.fill = ip + E;
    s.mem = ip + E + R;
    s.slot = ip + 2 * E + R;
    s.cb = ip + 3 * E + R;
    s.list = ip + 4 * E + R;

    // greedy seed: lane j of warp w keeps the candidate of row w + 32 j
    const int a_own = wp + 32 * lane;
    const bool own = a_own < E;

    if (seed_mode == MD_SEED_CONTIGUOUS) {
        for (int e = tid; e < E; e += kThreads) s.p[e] = e / cap;
        __syncthreads();
    } else {
        for (int e = tid; e < E; e += kThreads) s.p[e] = -1;
        for (int d = tid; d < R; d += kThreads) s.fill[d] = 0;
        if (tid == 0) {
            s_maxfree = cap;
            s_roomiest = 0;
        }
        __syncthreads();
        uint32_t cw = 0;
        int cb = -2;  // -2: not scanned yet, -1: no eligible partner left
        for (int it = 0; it < E; ++it) {
            const int maxfree = s_maxfree;
            const bool need = own && (cb == -2 || (cb >= 0 && !eligible(s, a_own, cb, cap, maxfree)));
            unsigned m = __ballot_sync(0xffffffffu, need);
            while (m) {
                const int j = __ffs(m) - 1;
                m &= m - 1;
                uint32_t w2;
                int b2;
                greedy_row(W, s, E, wp + 32 * j, cap, maxfree, w2, b2);
                if (lane == j) {
                    cw = w2;
                    cb = b2;
                }
            }
            Cand v = {0, -1, -1, 0, 0};
            if (own && cb >= 0) v = Cand{(long long)cw, a_own, cb, 0, 0};
            v = warp_best(v);
            if (lane == 0) s_red[wp] = v;
            __syncthreads();
            const Cand win = warp_best(s_red[lane]);
            if (win.a < 0) break;  // uniform: every thread holds the same winner
            if (wp == 0) {
                if (lane == 0) {
                    const int pa = s.p[win.a], pb = s.p[win.b];
                    if (pa < 0 && pb < 0) {
                        const int best = s_roomiest;
                        s.p[win.a] = best;
                        s.p[win.b] = best;
                        s.fill[best] += 2;
                    } else if (pa >= 0) {
                        s.p[win.b] = pa;
                        s.fill[pa] += 1;
                    } else {
                        s.p[win.a] = pb;
                        s.fill[pb] += 1;
                    }
                }
                __syncwarp();
                // the rank with the most free slots, lowest index on ties
                unsigned key = 0xffffffffu;
                for (int d = lane; d < R; d += 32) key = min(key, (unsigned)s.fill[d] * 64u + (unsigned)d);
                key = __reduce_min_sync(0xffffffffu, key);
                if (lane == 0) {
                    s_maxfree = cap - (int)(key >> 6);
                    s_roomiest = (int)(key & 63u);
                }
            }
            __syncthreads();
        }
        __syncthreads();
        if (tid == 0) {
            // leftovers ascending into the lowest rank with room; ranks only
            // fill up, so that rank never moves backwards
            int d = 0;
            for (int e = 0; e < E; ++e) {
                if (s.p[e] >= 0) continue;
                while (s.fill[d] >= cap) ++d;
                s.p[e] = d;
                s.fill[d] += 1;
            }
        }
        __syncthreads();
    }

    if (refine) {
        // member lists (in any order: every use breaks ties by expert id) and A
        for (int d = tid; d < R; d += kThreads) s.fill[d] = 0;
        for (int64_t i = tid; i < (int64_t)E * s.ar; i += kThreads) s.A[i] = 0;
        __syncthreads();
        for (int e = tid; e < E; e += kThreads) {
            const int d = s.p[e];
            const int sl = atomicAdd(&s.fill[d], 1);
            s.slot[e] = sl;
            s.mem[d * cap + sl] = e;
        }
        __syncthreads();
        for (int e = wp; e < E; e += kWarps) {
            const uint32_t *row = W + (int64_t)e * E;
            long long *Ae = s.A + (int64_t)e * s.ar;
            for (int e2 = lane; e2 < E; e2 += 32)
                if (e2 != e && row[e2])
                    atomicAdd(reinterpret_cast<unsigned long long *>(&Ae[s.p[e2]]),
                              (unsigned long long)row[e2]);
        }
        __syncthreads();

        for (int a = tid; a < E; a += kThreads) {
            s.cb[a] = -1;
            s.cg[a] = 0;
        }
        if (tid == 0) s_nlist = 0;
        __syncthreads();
        int lastP = -1, lastQ = -1;  // ranks of the last swap (-1: scan every row)
        for (long long it = 0; it < (long long)E * E; ++it) {
            // one thread per row: rows on lastP / lastQ, and rows whose partner
            // sits there, are queued for a full rescan; every other row only
            // compares its candidate with the pairs it forms with those ranks
            for (int a = tid; a < E; a += kThreads) {
                const int pa = s.p[a];
                long long cg = s.cg[a];
                int cb = s.cb[a];
                if (lastP < 0 || pa == lastP || pa == lastQ ||
                    (cb >= 0 && (s.p[cb] == lastP || s.p[cb] == lastQ))) {
                    s.list[atomicAdd(&s_nlist, 1)] = a;
                    continue;
                }
                const uint32_t *row = W + (int64_t)a * E;
                for (int i0 = 0; i0 < 2 * cap; i0 += kBatch) {
                    int bv[kBatch];
                    uint32_t wv[kBatch];
#pragma unroll
                    for (int u = 0; u < kBatch; ++u) {
                        const int i = i0 + u;
                        bv[u] = i < 2 * cap ? s.mem[(i < cap ? lastP * cap + i : lastQ * cap + i - cap)]
                                            : -1;
                        wv[u] = bv[u] > a ? __ldg(row + bv[u]) : 0u;
                    }
#pragma unroll
                    for (int u = 0; u < kBatch; ++u) {
                        const int b = bv[u];
                        if (b <= a) continue;
                        const long long g = gain_w(s, R, a, b, wv[u]);
                        if (g > 0 && (cb < 0 || g > cg || (g == cg && b < cb))) {
                            cg = g;
                            cb = b;
                        }
                    }
                }
                s.cg[a] = cg;
                s.cb[a] = cb;
            }
            __syncthreads();
            // the queued rows, one warp per row over all warps
            const int nl = s_nlist;
            for (int i = wp; i < nl; i += kWarps) {
                const int a = s.list[i];
                long long g2;
                int b2;
                refine_row(W, s, E, R, a, g2, b2);
                if (lane == 0) {
                    s.cg[a] = g2;
                    s.cb[a] = b2;
                }
            }
            __syncthreads();
            Cand v = {0, -1, -1, 0, 0};
            for (int a = tid; a < E; a += kThreads) {
                const int cb = s.cb[a];
                if (cb < 0) continue;
                const Cand c = {s.cg[a], a, cb, s.p[a], s.p[cb]};
                if (better(c, v)) v = c;
            }
            v = warp_best(v);
            if (lane == 0) s_red[wp] = v;
            __syncthreads();
            const Cand win = warp_best(s_red[lane]);
            if (win.a < 0) break;
            const int a = win.a, b = win.b, P = win.P, Q = win.Q;
            for (int e = tid; e < E; e += kThreads) {
                const long long wa = e != a ? (long long)__ldg(W + (int64_t)e * E + a) : 0;
                const long long wb = e != b ? (long long)__ldg(W + (int64_t)e * E + b) : 0;
                s.A[(int64_t)e * s.ar + P] += wb - wa;
                s.A[(int64_t)e * s.ar + Q] += wa - wb;
            }
            if (tid == 0) {
                const int sa = s.slot[a], sb = s.slot[b];
                s.mem[P * cap + sa] = b;
                s.mem[Q * cap + sb] = a;
                s.slot[a] = sb;
                s.slot[b] = sa;
                s.p[a] = Q;
                s.p[b] = P;
                s_nlist = 0;
            }
            lastP = P;
            lastQ = Q;
            __syncthreads();
        }
    }
    for (int e = tid; e < E; e += kThreads) p_out[e] = s.p[e];
}

size_t int_smem(int E, int R) { return (size_t)E * sizeof(long long) + (size_t)(5 * E + R) * sizeof(int); }

}  // namespace

extern "C" size_t md_place_correlated_workspace_size(int E, int R)
{
    if (E < 1 || R < 1) return 0;
    return md::align_up((size_t)E * (R + 1) * sizeof(long long), 256);
}

extern "C" int md_place_correlated(const uint32_t *W, int E, int R, int seed_mode, int refine,
                                   int32_t *expert_to_rank, void *workspace,
                                   size_t workspace_bytes, int32_t *dev_status, void *stream)
{
    if (E < 1 || R < 1 || E % R != 0) return MD_ERR_ARG;
    if (E > MD_MAX_EXPERTS || R > MD_MAX_RANKS) return MD_ERR_UNSUPPORTED;
    if (seed_mode != MD_SEED_CONTIGUOUS && seed_mode != MD_SEED_GREEDY_PAIRS) return MD_ERR_ARG;
    if (!W || !expert_to_rank) return MD_ERR_ARG;
    if (refine && (!workspace || workspace_bytes < md_place_correlated_workspace_size(E, R)))
        return MD_ERR_WORKSPACE;
    cudaStream_t s = md::as_stream(stream);
    int rc = md::clear_status(dev_status, s);
    if (rc != MD_OK) return rc;
    const size_t a_bytes = (size_t)E * (R + 1) * sizeof(long long);
    const int a_in_smem = refine && a_bytes <= kSmemA ? 1 : 0;
    const size_t smem = int_smem(E, R) + (a_in_smem ? a_bytes : 0);
    if (cudaFuncSetAttribute(k_place, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return MD_ERR_CUDA;
    k_place<<<1, kThreads, smem, s>>>(W, E, R, seed_mode, refine ? 1 : 0, expert_to_rank,
                                      static_cast<long long *>(workspace), a_in_smem);
    md::count_launches(1);
    return md::launch_status();
}
