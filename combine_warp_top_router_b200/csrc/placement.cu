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
// For E <= 256, when W is symmetric with entries below 2^16 (co-selection
// counts fitted on fewer than 65536 tokens, or sparse enough), W is copied
// into shared memory as uint16 and A kept as int32 beside it, so that no
// step waits on L2; otherwise W is read from global memory.  The choice is
// made on the device from the data, per problem.
#include <climits>

#include "common.cuh"

namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr size_t kSmemA = 160 * 1024;  // largest A kept in shared memory
constexpr int kCompactMaxE = 256;      // largest E whose W (uint16) fits beside A

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
    unsigned char *lock;  // [E] KL: moved in this pass
    int *ka, *kb, *kP, *kQ;  // [E/2] KL: the moves of this pass
    long long *kg;        // [E/2] KL: their gains
};

// Where W and A live.
//   Store<false>: W (uint32) in global memory, read through L1/L2; A (int64)
//     in shared memory when it fits, else in the workspace.
//   Store<true>, when W is symmetric with entries below 2^16 and row sums
//     below 2^31 (E <= 256): W as uint16 and A as int32, both in shared
//     memory.  Symmetry lets column reads use rows, so threads on
//     consecutive experts read consecutive halfwords.
// A[e][d] sits at A[e * ar + d] with ar = R + 1, so that consecutive rows
// fall in different banks.
template <bool COMPACT>
struct Store;

template <>
struct Store<false> {
    const uint32_t *W;
    long long *A;
    int E, ar;
    __device__ __forceinline__ uint32_t w_row(int a, int b) const  // threads vary b
    {
        return __ldg(W + (int64_t)a * E + b);
    }
    __device__ __forceinline__ uint32_t w_col(int a, int b) const  // threads vary a
    {
        return __ldg(W + (int64_t)a * E + b);
    }
    __device__ __forceinline__ long long a_get(int e, int d) const { return A[(int64_t)e * ar + d]; }
    __device__ __forceinline__ void a_add(int e, int d, long long v) const { A[(int64_t)e * ar + d] += v; }
    __device__ __forceinline__ void a_atomic_add(int e, int d, uint32_t v) const
    {
        atomicAdd(reinterpret_cast<unsigned long long *>(A + (int64_t)e * ar + d), (unsigned long long)v);
    }
    __device__ __forceinline__ void a_zero(int64_t i) const { A[i] = 0; }
};

template <>
struct Store<true> {
    const uint16_t *W;
    int *A;
    int E, ar;
    __device__ __forceinline__ uint32_t w_row(int a, int b) const { return W[a * E + b]; }
    __device__ __forceinline__ uint32_t w_col(int a, int b) const { return W[b * E + a]; }
    __device__ __forceinline__ long long a_get(int e, int d) const { return A[e * ar + d]; }
    __device__ __forceinline__ void a_add(int e, int d, long long v) const { A[e * ar + d] += (int)v; }
    __device__ __forceinline__ void a_atomic_add(int e, int d, uint32_t v) const
    {
        atomicAdd(A + e * ar + d, (int)v);
    }
    __device__ __forceinline__ void a_zero(int64_t i) const { A[i] = 0; }
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

template <class St>
__device__ __forceinline__ void greedy_row(const St &st, const Smem &s, int E, int a, int cap,
                                           int maxfree, uint32_t &w_out, int &b_out)
{
    const int lane = threadIdx.x & 31;
    uint32_t bw = 0;
    int bb = INT_MAX;
    for (int b0 = a + 1; b0 < E; b0 += 32 * kBatch) {
        uint32_t wv[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int b = b0 + u * 32 + lane;
            wv[u] = b < E ? st.w_row(a, b) : 0u;
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
template <class St>
__device__ __forceinline__ long long gain_w(const St &st, const Smem &s, int a, int b, uint32_t wab)
{
    const int P = s.p[a], Q = s.p[b];
    return st.a_get(a, Q) - st.a_get(a, P) + st.a_get(b, P) - st.a_get(b, Q) - 2ll * (long long)wab;
}

// Best partner b > a (p[b] != p[a]) of row a, lowest b on ties: with a
// positive gain for the swap search; any gain, among unlocked experts, in a
// Kernighan-Lin pass (KL).  b = -1 when there is none.
template <bool KL, class St>
__device__ __forceinline__ void refine_row(const St &st, const Smem &s, int E, int a,
                                           long long &g_out, int &b_out)
{
    const int lane = threadIdx.x & 31;
    const int P = s.p[a];
    long long bg = 0;
    int bb = -1;
    for (int b0 = a + 1; b0 < E; b0 += 32 * kBatch) {
        uint32_t wv[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int b = b0 + u * 32 + lane;
            wv[u] = b < E ? st.w_row(a, b) : 0u;
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int b = b0 + u * 32 + lane;
            if (b >= E || s.p[b] == P || (KL && s.lock[b])) continue;
            const long long g = gain_w(st, s, a, b, wv[u]);
            if (KL ? (bb < 0 || g > bg) : g > bg) {
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

// Move a (rank P) to Q and b (rank Q) to P: columns P and Q of A, and (thread
// 0) the rank lists.  The caller synchronises.
template <class St>
__device__ __forceinline__ void apply_swap(const St &st, const Smem &s, int E, int cap, int a,
                                           int b, int P, int Q)
{
    for (int e = threadIdx.x; e < E; e += kThreads) {
        const long long wa = e != a ? (long long)st.w_col(e, a) : 0;
        const long long wb = e != b ? (long long)st.w_col(e, b) : 0;
        st.a_add(e, P, wb - wa);
        st.a_add(e, Q, wa - wb);
    }
    if (threadIdx.x == 0) {
        const int sa = s.slot[a], sb = s.slot[b];
        s.mem[P * cap + sa] = b;
        s.mem[Q * cap + sb] = a;
        s.slot[a] = sb;
        s.slot[b] = sa;
        s.p[a] = Q;
        s.p[b] = P;
    }
}

// The refinement.  !KL: repeat the best positive swap while there is one
// (at most E*E).  KL: passes of tentative moves; each move is the best swap
// among experts not yet moved in the pass, whatever its sign; the pass keeps
// the shortest prefix of moves with the largest positive total and undoes
// the rest; passes repeat while that total is positive (at most E passes).
template <bool KL, class St>
__device__ void search(const St &st, const Smem &s, int E, int R, int cap, Cand *s_red, int *s_nlist,
                       long long *s_keep, int *s_keep_m)
{
    const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
    const long long max_passes = KL ? E : 1;
    const long long max_steps = KL ? E / 2 : (long long)E * E;
    for (long long pass = 0; pass < max_passes; ++pass) {
        for (int a = tid; a < E; a += kThreads) {
            s.cb[a] = -1;
            s.cg[a] = 0;
            if (KL) s.lock[a] = 0;
        }
        if (tid == 0) *s_nlist = 0;
        __syncthreads();
        int lastP = -1, lastQ = -1;  // ranks of the last move (-1: scan every row)
        int moves = 0;
        for (long long it = 0; it < max_steps; ++it) {
            // one thread per row: rows on lastP / lastQ, and rows whose partner
            // sits there, are queued for a full rescan; every other row only
            // compares its candidate with the pairs it forms with those ranks
            for (int a = tid; a < E; a += kThreads) {
                if (KL && s.lock[a]) {
                    s.cb[a] = -1;
                    continue;
                }
                const int pa = s.p[a];
                long long cg = s.cg[a];
                int cb = s.cb[a];
                if (lastP < 0 || pa == lastP || pa == lastQ ||
                    (cb >= 0 && (s.p[cb] == lastP || s.p[cb] == lastQ))) {
                    s.list[atomicAdd(s_nlist, 1)] = a;
                    continue;
                }
                for (int i0 = 0; i0 < 2 * cap; i0 += kBatch) {
                    int bv[kBatch];
                    uint32_t wv[kBatch];
#pragma unroll
                    for (int u = 0; u < kBatch; ++u) {
                        const int i = i0 + u;
                        bv[u] = i < 2 * cap ? s.mem[(i < cap ? lastP * cap + i : lastQ * cap + i - cap)]
                                            : -1;
                        wv[u] = bv[u] > a ? st.w_col(a, bv[u]) : 0u;
                    }
#pragma unroll
                    for (int u = 0; u < kBatch; ++u) {
                        const int b = bv[u];
                        if (b <= a || (KL && s.lock[b])) continue;
                        const long long g = gain_w(st, s, a, b, wv[u]);
                        if ((KL || g > 0) && (cb < 0 || g > cg || (g == cg && b < cb))) {
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
            const int nl = *s_nlist;
            for (int i = wp; i < nl; i += kWarps) {
                const int a = s.list[i];
                long long g2;
                int b2;
                refine_row<KL>(st, s, E, a, g2, b2);
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
            if (win.a < 0) break;  // uniform: every thread holds the same winner
            apply_swap(st, s, E, cap, win.a, win.b, win.P, win.Q);
            if (tid == 0) {
                *s_nlist = 0;
                if (KL) {
                    s.lock[win.a] = 1;
                    s.lock[win.b] = 1;
                    s.ka[moves] = win.a;
                    s.kb[moves] = win.b;
                    s.kP[moves] = win.P;
                    s.kQ[moves] = win.Q;
                    s.kg[moves] = win.g;
                }
            }
            ++moves;
            lastP = win.P;
            lastQ = win.Q;
            __syncthreads();
        }
        if (!KL) break;
        // keep the shortest prefix with the largest total gain, undo the rest
        if (tid == 0) {
            long long run = 0, keep = 0;
            int m = 0;
            for (int i = 0; i < moves; ++i) {
                run += s.kg[i];
                if (run > keep) {
                    keep = run;
                    m = i + 1;
                }
            }
            *s_keep = keep;
            *s_keep_m = m;
        }
        __syncthreads();
        const int m = *s_keep_m;
        const long long keep = *s_keep;
        for (int i = moves - 1; i >= m; --i) {
            // move i took a from P to Q and b from Q to P; take them back
            apply_swap(st, s, E, cap, s.ka[i], s.kb[i], s.kQ[i], s.kP[i]);
            __syncthreads();
        }
        if (keep <= 0) break;
    }
}

// Seed and refinement of one problem, with W and A where `st` says.
template <class St>
__device__ void place_body(const St &st, const Smem &s, int E, int R, int seed_mode, int refine,
                           Cand *s_red, int *s_maxfree, int *s_roomiest, int *s_nlist,
                           long long *s_keep, int *s_keep_m)
{
    const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
    const int cap = E / R;
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
            *s_maxfree = cap;
            *s_roomiest = 0;
        }
        __syncthreads();
        uint32_t cw = 0;
        int cb = -2;  // -2: not scanned yet, -1: no eligible partner left
        for (int it = 0; it < E; ++it) {
            const int maxfree = *s_maxfree;
            const bool need = own && (cb == -2 || (cb >= 0 && !eligible(s, a_own, cb, cap, maxfree)));
            unsigned m = __ballot_sync(0xffffffffu, need);
            while (m) {
                const int j = __ffs(m) - 1;
                m &= m - 1;
                uint32_t w2;
                int b2;
                greedy_row(st, s, E, wp + 32 * j, cap, maxfree, w2, b2);
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
                        const int best = *s_roomiest;
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
                    *s_maxfree = cap - (int)(key >> 6);
                    *s_roomiest = (int)(key & 63u);
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
        for (int64_t i = tid; i < (int64_t)E * st.ar; i += kThreads) st.a_zero(i);
        __syncthreads();
        for (int e = tid; e < E; e += kThreads) {
            const int d = s.p[e];
            const int sl = atomicAdd(&s.fill[d], 1);
            s.slot[e] = sl;
            s.mem[d * cap + sl] = e;
        }
        __syncthreads();
        for (int e = wp; e < E; e += kWarps)
            for (int e2 = lane; e2 < E; e2 += 32) {
                const uint32_t v = st.w_row(e, e2);
                if (e2 != e && v) st.a_atomic_add(e, s.p[e2], v);
            }
        __syncthreads();
        if (refine == 1) search<false>(st, s, E, R, cap, s_red, s_nlist, s_keep, s_keep_m);
        else search<true>(st, s, E, R, cap, s_red, s_nlist, s_keep, s_keep_m);
    }
}

// One CTA per independent problem (blockIdx.x): W, p_out and A_global point
// at problem 0 and advance by E*E, E and E*(R+1).  refine: 0 none, 1 best
// single swaps, 2 Kernighan-Lin passes.  The first `region` bytes of dynamic
// shared memory hold A (a_in_smem), or W and A compacted when compact_ok and
// the problem's W allows it; the index arrays follow.
__global__ void __launch_bounds__(kThreads, 1)
    k_place(const uint32_t *__restrict__ W, int E, int R, int seed_mode, int refine,
            int32_t *__restrict__ p_out, long long *__restrict__ A_global, int a_in_smem,
            int compact_ok, int region)
{
    extern __shared__ __align__(16) unsigned char sm_raw[];
    __shared__ Cand s_red[kWarps];
    __shared__ int s_maxfree, s_roomiest, s_nlist, s_keep_m;
    __shared__ long long s_keep;
    const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
    W += (int64_t)blockIdx.x * E * E;
    p_out += (int64_t)blockIdx.x * E;
    if (A_global) A_global += (int64_t)blockIdx.x * E * (R + 1);

    Smem s;
    s.cg = reinterpret_cast<long long *>(sm_raw + region);
    int *ip = reinterpret_cast<int *>(s.cg + E);
    s.p = ip;
    s.fill = ip + E;
    s.mem = ip + E + R;
    s.slot = ip + 2 * E + R;
    s.cb = ip + 3 * E + R;
    s.list = ip + 4 * E + R;
    {
        // KL records after the int arrays: ka, kb, kP, kQ [E/2 + 1] ints, kg
        // [E/2 + 1] int64 (8-byte aligned), lock [E] bytes
        int *kp = ip + 5 * E + R;
        const int h = E / 2 + 1;
        s.ka = kp;
        s.kb = kp + h;
        s.kP = kp + 2 * h;
        s.kQ = kp + 3 * h;
        unsigned char *after = reinterpret_cast<unsigned char *>(kp + 4 * h);
        after = reinterpret_cast<unsigned char *>(((uintptr_t)after + 7) & ~(uintptr_t)7);
        s.kg = reinterpret_cast<long long *>(after);
        s.lock = reinterpret_cast<unsigned char *>(s.kg + h);
    }

    int compact = 0;
    if (compact_ok) {
        // W symmetric, entries below 2^16, row sums (off the diagonal) below 2^31
        int bad = 0;
        for (int64_t i = tid; i < (int64_t)E * E; i += kThreads) {
            const int a = (int)(i / E), b = (int)(i - (int64_t)a * E);
            const uint32_t v = __ldg(W + i);
            if (v > 0xffffu || (b > a && v != __ldg(W + (int64_t)b * E + a))) bad = 1;
        }
        for (int e = wp; e < E; e += kWarps) {
            unsigned long long rs = 0;
            for (int e2 = lane; e2 < E; e2 += 32)
                if (e2 != e) rs += __ldg(W + (int64_t)e * E + e2);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) rs += __shfl_xor_sync(0xffffffffu, rs, o);
            if (rs >= (1ull << 31)) bad = 1;
        }
        compact = !__syncthreads_or(bad);
        if (compact) {
            uint16_t *w16 = reinterpret_cast<uint16_t *>(sm_raw);
            for (int64_t i = tid; i < (int64_t)E * E; i += kThreads) w16[i] = (uint16_t)__ldg(W + i);
        }
        __syncthreads();
    }
    if (compact) {
        const size_t wb = ((size_t)E * E * 2 + 15) & ~(size_t)15;
        const Store<true> st{reinterpret_cast<const uint16_t *>(sm_raw),
                             reinterpret_cast<int *>(sm_raw + wb), E, R + 1};
        place_body(st, s, E, R, seed_mode, refine, s_red, &s_maxfree, &s_roomiest, &s_nlist, &s_keep,
                   &s_keep_m);
    } else {
        const Store<false> st{W, a_in_smem ? reinterpret_cast<long long *>(sm_raw) : A_global, E, R + 1};
        place_body(st, s, E, R, seed_mode, refine, s_red, &s_maxfree, &s_roomiest, &s_nlist, &s_keep,
                   &s_keep_m);
    }
    for (int e = tid; e < E; e += kThreads) p_out[e] = s.p[e];
}

size_t int_smem(int E, int R)
{
    const size_t h = (size_t)E / 2 + 1;
    return (size_t)E * sizeof(long long) + (size_t)(5 * E + R) * sizeof(int) + 4 * h * sizeof(int) +
           8 + h * sizeof(long long) + (size_t)E;
}

// Two-level placement, between the levels: the experts of each node in
// ascending id (mem[n*En + i]) and the node's restriction of W
// (sub[n][i][j] = W[mem_i][mem_j]).  One CTA; E <= 1024.
__global__ void __launch_bounds__(kThreads)
    k_node_split(const uint32_t *__restrict__ W, int E, int nodes, const int32_t *__restrict__ pn,
                 int32_t *__restrict__ mem, uint32_t *__restrict__ sub)
{
    const int En = E / nodes;
    for (int e = threadIdx.x; e < E; e += kThreads) {
        const int n = pn[e];
        int pos = 0;
        for (int e2 = 0; e2 < e; ++e2) pos += pn[e2] == n;
        mem[n * En + pos] = e;
    }
    __syncthreads();
    const int64_t cells = (int64_t)E * En;  // nodes * En * En
    for (int64_t c = threadIdx.x; c < cells; c += kThreads) {
        const int n = (int)(c / ((int64_t)En * En));
        const int64_t r = c - (int64_t)n * En * En;
        const int i = (int)(r / En), j = (int)(r - (int64_t)i * En);
        sub[c] = W[(int64_t)mem[n * En + i] * E + mem[n * En + j]];
    }
}

// p[mem[n*En + i]] = n * G + pg[n*En + i]
__global__ void k_node_merge(int E, int nodes, int G, const int32_t *__restrict__ mem,
                             const int32_t *__restrict__ pg, int32_t *__restrict__ p)
{
    const int En = E / nodes;
    for (int c = blockIdx.x * blockDim.x + threadIdx.x; c < E; c += gridDim.x * blockDim.x)
        p[mem[c]] = (c / En) * G + pg[c];
}

int launch_place(const uint32_t *W, int problems, int E, int R, int seed_mode, int refine,
                 int32_t *p, long long *A, cudaStream_t s)
{
    const size_t a_bytes = (size_t)E * (R + 1) * sizeof(long long);
    const int a_in_smem = refine && a_bytes <= kSmemA ? 1 : 0;
    // W (uint16) and A (int32) in shared memory, if the data allows it
    const size_t c_bytes = ((size_t)E * E * 2 + 15) / 16 * 16 + (size_t)E * (R + 1) * sizeof(int);
    const int compact_ok = E <= kCompactMaxE ? 1 : 0;
    size_t region = a_in_smem ? a_bytes : 0;
    if (compact_ok && c_bytes > region) region = c_bytes;
    region = md::align_up(region, 16);
    const size_t smem = region + int_smem(E, R);
    if (cudaFuncSetAttribute(k_place, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return MD_ERR_CUDA;
    k_place<<<problems, kThreads, smem, s>>>(W, E, R, seed_mode, refine, p, A, a_in_smem, compact_ok,
                                             (int)region);
    md::count_launches(1);
    return MD_OK;
}

struct PlaceWs {
    long long *A1, *A2;
    int32_t *pn, *mem, *pg;
    uint32_t *sub;
};

size_t place_layout(int E, int R, int nodes, PlaceWs *w, void *base)
{
    char *b = static_cast<char *>(base);
    size_t o = 0;
    auto take = [&](size_t bytes) {
        char *q = b ? b + o : nullptr;
        o += md::align_up(bytes, 256);
        return q;
    };
    PlaceWs x{};
    x.A1 = reinterpret_cast<long long *>(take((size_t)E * (nodes + 1) * sizeof(long long)));
    if (nodes > 1) {
        x.A2 = reinterpret_cast<long long *>(take((size_t)E * (R / nodes + 1) * sizeof(long long)));
        x.pn = reinterpret_cast<int32_t *>(take((size_t)E * 4));
        x.mem = reinterpret_cast<int32_t *>(take((size_t)E * 4));
        x.pg = reinterpret_cast<int32_t *>(take((size_t)E * 4));
        x.sub = reinterpret_cast<uint32_t *>(take((size_t)E * (E / nodes) * 4));
    }
    if (w) *w = x;
    return o;
}

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
    rc = launch_place(W, 1, E, R, seed_mode, refine ? 1 : 0, expert_to_rank,
                      static_cast<long long *>(workspace), s);
    return rc != MD_OK ? rc : md::launch_status();
}

extern "C" size_t md_place_two_level_workspace_size(int E, int R, int nodes)
{
    if (E < 1 || R < 1 || nodes < 1 || R % nodes != 0) return 0;
    return place_layout(E, R, nodes, nullptr, nullptr);
}

extern "C" int md_place_two_level(const uint32_t *W, int E, int R, int nodes, int seed_mode,
                                  int refine_mode, int32_t *expert_to_rank, void *workspace,
                                  size_t workspace_bytes, int32_t *dev_status, void *stream)
{
    if (E < 1 || R < 1 || nodes < 1 || R % nodes != 0 || E % R != 0) return MD_ERR_ARG;
    if (E > MD_MAX_EXPERTS || R > MD_MAX_RANKS) return MD_ERR_UNSUPPORTED;
    if (seed_mode != MD_SEED_CONTIGUOUS && seed_mode != MD_SEED_GREEDY_PAIRS) return MD_ERR_ARG;
    if (refine_mode != MD_REFINE_NONE && refine_mode != MD_REFINE_SWAPS &&
        refine_mode != MD_REFINE_KL)
        return MD_ERR_ARG;
    if (!W || !expert_to_rank) return MD_ERR_ARG;
    if (!workspace || workspace_bytes < md_place_two_level_workspace_size(E, R, nodes))
        return MD_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MD_ERR_ARG;
    cudaStream_t s = md::as_stream(stream);
    int rc = md::clear_status(dev_status, s);
    if (rc != MD_OK) return rc;
    PlaceWs w;
    place_layout(E, R, nodes, &w, workspace);
    if (nodes == 1) {
        rc = launch_place(W, 1, E, R, seed_mode, refine_mode, expert_to_rank, w.A1, s);
        return rc != MD_OK ? rc : md::launch_status();
    }
    const int G = R / nodes, En = E / nodes;
    rc = launch_place(W, 1, E, nodes, seed_mode, refine_mode, w.pn, w.A1, s);
    if (rc != MD_OK) return rc;
    k_node_split<<<1, kThreads, 0, s>>>(W, E, nodes, w.pn, w.mem, w.sub);
    md::count_launches(1);
    rc = launch_place(w.sub, nodes, En, G, seed_mode, refine_mode, w.pg, w.A2, s);
    if (rc != MD_OK) return rc;
    k_node_merge<<<(E + 255) / 256, 256, 0, s>>>(E, nodes, G, w.mem, w.pg, expert_to_rank);
    md::count_launches(1);
    return md::launch_status();
}
