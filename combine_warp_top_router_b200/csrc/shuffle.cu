// shuffle.cu -- capacity-constrained token shuffle (md_token_shuffle).
//
// "Expert Coupling in MoE Pretraining" (PicX summary), Method 2 (Token
// Shuffling), Mechanism: the planner predicts each token's owner rank at layer
// l+1; every rank must own exactly T/EP tokens, so tokens are assigned in
// decreasing confidence to their most preferred rank with capacity left.
// Single-expert prediction from the layer-l top-1 expert e1: first choice
// p_next[argmax_e' C[e1][e']], then the other ranks by their share of row e1.
//
// Everything a token needs depends only on e1, so it is computed per expert:
//   k_shuf_prefs    one CTA per expert row: row sum, arg-max, per-rank sums,
//                   preference list, confidence numerator / denominator.
//   k_shuf_class    class[e] = number of experts with strictly larger
//                   confidence (exact 128-bit cross products); empty rows
//                   get class E.  Equal confidences share a class.
//   bucket sort     stable counting sort of the tokens by class (so tokens
//                   are visited by confidence desc, t asc): per-tile
//                   histograms, a column scan, and a one-warp-per-tile
//                   stable scatter using __match_any_sync.
//   k_shuf_greedy   one CTA walks the sorted tokens 1024 at a time.  Each
//                   token takes its first preferred rank that is not full,
//                   looked up per expert.  A chunk in which no rank reaches
//                   T/R is committed at once; otherwise the CTA finds the
//                   first position where a rank fills, commits up to it,
//                   marks that rank full and re-evaluates the rest of the
//                   chunk, which gives exactly the sequential visit (at most
//                   R refills in all).
//   bucket sort     stable partition by assigned rank gives perm / inv: rank
//                   d's tokens take positions d*T/R .. in ascending t.
#include <climits>

#include "common.cuh"

namespace {

constexpr int kTile = 1024;  // items per bucket-sort tile

// bytes per token preference list in the pair form: a multiple of 16, so that
// a list moves by 16-byte async copies
inline __host__ __device__ int pref_stride(int R) { return (R + 15) / 16 * 16; }

struct ShufWs {
    int32_t *pref;                 // [E*R]
    unsigned long long *num, *den; // [E]
    int32_t *cls;                  // [E]
    int32_t *order;                // [T]
    int32_t *keys;                 // [T] bucket of each token in the current sort
    int32_t *tile_hist;            // [(n_tiles + 1) * max(E+1, R)]
};

size_t shuf_layout(int64_t T, int E, int R, ShufWs *w, void *base)
{
    char *b = static_cast<char *>(base);
    size_t o = 0;
    auto take = [&](size_t bytes) {
        char *p = b ? b + o : nullptr;
        o += md::align_up(bytes, 256);
        return p;
    };
    const int64_t n_tiles = (T + kTile - 1) / kTile;
    ShufWs x;
    x.pref = reinterpret_cast<int32_t *>(take((size_t)E * R * 4));
    x.num = reinterpret_cast<unsigned long long *>(take((size_t)E * 8));
    x.den = reinterpret_cast<unsigned long long *>(take((size_t)E * 8));
    x.cls = reinterpret_cast<int32_t *>(take((size_t)E * 4));
    x.order = reinterpret_cast<int32_t *>(take((size_t)(T > 0 ? T : 1) * 4));
    x.keys = reinterpret_cast<int32_t *>(take((size_t)(T > 0 ? T : 1) * 4));
    const int nbk = E + 1 > R ? E + 1 : R;
    x.tile_hist = reinterpret_cast<int32_t *>(take((size_t)((n_tiles > 0 ? n_tiles : 1) + 1) * nbk * 4));
    if (w) *w = x;
    return o;
}

// ------------------------------------------------------ per-expert tables
__global__ void __launch_bounds__(256)
    k_shuf_prefs(const uint32_t *__restrict__ C, const int32_t *__restrict__ p_next, int E, int R,
                 ShufWs ws, int32_t *status)
{
    __shared__ unsigned long long s_sig[MD_MAX_RANKS];
    __shared__ unsigned long long s_tot[8];
    __shared__ uint32_t s_bv[8];
    __shared__ int s_be[8];
    __shared__ int s_first;
    const int e1 = blockIdx.x, tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    for (int d = tid; d < R; d += 256) s_sig[d] = 0ull;
    __syncthreads();
    const uint32_t *row = C + (int64_t)e1 * E;
    unsigned long long tot = 0;
    uint32_t bv = 0;
    int be = INT_MAX;
    for (int e = tid; e < E; e += 256) {
        const uint32_t v = row[e];
        tot += v;
        if (v > bv || (v == bv && e < be)) { bv = v; be = e; }
        const int d = p_next[e];
        if (d < 0 || d >= R) {
            if (e1 == 0) md::report(status, MD_ERR_DATA);
            continue;
        }
        if (v) atomicAdd(&s_sig[d], (unsigned long long)v);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        tot += __shfl_xor_sync(0xffffffffu, tot, o);
        const uint32_t v2 = __shfl_xor_sync(0xffffffffu, bv, o);
        const int e2 = __shfl_xor_sync(0xffffffffu, be, o);
        if (v2 > bv || (v2 == bv && e2 < be)) { bv = v2; be = e2; }
    }
    if (lane == 0) { s_tot[w] = tot; s_bv[w] = bv; s_be[w] = be; }
    __syncthreads();
    if (tid == 0) {
        for (int i = 1; i < 8; ++i) {
            s_tot[0] += s_tot[i];
            if (s_bv[i] > s_bv[0] || (s_bv[i] == s_bv[0] && s_be[i] < s_be[0])) {
                s_bv[0] = s_bv[i];
                s_be[0] = s_be[i];
            }
        }
        int d0 = p_next[s_be[0]];
        if (d0 < 0 || d0 >= R) d0 = 0;
        s_first = d0;
        ws.num[e1] = s_bv[0];
        ws.den[e1] = s_tot[0];
    }
    __syncthreads();
    const int first = s_first;
    for (int d = tid; d < R; d += 256) {
        int pos = 0;
        if (d != first) {
            pos = 1;
            for (int d2 = 0; d2 < R; ++d2)
                if (d2 != first && d2 != d &&
                    (s_sig[d2] > s_sig[d] || (s_sig[d2] == s_sig[d] && d2 < d)))
                    ++pos;
        }
        ws.pref[(int64_t)e1 * R + pos] = d;
    }
}

__global__ void __launch_bounds__(256) k_shuf_class(int E, ShufWs ws)
{
    const int e = blockIdx.x * 256 + threadIdx.x;
    if (e >= E) return;
    const unsigned long long n = ws.num[e], d = ws.den[e];
    if (d == 0) { ws.cls[e] = E; return; }
    int c = 0;
    for (int e2 = 0; e2 < E; ++e2) {
        const unsigned long long d2 = ws.den[e2];
        if (d2 == 0) continue;
        // conf(e2) > conf(e)  <=>  num2 * d > n * d2
        if ((unsigned __int128)ws.num[e2] * d > (unsigned __int128)n * d2) ++c;
    }
    ws.cls[e] = c;
}

// ------------------------------------------------------------ bucket sort
// key source 0: confidence class of the token's top-1 expert (E+1 buckets);
// key source 1: assigned rank (R buckets).
__device__ __forceinline__ int bucket_key(int src, int64_t t, const int32_t *idx_l, int k,
                                          const int32_t *cls, int E, const int32_t *pred, int nbk)
{
    if (src == 0) {
        const int e1 = idx_l[t * k];
        return (e1 >= 0 && e1 < E) ? cls[e1] : E;
    }
    const int d = pred[t];
    return d >= 0 && d < nbk ? d : 0;  // every token is assigned; keep bounds anyway
}

// Per-tile histograms; each token's bucket is also stored for the scatter.
__global__ void __launch_bounds__(256)
    k_bucket_hist(int src, int64_t T, const int32_t *__restrict__ idx_l, int k,
                  const int32_t *__restrict__ cls, int E, const int32_t *__restrict__ pred, int nbk,
                  int32_t *__restrict__ keys, int32_t *__restrict__ tile_hist)
{
    extern __shared__ int h[];
    for (int b = threadIdx.x; b < nbk; b += 256) h[b] = 0;
    __syncthreads();
    const int64_t t0 = (int64_t)blockIdx.x * kTile;
    for (int i = threadIdx.x; i < kTile; i += 256) {
        const int64_t t = t0 + i;
        if (t < T) {
            const int key = bucket_key(src, t, idx_l, k, cls, E, pred, nbk);
            keys[t] = key;
            atomicAdd(&h[key], 1);
        }
    }
    __syncthreads();
    for (int b = threadIdx.x; b < nbk; b += 256) tile_hist[(int64_t)blockIdx.x * nbk + b] = h[b];
}

// LSD radix sort of the 64-bit confidence keys (pair form of the shuffle):
// 11-bit digits, at most six passes.
constexpr int kRadixBits = 11;
constexpr int kRadixBuckets = 1 << kRadixBits;
constexpr int kRadixPasses = (64 + kRadixBits - 1) / kRadixBits;

// Fewer digits suffice when the row totals are small.  With every total below
// 2^b, two different fractions differ by more than 2^-2b, so
// floor(num * 2^S / den) with S = 2b + 1 still orders them exactly and keeps
// equal ones equal; it is key >> (63 - S) (a floor of a floor), and it needs
// S + 1 bits.  The passes above those bits would see one constant digit, an
// identity for a stable sort, and are skipped.
struct RadixPlan {
    int r;      // right shift of the 63-bit key
    int passes; // LSD passes needed
};

__device__ __forceinline__ RadixPlan radix_plan(const uint32_t *maxden)
{
    const uint32_t d = *maxden;
    const int b = d ? 32 - __clz(d) : 0;
    const int S = 2 * b + 1 < 63 ? 2 * b + 1 : 63;
    return {63 - S, (S + 1 + kRadixBits - 1) / kRadixBits};
}

// tile_hist[tile][b] <- items of bucket b in the tiles before `tile` (column
// scan), and row n_tiles <- the first output position of bucket b (scan of
// the bucket totals); a scatter starts bucket b of a tile at the sum of the
// two.  One thread per bucket walks its column with 8 loads in flight
// (adjacent threads read adjacent buckets, so each tile row is coalesced).
constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads)
    k_bucket_scan(int32_t *__restrict__ tile_hist, int n_tiles, int nbk)
{
    extern __shared__ int tot[];
    __shared__ int s_warp[kScanThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
    for (int b = tid; b < nbk; b += kScanThreads) {
        int run = 0;
        for (int i0 = 0; i0 < n_tiles; i0 += 8) {
            int v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                v[u] = i0 + u < n_tiles ? tile_hist[(int64_t)(i0 + u) * nbk + b] : 0;
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (i0 + u < n_tiles) {
                    tile_hist[(int64_t)(i0 + u) * nbk + b] = run;
                    run += v[u];
                }
        }
        tot[b] = run;
    }
    __syncthreads();
    // exclusive scan of the bucket totals: thread i takes a contiguous run
    const int per = (nbk + kScanThreads - 1) / kScanThreads;
    const int lo = tid * per, hi = min(nbk, lo + per);
    int sum = 0;
    for (int b = lo; b < hi; ++b) sum += tot[b];
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) s_warp[wp] = incl;
    __syncthreads();
    if (wp == 0) {
        int w = s_warp[lane], wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += y;
        }
        s_warp[lane] = wi - w;
    }
    __syncthreads();
    int run = s_warp[wp] + incl - sum;
    int32_t *base = tile_hist + (int64_t)n_tiles * nbk;
    for (int b = lo; b < hi; ++b) {
        base[b] = run;
        run += tot[b];
    }
}

// One warp per tile: items in ascending t, stable within each bucket.  The
// tile's 1024 keys are loaded up front (32 per lane).
__global__ void __launch_bounds__(32)
    k_bucket_scatter(int src, int64_t T, int nbk, const int32_t *__restrict__ keys,
                     const int32_t *__restrict__ tile_hist, int32_t *__restrict__ order,
                     int32_t *__restrict__ perm, int32_t *__restrict__ inv)
{
    extern __shared__ int cnt[];
    const int lane = threadIdx.x;
    const int32_t *base = tile_hist + (int64_t)gridDim.x * nbk;
    for (int b = lane; b < nbk; b += 32) cnt[b] = tile_hist[(int64_t)blockIdx.x * nbk + b] + base[b];
    const int64_t t0 = (int64_t)blockIdx.x * kTile;
    int kv[kTile / 32];
#pragma unroll
    for (int c = 0; c < kTile / 32; ++c) {
        const int64_t t = t0 + c * 32 + lane;
        kv[c] = t < T ? keys[t] : -1;
    }
    __syncwarp();
#pragma unroll
    for (int c = 0; c < kTile / 32; ++c) {
        const int64_t t = t0 + c * 32 + lane;
        const int key = kv[c];
        const bool in = key >= 0;
        const unsigned g = __match_any_sync(0xffffffffu, in ? (unsigned)key : (0x80000000u | lane));
        int pos = 0;
        if (in) pos = cnt[key] + __popc(g & md::lanemask_lt());
        __syncwarp();
        if (in && (g >> lane) == 1u) cnt[key] += __popc(g);
        __syncwarp();
        if (in) {
            if (src == 0) {
                order[pos] = (int32_t)t;
            } else {
                perm[t] = pos;
                inv[pos] = (int32_t)t;
            }
        }
    }
}

// ----------------------------------------------------------------- greedy
// A token's choice depends only on its top-1 expert and on which ranks are
// full, and the set of full ranks changes at most R times.  So the CTA keeps
// first[e] = the first rank in e's preference list that is not full (-1 for
// an empty row), and walks the sorted tokens 1024 at a time:
//   every token looks up its choice; the chunk's per-rank totals are added
//   up (one shared atomic per warp and rank); if no rank goes past T/R the
//   whole chunk is committed at once.  Otherwise the first position where a
//   rank reaches T/R is found from per-warp counts, the chunk is committed up
//   to it, that rank is marked full, first[] is recomputed and the rest of
//   the chunk is re-evaluated: exactly the sequential visit.
// A chunk with no fill event crosses a single block barrier: the per-rank
// totals go to one of three buffers and the loads to one of two, and every
// warp reads them back after the barrier and reaches the same decision.
constexpr int kGreedyThreads = 1024;
constexpr int kGreedyWarps = kGreedyThreads / 32;

// PAIR: the prediction row differs per token, so instead of first[e] each
// token walks its own preference list, and an empty row is marked by a zero
// confidence key.  A thread's list is staged in shared memory by 16-byte
// async copies one chunk ahead (two buffers), so walks after a fill event
// read shared memory only.
template <bool PAIR>
__global__ void __launch_bounds__(kGreedyThreads, 1)
    k_shuf_greedy(const int32_t *__restrict__ order, const int32_t *__restrict__ idx_l, int k,
                  ShufWs ws, const unsigned char *__restrict__ tpref,
                  const unsigned long long *__restrict__ tconf, int64_t T, int E, int R, int64_t Tr,
                  int32_t *__restrict__ pred, int32_t *status,
                  const int32_t *__restrict__ order_even = nullptr,
                  const uint32_t *__restrict__ maxden = nullptr)
{
    // pair form: the radix sort ran radix_plan(maxden).passes passes, which
    // alternate between two buffers starting with `order`; an even count ends
    // in `order_even`
    if (PAIR && maxden && (radix_plan(maxden).passes & 1) == 0) order = order_even;
    extern __shared__ __align__(16) unsigned char g_raw[];
    int *s_first = reinterpret_cast<int *>(g_raw);                    // [E]
    unsigned char *s_pref = g_raw + (size_t)E * sizeof(int);          // [E*R]
    // per-rank loads (two buffers) and per-rank totals of an evaluation (three
    // buffers): a chunk with no fill event crosses one block barrier, so each
    // buffer is rewritten only once no thread can still read it
    __shared__ long long s_load[2][MD_MAX_RANKS];
    __shared__ int s_tot[3][MD_MAX_RANKS];
    __shared__ int s_cnt[kGreedyWarps][MD_MAX_RANKS];
    __shared__ unsigned s_msk[kGreedyWarps][MD_MAX_RANKS];
    __shared__ int s_pmin;
    const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;

    if (!PAIR)
        for (int i = tid; i < E * R; i += kGreedyThreads) s_pref[i] = (unsigned char)ws.pref[i];
    for (int i = tid; i < 2 * MD_MAX_RANKS; i += kGreedyThreads) (&s_load[0][0])[i] = 0;
    for (int i = tid; i < 3 * MD_MAX_RANKS; i += kGreedyThreads) (&s_tot[0][0])[i] = 0;
    __syncthreads();
    if (!PAIR)
        for (int e = tid; e < E; e += kGreedyThreads)
            s_first[e] = ws.den[e] == 0ull ? -1 : (int)s_pref[(size_t)e * R];
    __syncthreads();

    // The set of full ranks: every thread keeps the same copy, derived from
    // the same shared words after a barrier, so every branch on it is uniform.
    unsigned long long full = 0ull;
    const unsigned long long all_ranks = R == 64 ? ~0ull : (1ull << R) - 1ull;
    int first_any = 0;  // the lowest rank that is not full (0 once all are)
    int lb = 0, tb = 0;  // current load and total buffers
    auto refresh_first = [&]() {
        const unsigned long long open = ~full & all_ranks;
        first_any = open ? __ffsll((long long)open) - 1 : 0;
        for (int e = tid; !PAIR && e < E; e += kGreedyThreads) {
            if (s_first[e] < 0) continue;
            const unsigned char *pl = s_pref + (size_t)e * R;
            int n = 0;
            while (n < R && ((full >> pl[n]) & 1ull)) ++n;
            s_first[e] = n < R ? (int)pl[n] : 0;
        }
    };

    // token ids are fetched two chunks ahead and their top-1 experts one chunk
    // ahead, so neither load is waited on in the chunk that uses it
    auto token_at = [&](int64_t base) -> int64_t {
        const int64_t pos = base + tid;
        return pos < T ? (int64_t)order[pos] : -1;
    };
    // pair: per-thread list slots, two chunk buffers
    const int Rs = pref_stride(R);
    unsigned char *s_lists = g_raw;
    auto stage_list = [&](int64_t t, int buf) {
        if (PAIR && t >= 0) {
            unsigned char *dst = s_lists + ((size_t)buf * kGreedyThreads + tid) * Rs;
            const unsigned char *src = tpref + t * Rs;
            for (int o = 0; o < Rs; o += 16)
                asm volatile("cp.async.ca.shared.global [%0], [%1], 16;" ::"r"(md::smem_addr(dst + o)),
                             "l"(src + o)
                             : "memory");
        }
        if (PAIR) asm volatile("cp.async.commit_group;" ::: "memory");
    };
    // single: the top-1 expert; pair: 1 when the token's prediction row is empty
    auto key_of = [&](int64_t t) -> int {
        if (t < 0) return 0;
        if (PAIR) return tconf[t] == 0ull ? 1 : 0;
        return idx_l[t * k];
    };
    int64_t t_n1 = token_at(0);
    int e_n1 = key_of(t_n1);
    stage_list(t_n1, 0);
    int64_t t_n2 = token_at(kGreedyThreads);

    int chunk = 0;
    for (int64_t base = 0; base < T; base += kGreedyThreads, ++chunk) {
        const int64_t t = t_n1;
        int e1 = e_n1;
        t_n1 = t_n2;
        e_n1 = key_of(t_n1);
        stage_list(t_n1, (chunk + 1) & 1);
        t_n2 = token_at(base + 2 * kGreedyThreads);
        // this chunk's list copies are done (the next chunk's may be pending)
        if (PAIR) asm volatile("cp.async.wait_group 1;" ::: "memory");
        const unsigned char *my_list = s_lists + ((size_t)(chunk & 1) * kGreedyThreads + tid) * Rs;
        const bool have = t >= 0;
        if (!PAIR && have && (e1 < 0 || e1 >= E)) {
            md::report(status, MD_ERR_DATA);
            e1 = 0;
        }
        const int src_rank = have ? (int)(t / Tr) : 0;
        int start = 0;
        while (true) {
            // choice under the current set of full ranks
            int ch = -1;
            if (have && tid >= start) {
                int f;
                if (PAIR) {
                    f = -1;
                    if (!e1) {
                        const unsigned char *pl = my_list;
                        int n = 0;
                        while (n < R && ((full >> pl[n]) & 1ull)) ++n;
                        f = n < R ? (int)pl[n] : 0;
                    }
                } else {
                    f = s_first[e1];
                }
                ch = f >= 0 ? f : (((full >> src_rank) & 1ull) ? first_any : src_rank);
            }
            const unsigned g =
                __match_any_sync(0xffffffffu, ch >= 0 ? (unsigned)ch : (0x80000000u | lane));
            const bool leader = ch >= 0 && (g & md::lanemask_lt()) == 0u;
            if (leader) atomicAdd(&s_tot[tb][ch], __popc(g));
            __syncthreads();
            // every warp reads the loads and this evaluation's totals: does a
            // rank go past T/R, and which ranks end exactly at T/R
            bool over = false;
            unsigned long long at_cap = 0ull;
            for (int d0 = 0; d0 < R; d0 += 32) {
                const int d = d0 + lane;
                const long long nl = d < R ? s_load[lb][d] + s_tot[tb][d] : 0;
                over |= __any_sync(0xffffffffu, d < R && nl > Tr);
                at_cap |= (unsigned long long)__ballot_sync(0xffffffffu, d < R && nl == Tr) << d0;
            }
            if (!over) {
                // no rank goes past T/R: commit the rest of the chunk at once
                if (ch >= 0) pred[t] = ch;
                for (int d = tid; d < R; d += kGreedyThreads) {
                    s_load[lb ^ 1][d] = s_load[lb][d] + s_tot[tb][d];
                    s_tot[tb == 0 ? 2 : tb - 1][d] = 0;  // the previous evaluation's buffer
                }
                lb ^= 1;
                tb = tb == 2 ? 0 : tb + 1;
                if (at_cap & ~full) {
                    full |= at_cap;
                    // every thread chose before the barrier above, so the
                    // per-expert choices can be rewritten now
                    refresh_first();
                    if (!PAIR) __syncthreads();
                }
                break;
            }
            // some rank goes past T/R: find the first position where a rank fills
            for (int i = tid; i < kGreedyWarps * MD_MAX_RANKS; i += kGreedyThreads)
                (&s_cnt[0][0])[i] = 0;
            if (tid == 0) s_pmin = INT_MAX;
            __syncthreads();
            if (leader) {
                s_cnt[wp][ch] = __popc(g);
                s_msk[wp][ch] = g;
            }
            __syncthreads();
            for (int d = wp; d < R; d += kGreedyWarps) {
                // ranks that fill inside this chunk (full ranks get no tokens)
                if (s_tot[tb][d] == 0 || s_load[lb][d] + s_tot[tb][d] < Tr) continue;
                const long long need = Tr - s_load[lb][d];  // tokens rank d still takes
                int c = s_cnt[lane][d];
                int incl = c;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += y;
                }
                const unsigned hit = __ballot_sync(0xffffffffu, incl >= need);
                const int w = __ffs(hit) - 1;  // the warp holding the filling token
                if (lane == w) {
                    // the nth (1-based) token of warp w that chose d fills it
                    const int nth = (int)(need - (incl - c));
                    unsigned m = s_msk[w][d];
                    for (int i = 1; i < nth; ++i) m &= m - 1u;
                    atomicMin(&s_pmin, w * 32 + __ffs(m) - 1);
                }
            }
            __syncthreads();
            const int pmin = s_pmin;
            const bool commit = ch >= 0 && tid <= pmin;
            if (commit) pred[t] = ch;
            const unsigned g2 =
                __match_any_sync(0xffffffffu, commit ? (unsigned)ch : (0x80000000u | lane));
            if (commit && (g2 & md::lanemask_lt()) == 0u)
                atomicAdd(reinterpret_cast<unsigned long long *>(&s_load[lb][ch]),
                          (unsigned long long)__popc(g2));
            for (int i = tid; i < 3 * MD_MAX_RANKS; i += kGreedyThreads) (&s_tot[0][0])[i] = 0;
            __syncthreads();
            for (int d0 = 0; d0 < R; d0 += 32) {
                const int d = d0 + lane;
                full |= (unsigned long long)__ballot_sync(0xffffffffu, d < R && s_load[lb][d] == Tr)
                        << d0;
            }
            refresh_first();
            __syncthreads();
            if (pmin >= kGreedyThreads - 1) break;
            start = pmin + 1;
        }
    }
}

// ------------------------------------------------------------ pair shuffle
// Each token's prediction row is the pair row C2[a][b] (a, b its top-1
// experts at layers l-1 and l) when that row's total reaches min_obs, else
// the single row C[b].  One warp per token computes from that row the
// preference list (R bytes) and an exact confidence key:
//     key = floor(num * 2^63 / den)   (0 for an empty row).
// For den < 2^31, two different fractions num/den <= 1 differ by at least
// 2^-62, i.e. by at least 2 after scaling, so the keys order the
// confidences exactly and equal confidences get equal keys.  Tokens are then
// sorted by (key desc, t asc) with a stable LSD radix sort (11-bit digits,
// only as many passes as the largest row total calls for: radix_plan), and
// the greedy walks each token's own preference list.
constexpr int kPairWarps = 8;

struct PairWs {
    unsigned char *tpref;      // [T*Rs] preference list of each token, Rs = R rounded up to 16
    unsigned long long *conf;  // [T]   confidence key of each token
    int32_t *seq_a, *seq_b;    // [T]   radix sort ping-pong
    int32_t *keys;             // [T]   bucket of each token in the final partition
    int32_t *tile_hist;        // [(n_tiles + 1) * max(2^11, R)]
    uint32_t *maxden;          // [1]   largest row total used by a token
    uint32_t *ticket;          // [1]   CTAs done in the current radix scan
};

size_t pair_layout(int64_t T, int R, PairWs *w, void *base)
{
    char *b = static_cast<char *>(base);
    size_t o = 0;
    auto take = [&](size_t bytes) {
        char *p = b ? b + o : nullptr;
        o += md::align_up(bytes, 256);
        return p;
    };
    const int64_t Tn = T > 0 ? T : 1;
    const int64_t n_tiles = (Tn + kTile - 1) / kTile;
    PairWs x;
    x.tpref = reinterpret_cast<unsigned char *>(take((size_t)Tn * pref_stride(R)));
    x.conf = reinterpret_cast<unsigned long long *>(take((size_t)Tn * 8));
    x.seq_a = reinterpret_cast<int32_t *>(take((size_t)Tn * 4));
    x.seq_b = reinterpret_cast<int32_t *>(take((size_t)Tn * 4));
    x.keys = reinterpret_cast<int32_t *>(take((size_t)Tn * 4));
    const int nbk = kRadixBuckets > R ? kRadixBuckets : R;
    x.tile_hist = reinterpret_cast<int32_t *>(take((size_t)(n_tiles + 1) * nbk * 4));
    x.maxden = reinterpret_cast<uint32_t *>(take(8));
    x.ticket = x.maxden ? x.maxden + 1 : nullptr;
    if (w) *w = x;
    return o;
}

// floor(num * 2^63 / den) for num <= den < 2^31, exactly, in two 64-bit
// long-division steps: num * 2^63 = (num * 2^32) * 2^31, and the remainder
// of the first step (< den) shifted by 31 still fits in 64 bits.
__device__ __forceinline__ unsigned long long conf_key(uint64_t num, uint64_t den)
{
    const uint64_t a = num << 32;
    const uint64_t q1 = a / den, r1 = a - q1 * den;
    const uint64_t q2 = (r1 << 31) / den;
    return (q1 << 31) + q2;
}

// One warp per token.  Lane j holds the row entries of experts j, j+32, ...
// (E <= 256: at most 8), so the row is read once; the per-rank sums are
// shared-memory atomics of those entries, and the preference order compares
// one 64-bit key per rank, (sum << 7) | (127 - rank): larger sum first, lower
// rank on ties.
constexpr int kPairPerLane = MD_MAX_PAIR_EXPERTS / 32;

__global__ void __launch_bounds__(kPairWarps * 32, 4)
    k_pair_rows(const int32_t *__restrict__ idx_p, const int32_t *__restrict__ idx_l, int k,
                const uint32_t *__restrict__ C, const uint32_t *__restrict__ C2,
                const int32_t *__restrict__ p_next, int64_t T, int E, int R, uint32_t min_obs,
                PairWs ws, int32_t *__restrict__ use_pair, int32_t *status)
{
    __shared__ unsigned long long s_sig[kPairWarps][MD_MAX_RANKS];
    const int lane = threadIdx.x & 31, wl = threadIdx.x >> 5;
    unsigned long long *sig = s_sig[wl];
    // next-layer rank of each of this lane's experts; an out-of-range rank is
    // reported and the expert left out of every rank's sum
    int rk[kPairPerLane];
#pragma unroll
    for (int j = 0; j < kPairPerLane; ++j) {
        const int e = lane + 32 * j;
        int d = -1;
        if (e < E) {
            d = __ldg(p_next + e);
            if (d < 0 || d >= R) {
                if (blockIdx.x == 0 && wl == 0) md::report(status, MD_ERR_DATA);
                d = -1;
            }
        }
        rk[j] = d;
    }
    const int64_t w0 = (int64_t)blockIdx.x * kPairWarps + wl;
    const int64_t nw = (int64_t)gridDim.x * kPairWarps;
    uint32_t maxden = 0;  // lane 0: the largest row total of this warp's tokens
    for (int64_t t = w0; t < T; t += nw) {
        int a = __ldg(idx_p + t * k), b = __ldg(idx_l + t * k);
        if (a < 0 || a >= E || b < 0 || b >= E) {
            md::report(status, MD_ERR_DATA);
            a = a < 0 || a >= E ? 0 : a;
            b = b < 0 || b >= E ? 0 : b;
        }
        const uint32_t *prow = C2 + ((int64_t)a * E + b) * E;
        uint32_t v[kPairPerLane];
        unsigned long long psum = 0;
#pragma unroll
        for (int j = 0; j < kPairPerLane; ++j) {
            v[j] = lane + 32 * j < E ? __ldg(prow + lane + 32 * j) : 0u;
            psum += v[j];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o);
        const bool use = psum >= min_obs;
        if (!use) {
            const uint32_t *row = C + (int64_t)b * E;
#pragma unroll
            for (int j = 0; j < kPairPerLane; ++j)
                v[j] = lane + 32 * j < E ? __ldg(row + lane + 32 * j) : 0u;
        }
        for (int d = lane; d < R; d += 32) sig[d] = 0ull;
        __syncwarp();
        // per-rank sums, total and arg-max (lowest expert on ties)
        unsigned long long tot = 0, best = 0;
#pragma unroll
        for (int j = 0; j < kPairPerLane; ++j) {
            const int e = lane + 32 * j;
            if (e >= E) continue;
            if (rk[j] >= 0 && v[j]) atomicAdd(&sig[rk[j]], (unsigned long long)v[j]);
            tot += v[j];
            const unsigned long long c = ((unsigned long long)v[j] << 32) | (0xffffffffu - (unsigned)e);
            best = c > best ? c : best;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            tot += __shfl_xor_sync(0xffffffffu, tot, o);
            const unsigned long long c = __shfl_xor_sync(0xffffffffu, best, o);
            best = c > best ? c : best;
        }
        const uint32_t bv = (uint32_t)(best >> 32);
        const int be = (int)(0xffffffffu - (uint32_t)best);
        __syncwarp();
        for (int d = lane; d < R; d += 32) {
            const unsigned long long sd = sig[d];
            sig[d] = ((sd < (1ull << 56) ? sd : (1ull << 56) - 1) << 7) | (unsigned)(127 - d);
        }
        __syncwarp();
        int first = __ldg(p_next + be);
        if (first < 0 || first >= R) first = 0;
        unsigned char *pl = ws.tpref + t * pref_stride(R);
        // position of rank d: 0 for `first`; else 1 + the ranks other than
        // `first` whose key is larger.  With R <= 16 the two half-warps each
        // count half of the ranks.
        if (R <= 16) {
            const int d = lane & 15, half = lane >> 4;
            int n = 0;
            if (d < R) {
                const unsigned long long kd = sig[d];
                const int lo = half * 8, hi = min(R, lo + 8);
                for (int d2 = lo; d2 < hi; ++d2) n += d2 != first && sig[d2] > kd;
            }
            n += __shfl_xor_sync(0xffffffffu, n, 16);
            if (half == 0 && d < R) pl[d == first ? 0 : 1 + n] = (unsigned char)d;
        } else {
            for (int d = lane; d < R; d += 32) {
                const unsigned long long kd = sig[d];
                int n = 0;
                for (int d2 = 0; d2 < R; ++d2) n += d2 != first && sig[d2] > kd;
                pl[d == first ? 0 : 1 + n] = (unsigned char)d;
            }
        }
        if (lane == 0) {
            unsigned long long key = 0ull;
            if (tot > 0) {
                if (tot >= (1ull << 31)) {
                    md::report(status, MD_ERR_UNSUPPORTED);
                } else {
                    key = conf_key(bv, tot);
                    maxden = (uint32_t)tot > maxden ? (uint32_t)tot : maxden;
                }
            }
            ws.conf[t] = key;
            if (use_pair) use_pair[t] = use ? 1 : 0;
        }
        __syncwarp();
    }
    if (lane == 0 && maxden) atomicMax(ws.maxden, maxden);
}

// digit of the sort key for one LSD pass: confidence descending
__device__ __forceinline__ int radix_digit(const unsigned long long *conf, int32_t tok, int shift, int r)
{
    return (int)((~(conf[tok] >> r) >> shift) & (kRadixBuckets - 1));
}

__global__ void __launch_bounds__(256)
    k_radix_hist(const int32_t *__restrict__ seq, const unsigned long long *__restrict__ conf,
                 int64_t T, int pass, const uint32_t *__restrict__ maxden,
                 int32_t *__restrict__ tile_hist)
{
    const RadixPlan pl = radix_plan(maxden);
    if (pass >= pl.passes) return;
    const int shift = pass * kRadixBits;
    __shared__ int h[kRadixBuckets];
    for (int b = threadIdx.x; b < kRadixBuckets; b += 256) h[b] = 0;
    __syncthreads();
    const int64_t t0 = (int64_t)blockIdx.x * kTile;
    for (int i = threadIdx.x; i < kTile; i += 256) {
        const int64_t pos = t0 + i;
        if (pos < T) atomicAdd(&h[radix_digit(conf, seq ? seq[pos] : (int32_t)pos, shift, pl.r)], 1);
    }
    __syncthreads();
    for (int b = threadIdx.x; b < kRadixBuckets; b += 256)
        tile_hist[(int64_t)blockIdx.x * kRadixBuckets + b] = h[b];
}

// Column scan of the radix histogram, spread over the GPU: CTA c takes
// digits [32c, 32c+32) (a lane each, so every tile row is read in 128-byte
// pieces) and its 8 warps split the tiles into 8 runs; a run's sum goes
// through shared memory to the runs after it.  tile_hist[tile][b] becomes
// the items of digit b in the tiles before `tile`; the last warp leaves the
// column total in row n_tiles.  The last CTA to finish (a ticket, no wait)
// turns that row into the exclusive scan over the digits and puts the ticket
// back to 0 for the next pass.
constexpr int kRsWarps = 8;

__global__ void __launch_bounds__(kRsWarps * 32)
    k_radix_scan(int32_t *__restrict__ tile_hist, int n_tiles, int pass,
                 const uint32_t *__restrict__ maxden, uint32_t *__restrict__ ticket)
{
    if (pass >= radix_plan(maxden).passes) return;
    __shared__ int s_seg[kRsWarps][32];
    __shared__ int s_warp[kRsWarps];
    __shared__ int s_last;
    const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
    const int b = blockIdx.x * 32 + lane;
    const int per = (n_tiles + kRsWarps - 1) / kRsWarps;
    const int lo = min(n_tiles, wp * per), hi = min(n_tiles, lo + per);
    int sum = 0;
    for (int i0 = lo; i0 < hi; i0 += 8) {
        int v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
            v[u] = i0 + u < hi ? tile_hist[(int64_t)(i0 + u) * kRadixBuckets + b] : 0;
#pragma unroll
        for (int u = 0; u < 8; ++u) sum += v[u];
    }
    s_seg[wp][lane] = sum;
    __syncthreads();
    int run = 0;
    for (int w = 0; w < wp; ++w) run += s_seg[w][lane];
    for (int i0 = lo; i0 < hi; i0 += 8) {
        int v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
            v[u] = i0 + u < hi ? tile_hist[(int64_t)(i0 + u) * kRadixBuckets + b] : 0;
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (i0 + u < hi) {
                tile_hist[(int64_t)(i0 + u) * kRadixBuckets + b] = run;
                run += v[u];
            }
    }
    int32_t *totals = tile_hist + (int64_t)n_tiles * kRadixBuckets;
    if (wp == kRsWarps - 1) totals[b] = run;
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(ticket, 1u) == gridDim.x - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    constexpr int kPer = kRadixBuckets / (kRsWarps * 32);
    int t[kPer];
    int own = 0;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
        t[j] = __ldcg(totals + tid * kPer + j);
        own += t[j];
    }
    int incl = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) s_warp[wp] = incl;
    __syncthreads();
    int acc = incl - own;
    for (int w = 0; w < wp; ++w) acc += s_warp[w];
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
        totals[tid * kPer + j] = acc;
        acc += t[j];
    }
    if (tid == 0) *ticket = 0u;
}

// One tile per CTA, items in sequence order, stable within each digit.  The
// tile's four warps take a quarter each: a warp ranks its items per digit
// (__match_any_sync, 8 rounds of 32), then every digit's start is laid out
// over the warps in order, and each item goes to its warp's start plus its
// rank.
constexpr int kScatWarps = 4;
constexpr int kScatItems = kTile / (kScatWarps * 32);

__global__ void __launch_bounds__(kScatWarps * 32)
    k_radix_scatter(const int32_t *__restrict__ seq, const unsigned long long *__restrict__ conf,
                    int64_t T, int pass, const uint32_t *__restrict__ maxden,
                    const int32_t *__restrict__ tile_hist, int32_t *__restrict__ seq_out)
{
    __shared__ int wcnt[kScatWarps][kRadixBuckets];
    const RadixPlan pl = radix_plan(maxden);
    if (pass >= pl.passes) return;  // identity: the reader takes the last pass's buffer
    const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
    const int shift = pass * kRadixBits;
    for (int i = tid; i < kScatWarps * kRadixBuckets; i += kScatWarps * 32) (&wcnt[0][0])[i] = 0;
    const int64_t t0 = (int64_t)blockIdx.x * kTile + wp * (kTile / kScatWarps);
    int tok[kScatItems], dg[kScatItems], rk[kScatItems];
#pragma unroll
    for (int c = 0; c < kScatItems; ++c) {
        const int64_t pos = t0 + c * 32 + lane;
        tok[c] = pos < T ? (seq ? seq[pos] : (int32_t)pos) : -1;
    }
#pragma unroll
    for (int c = 0; c < kScatItems; ++c)
        dg[c] = tok[c] >= 0 ? radix_digit(conf, tok[c], shift, pl.r) : -1;
    __syncthreads();
    int *cw = wcnt[wp];
#pragma unroll
    for (int c = 0; c < kScatItems; ++c) {
        const int key = dg[c];
        const bool in = key >= 0;
        const unsigned g = __match_any_sync(0xffffffffu, in ? (unsigned)key : (0x80000000u | lane));
        rk[c] = in ? cw[key] + __popc(g & md::lanemask_lt()) : 0;
        __syncwarp();
        if (in && (g >> lane) == 1u) cw[key] += __popc(g);
        __syncwarp();
    }
    __syncthreads();
    const int32_t *row = tile_hist + (int64_t)blockIdx.x * kRadixBuckets;
    const int32_t *base = tile_hist + (int64_t)gridDim.x * kRadixBuckets;
    for (int b = tid; b < kRadixBuckets; b += kScatWarps * 32) {
        int run = row[b] + base[b];
#pragma unroll
        for (int w = 0; w < kScatWarps; ++w) {
            const int c = wcnt[w][b];
            wcnt[w][b] = run;
            run += c;
        }
    }
    __syncthreads();
#pragma unroll
    for (int c = 0; c < kScatItems; ++c)
        if (dg[c] >= 0) seq_out[cw[dg[c]] + rk[c]] = tok[c];
}

// ------------------------------------------------------ rounds assignment
// A parallel alternative to the sequential visit.  In each round every
// unassigned token proposes to the first rank of its preference list that
// was not full when the round began, and each rank accepts its
// highest-priority proposers up to its remaining capacity.  One cooperative
// launch: CTA c owns positions [c*1024, (c+1)*1024) of the priority order.
// Phase 1 counts the tile's proposals per rank; after a grid barrier, phase
// 2 places each proposer among the proposers of its rank (earlier tiles
// first, then tile order: each warp ranks its 128 positions with
// __match_any_sync, then a prefix over the warps) and accepts it if that
// place is inside the remaining capacity; after a second barrier the
// next round starts.  At most R + 1 rounds.  The grid barrier waits are
// bounded (MD_ERR_TIMEOUT, and every CTA then stops).
constexpr int kRoundThreads = 256;
constexpr long long kBarrierPolls = 1ll << 22;

struct RoundWs {
    int32_t *rem;        // [R] capacity left at the start of the round
    int32_t *cnt;        // [n_tiles * R] proposals per tile and rank
    unsigned *bar;       // [0] arrivals, [1] generation
    int32_t *abort;      // [0] set when a barrier wait ran out
    int32_t *rounds;     // [0] rounds that accepted a token
};

size_t round_layout(int64_t T, int R, RoundWs *w, void *base)
{
    char *b = static_cast<char *>(base);
    size_t o = 0;
    auto take = [&](size_t bytes) {
        char *q = b ? b + o : nullptr;
        o += md::align_up(bytes, 256);
        return q;
    };
    const int64_t n_tiles = T > 0 ? (T + kTile - 1) / kTile : 1;
    RoundWs x;
    x.bar = reinterpret_cast<unsigned *>(take(4 * sizeof(unsigned)));
    x.abort = reinterpret_cast<int32_t *>(take(sizeof(int32_t)));
    x.rounds = reinterpret_cast<int32_t *>(take(sizeof(int32_t)));
    x.rem = reinterpret_cast<int32_t *>(take((size_t)R * 4));
    x.cnt = reinterpret_cast<int32_t *>(take((size_t)n_tiles * R * 4));
    if (w) *w = x;
    return o;
}

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned *p)
{
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ unsigned atom_add_acq_rel_u32(unsigned *p, unsigned v)
{
    unsigned old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

__device__ __forceinline__ void atom_add_release_u32(unsigned *p, unsigned v)
{
    unsigned old;
    asm volatile("atom.release.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void st_relaxed_u32(unsigned *p, unsigned v)
{
    asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// All CTAs of the (cooperative, hence co-resident) grid meet here; false if
// a wait ran out somewhere.  The block barrier before thread 0's release
// (and after its acquire) carries every thread's global writes across.
__device__ bool grid_barrier(RoundWs rw, unsigned n_ctas, int32_t *status)
{
    __shared__ int s_ok;
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned gen = ld_acquire_u32(rw.bar + 1);
        if (atom_add_acq_rel_u32(rw.bar, 1u) + 1u == n_ctas) {
            st_relaxed_u32(rw.bar, 0u);          // ordered before the release below
            atom_add_release_u32(rw.bar + 1, 1u);
        } else {
            long long n = 0;
            while (ld_acquire_u32(rw.bar + 1) == gen) {
                if (++n > kBarrierPolls || *(volatile int32_t *)rw.abort) {
                    md::report(status, MD_ERR_TIMEOUT);
                    atomicExch(rw.abort, 1);
                    break;
                }
                if ((n & 63) == 0) __nanosleep(32);
            }
        }
        s_ok = *(volatile int32_t *)rw.abort == 0;
    }
    __syncthreads();
    return s_ok != 0;
}

__global__ void __launch_bounds__(kRoundThreads)
    k_shuf_rounds(const int32_t *__restrict__ order, const int32_t *__restrict__ idx_l, int k,
                  ShufWs ws, RoundWs rw, int64_t T, int E, int R, int64_t Tr,
                  int32_t *__restrict__ pred, int32_t *status)
{
    extern __shared__ unsigned char s_pref[];  // [E*R] preference lists, staged once
    __shared__ int s_tok[kTile];              // token at each position of the tile (-1: none)
    __shared__ short s_key[kTile];            // its top-1 expert, or -1 for an empty row
    __shared__ signed char s_prop[kTile];     // this round's proposal (-1: none)
    __shared__ unsigned char s_done[kTile];   // placed in an earlier round
    __shared__ short s_rank[kTile];           // place among its warp's proposers of its rank
    __shared__ int s_wcnt[kRoundThreads / 32][MD_MAX_RANKS];  // proposals per warp and rank
    __shared__ int s_cnt[MD_MAX_RANKS], s_rem[MD_MAX_RANKS], s_base[MD_MAX_RANKS], s_tot[MD_MAX_RANKS];
    __shared__ unsigned long long s_full;
    __shared__ int s_any;
    const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
    const int tile = blockIdx.x;
    const unsigned n_ctas = gridDim.x;
    const int64_t p0 = (int64_t)tile * kTile;

    for (int i = tid; i < E * R; i += kRoundThreads) s_pref[i] = (unsigned char)ws.pref[i];
    for (int i = tid; i < kTile; i += kRoundThreads) {
        const int64_t pos = p0 + i;
        int t = -1, key = -1;
        s_done[i] = 0;
        if (pos < T) {
            t = order[pos];
            int e1 = idx_l[(int64_t)t * k];
            if (e1 < 0 || e1 >= E) {
                md::report(status, MD_ERR_DATA);
                e1 = 0;
            }
            key = ws.den[e1] == 0ull ? -1 : e1;
            pred[t] = -1;
        }
        s_tok[i] = t;
        s_key[i] = (short)key;
    }
    if (tile == 0) {
        for (int d = tid; d < R; d += kRoundThreads) rw.rem[d] = (int)Tr;
        if (tid == 0) *rw.rounds = 0;
    }
    if (!grid_barrier(rw, n_ctas, status)) return;

    for (int round = 0; round <= R; ++round) {
        // ---- phase 1: proposals
        for (int d = tid; d < R; d += kRoundThreads) {
            s_rem[d] = rw.rem[d];
            s_cnt[d] = 0;
        }
        __syncthreads();
        if (tid == 0) {
            unsigned long long f = 0ull;
            for (int d = 0; d < R; ++d)
                if (s_rem[d] <= 0) f |= 1ull << d;
            s_full = f;
        }
        __syncthreads();
        const unsigned long long full = s_full;
        for (int i = tid; i < kTile; i += kRoundThreads) {
            const int t = s_tok[i];
            int d = -1;
            if (t >= 0 && !s_done[i]) {
                const int key = s_key[i];
                if (key < 0) {
                    const int src = (int)(t / Tr);
                    if (!((full >> src) & 1ull)) d = src;
                    for (int q = 0; d < 0 && q < R; ++q)
                        if (!((full >> q) & 1ull)) d = q;
                } else {
                    const unsigned char *pl = s_pref + (size_t)key * R;
                    for (int n = 0; d < 0 && n < R; ++n)
                        if (!((full >> pl[n]) & 1ull)) d = pl[n];
                }
                if (d >= 0) atomicAdd(&s_cnt[d], 1);
            }
            s_prop[i] = (signed char)d;
        }
        __syncthreads();
        for (int d = tid; d < R; d += kRoundThreads) rw.cnt[(int64_t)tile * R + d] = s_cnt[d];
        if (!grid_barrier(rw, n_ctas, status)) return;

        // ---- phase 2: places among each rank's proposers, acceptance.  The
        // (tile, rank) counts are summed by all threads at once: the earlier
        // tiles' counts give this tile's base, all tiles' the rank's total.
        for (int d = tid; d < R; d += kRoundThreads) {
            s_base[d] = 0;
            s_tot[d] = 0;
            s_cnt[d] = 0;
        }
        if (tid == 0) s_any = 0;
        __syncthreads();
        for (int64_t c = tid; c < (int64_t)n_ctas * R; c += kRoundThreads) {
            const int v = rw.cnt[c];
            if (!v) continue;
            const int j = (int)(c / R), d = (int)(c - (int64_t)j * R);
            atomicAdd(&s_tot[d], v);
            if (j < tile) atomicAdd(&s_base[d], v);
            s_any = 1;
        }
        __syncthreads();
        if (!s_any) break;  // every token placed (the same on every CTA)
        // warp w ranks positions [w*128, w*128+128) in order; then a prefix
        // over the warps per rank gives each proposer its place in the tile
        constexpr int kPerWarp = kTile / (kRoundThreads / 32);
        for (int d = lane; d < R; d += 32) s_wcnt[wp][d] = 0;
        __syncwarp();
        for (int c0 = wp * kPerWarp; c0 < (wp + 1) * kPerWarp; c0 += 32) {
            const int i = c0 + lane;
            const int d = s_prop[i];
            const unsigned g = __match_any_sync(0xffffffffu, d >= 0 ? (unsigned)d : (0x80000000u | lane));
            if (d >= 0) s_rank[i] = (short)(s_wcnt[wp][d] + __popc(g & md::lanemask_lt()));
            __syncwarp();
            if (d >= 0 && (g & md::lanemask_lt()) == 0u) s_wcnt[wp][d] += __popc(g);
            __syncwarp();
        }
        __syncthreads();
        for (int d = tid; d < R; d += kRoundThreads) {
            int run = 0;
            for (int w2 = 0; w2 < kRoundThreads / 32; ++w2) {
                const int c = s_wcnt[w2][d];
                s_wcnt[w2][d] = run;
                run += c;
            }
        }
        __syncthreads();
        for (int i = tid; i < kTile; i += kRoundThreads) {
            const int d = s_prop[i];
            if (d >= 0 && s_base[d] + s_wcnt[i / kPerWarp][d] + s_rank[i] < s_rem[d]) {
                pred[s_tok[i]] = d;
                s_done[i] = 1;
            }
        }
        if (tile == 0) {
            for (int d = tid; d < R; d += kRoundThreads) {
                const int left = s_rem[d] - s_tot[d];
                rw.rem[d] = left > 0 ? left : 0;
            }
            if (tid == 0) *rw.rounds += 1;
        }
        if (!grid_barrier(rw, n_ctas, status)) return;
    }
}

}  // namespace

extern "C" size_t md_token_shuffle_workspace_size(int64_t T, int E, int R)
{
    if (T < 0 || E < 1 || R < 1) return 0;
    return shuf_layout(T, E, R, nullptr, nullptr);
}

namespace {

// Raises the greedy's shared-memory limit once per device, to the largest size
// either form asks for (single: E first ranks and E*R preferences; pair: two
// chunks of per-token lists); false if CUDA refuses.
bool greedy_smem_ready()
{
    static std::atomic<uint64_t> done{0};
    static std::atomic<int> ok_dev[64];
    md::once_per_device(done, [] {
        int dev = 0;
        cudaGetDevice(&dev);
        const int single = MD_MAX_EXPERTS * (int)sizeof(int) + MD_MAX_EXPERTS * MD_MAX_RANKS;
        const int pair = 2 * kGreedyThreads * pref_stride(MD_MAX_RANKS);
        const bool ok =
            cudaFuncSetAttribute(k_shuf_greedy<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, single) ==
                cudaSuccess &&
            cudaFuncSetAttribute(k_shuf_greedy<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, pair) ==
                cudaSuccess;
        if (!ok) cudaGetLastError();
        ok_dev[dev & 63].store(ok ? 1 : 0);
    });
    int dev = 0;
    cudaGetDevice(&dev);
    return ok_dev[dev & 63].load() != 0;
}

}  // namespace

extern "C" int md_token_shuffle(const int32_t *idx_l, int k, const uint32_t *C,
                                const int32_t *expert_to_rank_next, int64_t T, int E, int R,
                                int32_t *pred_rank, int32_t *perm, int32_t *inv, void *workspace,
                                size_t workspace_bytes, int32_t *dev_status, void *stream)
{
    if (T < 0 || E < 1 || R < 1 || k < 1 || k > MD_MAX_TOPK) return MD_ERR_ARG;
    if (E > MD_MAX_EXPERTS || R > MD_MAX_RANKS || T >= ((int64_t)1 << 31)) return MD_ERR_UNSUPPORTED;
    if (T % R != 0) return MD_ERR_ARG;
    if (!C || !expert_to_rank_next) return MD_ERR_ARG;
    if (T > 0 && (!idx_l || !pred_rank || !perm || !inv)) return MD_ERR_ARG;
    const size_t need = shuf_layout(T, E, R, nullptr, nullptr);
    if (!workspace || workspace_bytes < need) return MD_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MD_ERR_ARG;
    cudaStream_t s = md::as_stream(stream);
    int rc = md::clear_status(dev_status, s);
    if (rc != MD_OK || T == 0) return rc;
    ShufWs ws;
    shuf_layout(T, E, R, &ws, workspace);
    const int n_tiles = (int)((T + kTile - 1) / kTile);
    const int64_t Tr = T / R;

    k_shuf_prefs<<<E, 256, 0, s>>>(C, expert_to_rank_next, E, R, ws, dev_status);
    k_shuf_class<<<(E + 255) / 256, 256, 0, s>>>(E, ws);
    // visit order: by confidence class, then t
    const int nbk0 = E + 1;
    k_bucket_hist<<<n_tiles, 256, nbk0 * sizeof(int), s>>>(0, T, idx_l, k, ws.cls, E, nullptr, nbk0,
                                                          ws.keys, ws.tile_hist);
    k_bucket_scan<<<1, kScanThreads, nbk0 * sizeof(int), s>>>(ws.tile_hist, n_tiles, nbk0);
    k_bucket_scatter<<<n_tiles, 32, nbk0 * sizeof(int), s>>>(0, T, nbk0, ws.keys, ws.tile_hist,
                                                            ws.order, nullptr, nullptr);
    const size_t gsm = (size_t)E * sizeof(int) + (size_t)E * R;
    if (!greedy_smem_ready()) return MD_ERR_CUDA;
    k_shuf_greedy<false><<<1, kGreedyThreads, gsm, s>>>(ws.order, idx_l, k, ws, nullptr, nullptr, T,
                                                        E, R, Tr, pred_rank, dev_status);
    // new positions: stable partition by assigned rank
    k_bucket_hist<<<n_tiles, 256, R * sizeof(int), s>>>(1, T, nullptr, k, nullptr, E, pred_rank, R,
                                                       ws.keys, ws.tile_hist);
    k_bucket_scan<<<1, kScanThreads, R * sizeof(int), s>>>(ws.tile_hist, n_tiles, R);
    k_bucket_scatter<<<n_tiles, 32, R * sizeof(int), s>>>(1, T, R, ws.keys, ws.tile_hist, nullptr,
                                                         perm, inv);
    md::count_launches(9);
    return md::launch_status();
}

extern "C" size_t md_token_shuffle_pair_workspace_size(int64_t T, int E, int R)
{
    if (T < 0 || E < 1 || R < 1) return 0;
    return pair_layout(T, R, nullptr, nullptr);
}

extern "C" int md_token_shuffle_pair(const int32_t *idx_prev, const int32_t *idx_l, int k,
                                     const uint32_t *C, const uint32_t *C2,
                                     const int32_t *expert_to_rank_next, int64_t T, int E, int R,
                                     uint32_t min_obs, int32_t *pred_rank, int32_t *perm,
                                     int32_t *inv, int32_t *use_pair, void *workspace,
                                     size_t workspace_bytes, int32_t *dev_status, void *stream)
{
    if (T < 0 || E < 1 || R < 1 || k < 1 || k > MD_MAX_TOPK || min_obs < 1) return MD_ERR_ARG;
    if (E > MD_MAX_PAIR_EXPERTS || R > MD_MAX_RANKS || T >= ((int64_t)1 << 31))
        return MD_ERR_UNSUPPORTED;
    if (T % R != 0) return MD_ERR_ARG;
    if (!C || !C2 || !expert_to_rank_next) return MD_ERR_ARG;
    if (T > 0 && (!idx_prev || !idx_l || !pred_rank || !perm || !inv)) return MD_ERR_ARG;
    const size_t need = pair_layout(T, R, nullptr, nullptr);
    if (!workspace || workspace_bytes < need) return MD_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MD_ERR_ARG;
    cudaStream_t s = md::as_stream(stream);
    int rc = md::clear_status(dev_status, s);
    if (rc != MD_OK || T == 0) return rc;
    PairWs pw;
    pair_layout(T, R, &pw, workspace);
    const int n_tiles = (int)((T + kTile - 1) / kTile);
    const int64_t Tr = T / R;
    md::count_memsets(1);
    if (cudaMemsetAsync(pw.maxden, 0, 2 * sizeof(uint32_t), s) != cudaSuccess) return MD_ERR_CUDA;

    int64_t blocks = (T + kPairWarps - 1) / kPairWarps;
    const int64_t cap = (int64_t)md::sm_count() * 4;  // one wave: 4 CTAs per SM
    if (blocks > cap) blocks = cap;
    k_pair_rows<<<(unsigned)blocks, kPairWarps * 32, 0, s>>>(idx_prev, idx_l, k, C, C2,
                                                             expert_to_rank_next, T, E, R, min_obs,
                                                             pw, use_pair, dev_status);
    // visit order: stable LSD radix sort by (confidence key desc), from t
    // ascending; the passes above the key's significant digits do nothing
    const int32_t *in = nullptr;
    int32_t *out = pw.seq_a;
    for (int pass = 0; pass < kRadixPasses; ++pass) {
        k_radix_hist<<<n_tiles, 256, 0, s>>>(in, pw.conf, T, pass, pw.maxden, pw.tile_hist);
        k_radix_scan<<<kRadixBuckets / 32, kRsWarps * 32, 0, s>>>(pw.tile_hist, n_tiles, pass,
                                                                  pw.maxden, pw.ticket);
        k_radix_scatter<<<n_tiles, kScatWarps * 32, 0, s>>>(in, pw.conf, T, pass, pw.maxden,
                                                            pw.tile_hist, out);
        in = out;
        out = out == pw.seq_a ? pw.seq_b : pw.seq_a;
    }
    ShufWs none{};
    const size_t lsm = (size_t)2 * kGreedyThreads * pref_stride(R);
    if (!greedy_smem_ready()) return MD_ERR_CUDA;
    k_shuf_greedy<true><<<1, kGreedyThreads, lsm, s>>>(pw.seq_a, nullptr, k, none, pw.tpref, pw.conf,
                                                       T, E, R, Tr, pred_rank, dev_status, pw.seq_b,
                                                       pw.maxden);
    // new positions: stable partition by assigned rank
    k_bucket_hist<<<n_tiles, 256, R * sizeof(int), s>>>(1, T, nullptr, k, nullptr, E, pred_rank, R,
                                                       pw.keys, pw.tile_hist);
    k_bucket_scan<<<1, kScanThreads, R * sizeof(int), s>>>(pw.tile_hist, n_tiles, R);
    k_bucket_scatter<<<n_tiles, 32, R * sizeof(int), s>>>(1, T, R, pw.keys, pw.tile_hist, nullptr,
                                                         perm, inv);
    md::count_launches(1 + 3 * kRadixPasses + 1 + 3);
    return md::launch_status();
}

namespace {

// CTAs of k_shuf_rounds resident per SM with rsm bytes of dynamic shared
// memory; -1 if CUDA refuses.  The shared-memory limit is raised once per
// device to the largest size (E*R <= 64 KiB); the occupancy query itself is
// host arithmetic and depends on rsm, so it runs per call.
int rounds_per_sm(size_t rsm)
{
    static std::atomic<uint64_t> done{0};
    static std::atomic<int> attr_ok[64];
    md::once_per_device(done, [] {
        int dev = 0;
        cudaGetDevice(&dev);
        const bool ok = cudaFuncSetAttribute(k_shuf_rounds, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             MD_MAX_EXPERTS * MD_MAX_RANKS) == cudaSuccess;
        if (!ok) cudaGetLastError();
        attr_ok[dev & 63].store(ok ? 1 : 0);
    });
    int dev = 0;
    cudaGetDevice(&dev);
    if (!attr_ok[dev & 63].load()) return -1;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_shuf_rounds, kRoundThreads, rsm) !=
        cudaSuccess) {
        cudaGetLastError();
        return -1;
    }
    return per_sm;
}

}  // namespace

extern "C" size_t md_token_shuffle_rounds_workspace_size(int64_t T, int E, int R)
{
    if (T < 0 || E < 1 || R < 1) return 0;
    return shuf_layout(T, E, R, nullptr, nullptr) + round_layout(T, R, nullptr, nullptr);
}

extern "C" int md_token_shuffle_rounds(const int32_t *idx_l, int k, const uint32_t *C,
                                       const int32_t *expert_to_rank_next, int64_t T, int E, int R,
                                       int32_t *pred_rank, int32_t *perm, int32_t *inv,
                                       int32_t *rounds, void *workspace, size_t workspace_bytes,
                                       int32_t *dev_status, void *stream)
{
    if (T < 0 || E < 1 || R < 1 || k < 1 || k > MD_MAX_TOPK) return MD_ERR_ARG;
    if (E > MD_MAX_EXPERTS || R > MD_MAX_RANKS || T >= ((int64_t)1 << 31)) return MD_ERR_UNSUPPORTED;
    if (E > 32767) return MD_ERR_UNSUPPORTED;
    if (T % R != 0) return MD_ERR_ARG;
    if (!C || !expert_to_rank_next) return MD_ERR_ARG;
    if (T > 0 && (!idx_l || !pred_rank || !perm || !inv)) return MD_ERR_ARG;
    const size_t need_s = shuf_layout(T, E, R, nullptr, nullptr);
    const size_t need = need_s + round_layout(T, R, nullptr, nullptr);
    if (!workspace || workspace_bytes < need) return MD_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MD_ERR_ARG;
    const int n_tiles = (int)((T + kTile - 1) / kTile);
    // every CTA must be resident at once (cooperative launch)
    const size_t rsm = (size_t)E * R;
    const int per_sm = rounds_per_sm(rsm);
    if (per_sm < 0) return MD_ERR_CUDA;
    if (T > 0 && (int64_t)per_sm * md::sm_count() < n_tiles) return MD_ERR_UNSUPPORTED;
    cudaStream_t s = md::as_stream(stream);
    int rc = md::clear_status(dev_status, s);
    if (rc != MD_OK) return rc;
    ShufWs ws;
    shuf_layout(T, E, R, &ws, workspace);
    RoundWs rw;
    round_layout(T, R, &rw, static_cast<char *>(workspace) + need_s);
    md::count_memsets(1);
    if (cudaMemsetAsync(rw.bar, 0, 256 * 3, s) != cudaSuccess) return MD_ERR_CUDA;  // bar, abort, rounds
    if (T == 0) {
        if (rounds) {
            md::count_memsets(1);
            if (cudaMemsetAsync(rounds, 0, sizeof(int32_t), s) != cudaSuccess) return MD_ERR_CUDA;
        }
        return MD_OK;
    }
    const int64_t Tr = T / R;
    k_shuf_prefs<<<E, 256, 0, s>>>(C, expert_to_rank_next, E, R, ws, dev_status);
    k_shuf_class<<<(E + 255) / 256, 256, 0, s>>>(E, ws);
    const int nbk0 = E + 1;
    k_bucket_hist<<<n_tiles, 256, nbk0 * sizeof(int), s>>>(0, T, idx_l, k, ws.cls, E, nullptr, nbk0,
                                                          ws.keys, ws.tile_hist);
    k_bucket_scan<<<1, kScanThreads, nbk0 * sizeof(int), s>>>(ws.tile_hist, n_tiles, nbk0);
    k_bucket_scatter<<<n_tiles, 32, nbk0 * sizeof(int), s>>>(0, T, nbk0, ws.keys, ws.tile_hist,
                                                            ws.order, nullptr, nullptr);
    const int32_t *order = ws.order;
    int kk = k;
    int64_t TT = T, TTr = Tr;
    int EE = E, RR = R;
    void *args[] = {(void *)&order, (void *)&idx_l, (void *)&kk, (void *)&ws, (void *)&rw,
                    (void *)&TT, (void *)&EE, (void *)&RR, (void *)&TTr, (void *)&pred_rank,
                    (void *)&dev_status};
    if (cudaLaunchCooperativeKernel((const void *)k_shuf_rounds, dim3(n_tiles), dim3(kRoundThreads),
                                    args, rsm, s) != cudaSuccess) {
        cudaGetLastError();  // a refused launch must not be blamed on a later call
        return MD_ERR_CUDA;
    }
    k_bucket_hist<<<n_tiles, 256, R * sizeof(int), s>>>(1, T, nullptr, k, nullptr, E, pred_rank, R,
                                                       ws.keys, ws.tile_hist);
    k_bucket_scan<<<1, kScanThreads, R * sizeof(int), s>>>(ws.tile_hist, n_tiles, R);
    k_bucket_scatter<<<n_tiles, 32, R * sizeof(int), s>>>(1, T, R, ws.keys, ws.tile_hist, nullptr,
                                                         perm, inv);
    md::count_launches(9);
    if (rounds) {
        md::count_memsets(1);
        if (cudaMemcpyAsync(rounds, rw.rounds, sizeof(int32_t), cudaMemcpyDeviceToDevice, s) !=
            cudaSuccess)
            return MD_ERR_CUDA;
    }
    return md::launch_status();
}
