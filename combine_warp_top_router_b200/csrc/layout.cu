// layout.cu -- dispatch layout: rows, positions and the send matrix
// (md_dispatch_layout).
//
// "DODOCO: MoE AlltoAll Traffic Matrices on Real Text", send_matrices.csv and
// Reading the counts: send_counts[s][d] counts what source rank s sends to
// rank d (token-expert assignments for the conventional dispatcher, so each
// row sums to T/R x k); combine returns the transposed volumes.
// "Expert Coupling in MoE Pretraining", Method 1: the deduplicating
// dispatcher sends one row per distinct (token, destination rank) pair.
//
// Rows are stable-sorted buckets: conventional rows by (p[e], e, t), dedup
// rows by (d, t).  Two kernels, one thread per token, the token's k experts in
// registers (k is a template parameter for the common values):
//   k_layout_hist  bucket totals (assignments per expert, the send matrix)
//                  in shared-memory histograms, flushed to the workspace.
//   k_layout_rank  one tile of tokens per CTA, tiles in atomic-ticket order.
//                  Every CTA turns the totals into bucket bases.  Inside the
//                  tile, each warp marks which of its lanes hit each bucket
//                  (a 32-bit set per bucket, built with shared atomicOr), so a
//                  pair's rank among the warp's earlier tokens is a popcount.
//                  The CTA publishes its bucket counts and gets the counts of
//                  all earlier tiles by a single-pass decoupled lookback with
//                  bounded waits; rows are staged in shared memory in bucket
//                  order and written out in runs.
#include "common.cuh"

namespace {

constexpr int kHistThreads = 256;  // one token per thread
constexpr int kRankThreads = 512;  // one token per thread
constexpr int kRankWarps = kRankThreads / 32;
constexpr int kStageRows = 4096;   // output rows a rank tile can stage
constexpr int kLookBatch = 8;      // buckets a warp looks back on at once
constexpr unsigned long long kFlagA = 1ull << 62;  // tile aggregate published
constexpr unsigned long long kFlagP = 2ull << 62;  // tile inclusive prefix published
constexpr unsigned long long kValMask = (1ull << 62) - 1;
constexpr long long kPollLimit = 1ll << 22;

struct Ws {
    long long poll_limit;         // bound of every lookback wait
    int skip_tile;                // test hook: this tile publishes nothing (-1: none)
    unsigned int *ctrl;           // [0] rank tile ticket
    int *hist_e;                  // [E]   assignments per expert
    int *send;                    // [R*R] rows per (source, destination)
    unsigned long long *tiles;    // [NB][n_tiles] lookback words, bucket-major
};

// tokens per rank tile: one per thread, fewer when k is large so that the
// tile's rows fit the staging area
int tile_tokens(int k)
{
    if (k <= kStageRows / kRankThreads) return kRankThreads;
    int t = kStageRows / k, p = 1;
    while (p * 2 <= t) p *= 2;
    return p;
}

struct Plan {
    size_t off_hist, off_send, off_tiles, total;
    int tile_tok, n_tiles, nb;
};

Plan plan(int64_t T, int E, int k, int R, int mode)
{
    Plan p;
    p.tile_tok = tile_tokens(k);
    p.n_tiles = (int)((T + p.tile_tok - 1) / p.tile_tok);
    if (p.n_tiles < 1) p.n_tiles = 1;  // tile 0 also writes the count outputs
    p.nb = E + (mode == MD_DEDUP ? R : 0);
    size_t o = 256;
    p.off_hist = o;
    o += md::align_up((size_t)E * 4, 256);
    p.off_send = o;
    o += md::align_up((size_t)R * R * 4, 256);
    p.off_tiles = o;
    o += md::align_up((size_t)p.n_tiles * p.nb * 8, 256);
    p.total = o;  // all of it must start at zero
    return p;
}

Ws carve(void *ws, const Plan &p)
{
    char *b = static_cast<char *>(ws);
    Ws w;
    w.poll_limit = md::hook_poll_limit(kPollLimit);
    w.skip_tile = md::hook_layout_skip_tile();
    w.ctrl = reinterpret_cast<unsigned int *>(b);
    w.hist_e = reinterpret_cast<int *>(b + p.off_hist);
    w.send = reinterpret_cast<int *>(b + p.off_send);
    w.tiles = reinterpret_cast<unsigned long long *>(b + p.off_tiles);
    return w;
}

__device__ __forceinline__ int warp_incl_scan(int v, int lane)
{
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += y;
    }
    return v;
}

// Clear the workspace (counters, totals, lookback words) and the status word.
__global__ void __launch_bounds__(256) k_layout_zero(uint4 *__restrict__ ws, size_t n16,
                                                     int32_t *status)
{
    for (size_t i = (size_t)blockIdx.x * 256 + threadIdx.x; i < n16; i += (size_t)gridDim.x * 256)
        ws[i] = make_uint4(0u, 0u, 0u, 0u);
    if (status && blockIdx.x == 0 && threadIdx.x == 0) *status = MD_OK;
    asm volatile("griddepcontrol.launch_dependents;");
}

// --------------------------------------------------------------- totals
// KC > 0: the token's k experts live in registers (k known at compile time);
// KC = 0: they are staged in shared memory with an odd row stride.
template <int KC>
__global__ void __launch_bounds__(kHistThreads, 2)
    k_layout_hist(const int32_t *__restrict__ idx, int64_t T, int E, int k, int R,
                  const int32_t *__restrict__ p_g, int mode, Ws ws, int32_t *status)
{
    extern __shared__ int smem[];
    int *s_p = smem;             // [E]
    int *s_hist = s_p + E;       // [E]
    int *s_send = s_hist + E;    // [R*R]
    int *s_idx = s_send + R * R; // [kHistThreads * (k | 1)]  (KC == 0 only)

    const int K = KC ? KC : k;
    const int tid = threadIdx.x;
    for (int e = tid; e < E; e += kHistThreads) {
        s_p[e] = p_g[e];
        s_hist[e] = 0;
    }
    for (int i = tid; i < R * R; i += kHistThreads) s_send[i] = 0;
    const int64_t Tr = T / R;
    const int64_t t0 = (int64_t)blockIdx.x * kHistThreads;
    const bool have = t0 + tid < T;
    const int64_t t = have ? t0 + tid : t0;
    int reg[KC ? KC : 1];
    const int ks = K | 1;
    if (KC) {
#pragma unroll
        for (int j = 0; j < (KC ? KC : 1); ++j) reg[j] = have ? __ldg(idx + t * K + j) : -1;
    } else {
        for (int j = 0; j < K; ++j) s_idx[tid * ks + j] = have ? __ldg(idx + t * K + j) : -1;
    }
    // the loads above overlap the clearing kernel; status and workspace are
    // touched only after it has completed
    asm volatile("griddepcontrol.wait;" ::: "memory");
    __syncthreads();
    auto ex = [&](int j) -> int { return KC ? reg[j] : s_idx[tid * ks + j]; };

    // rank of every slot, looked up once (-1: invalid expert or placement)
    int dr[KC ? KC : 1];
    if (KC) {
#pragma unroll
        for (int j = 0; j < (KC ? KC : 1); ++j) {
            const int e = ex(j);
            int d = (e >= 0 && e < E) ? s_p[e] : -1;
            dr[j] = (d >= 0 && d < R) ? d : -1;
        }
    }
    auto rk = [&](int j) -> int {
        if (KC) return dr[j];
        const int e = ex(j);
        const int d = (e >= 0 && e < E) ? s_p[e] : -1;
        return (d >= 0 && d < R) ? d : -1;
    };

    // shared-memory histograms
    const int src = (int)(t / Tr);
#pragma unroll
    for (int j = 0; j < (KC ? KC : MD_MAX_TOPK); ++j) {
        if (!KC && j >= K) break;
        int e = ex(j);
        int d = rk(j);
        if (have && d < 0) md::report(status, MD_ERR_DATA);
        if (d < 0) e = -1;
        bool rep = true;
#pragma unroll
        for (int j2 = 0; j2 < (KC ? KC : MD_MAX_TOPK); ++j2) {
            if (j2 >= j) break;
            if (e >= 0 && ex(j2) == e) md::report(status, MD_ERR_DATA);  // expert twice in one token
            if (rk(j2) == d) rep = false;
        }
        if (e >= 0) {
            atomicAdd(&s_hist[e], 1);
            if (mode == MD_CONV || rep) atomicAdd(&s_send[src * R + d], 1);
        }
    }
    asm volatile("griddepcontrol.launch_dependents;");
    __syncthreads();
    for (int e = tid; e < E; e += kHistThreads)
        if (s_hist[e]) atomicAdd(&ws.hist_e[e], s_hist[e]);
    for (int i = tid; i < R * R; i += kHistThreads)
        if (s_send[i]) atomicAdd(&ws.send[i], s_send[i]);
}

// --------------------------------------------------------------- ranks
// A token's k outputs are contiguous: vector stores where k allows.
template <int KC>
__device__ __forceinline__ void store_row(int32_t *dst, const int (&v)[KC ? KC : MD_MAX_TOPK], int K)
{
    if (KC == 8 || KC == 4) {
#pragma unroll
        for (int q = 0; q < (KC ? KC : 4) / 4; ++q)
            reinterpret_cast<int4 *>(dst)[q] = make_int4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    } else if (KC == 6 || KC == 2) {
#pragma unroll
        for (int q = 0; q < (KC ? KC : 2) / 2; ++q)
            reinterpret_cast<int2 *>(dst)[q] = make_int2(v[2 * q], v[2 * q + 1]);
    } else {
#pragma unroll
        for (int j = 0; j < (KC ? KC : MD_MAX_TOPK); ++j) {
            if (!KC && j >= K) break;
            dst[j] = v[j];
        }
    }
}

template <int KC>
__global__ void __launch_bounds__(kRankThreads, 1)
    k_layout_rank(const int32_t *__restrict__ idx, int64_t T, int E, int k, int R,
                  const int32_t *__restrict__ p_g, int mode, int tile_tok, Ws ws,
                  int32_t *__restrict__ row_of_slot, int32_t *__restrict__ assign_row,
                  int32_t *__restrict__ row_token, uint32_t *__restrict__ row_mask,
                  int64_t row_cap, int32_t *__restrict__ expert_counts,
                  int32_t *__restrict__ send_counts, int32_t *__restrict__ expert_offsets,
                  int32_t *__restrict__ rank_offsets, int32_t *__restrict__ n_rows,
                  int32_t *status)
{
    constexpr int KM = KC ? KC : MD_MAX_TOPK;
    const int K = KC ? KC : k;
    extern __shared__ int smem[];
    const bool dedup = mode == MD_DEDUP;
    const int NB = E + (dedup ? R : 0);
    const int n_tiles = gridDim.x;
    int *s_p = smem;                        // [E] placement
    int *s_he = s_p + E;                    // [E] assignments per expert (all tiles)
    int *s_base = s_he + E;                 // [NB] first row of each bucket
    int *s_pref = s_base + NB;              // [NB] tile total, then first row of the tile
    int *s_toff = s_pref + NB;              // [NB] tile-local start of each output bucket
    int *s_cnt = s_toff + NB;               // [16][NB] rows of earlier warps in the tile
    unsigned *s_bits = reinterpret_cast<unsigned *>(s_cnt + kRankWarps * NB);  // [16][NB]
    int *s_otok = reinterpret_cast<int *>(s_bits + kRankWarps * NB);           // [kStageRows]
    int *s_omsk = s_otok + kStageRows;
    int *s_opos = s_omsk + kStageRows;
    int *s_cs = s_opos + kStageRows;        // [E/32][R] per chunk and rank: sum, then start
    __shared__ int s_rt[2][MD_MAX_RANKS + 1];  // rank totals -> offsets: conventional, dedup
    __shared__ int s_per_rank[MD_MAX_RANKS];
    __shared__ int s_tile, s_timeout, s_nrows;

    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    if (tid == 0) {
        s_tile = (int)atomicAdd(&ws.ctrl[0], 1u);
        s_timeout = 0;
    }
    for (int e = tid; e < E; e += kRankThreads) s_p[e] = p_g[e];
    for (int i = tid; i < 2 * (MD_MAX_RANKS + 1); i += kRankThreads) (&s_rt[0][0])[i] = 0;
    for (int d = tid; d < R; d += kRankThreads) s_per_rank[d] = 0;
    for (int i = tid; i < kRankWarps * NB; i += kRankThreads) s_bits[i] = 0u;
    for (int i = tid; i < ((E + 31) >> 5) * R; i += kRankThreads) s_cs[i] = 0;
    __syncthreads();
    const int tile = s_tile;
    const int64_t t0 = (int64_t)tile * tile_tok;
    const bool have = tid < tile_tok && t0 + tid < T;
    const int64_t t = t0 + tid;

    // the token's experts: issued now, used after the bucket bases
    int e[KM];
#pragma unroll
    for (int j = 0; j < KM; ++j)
        if (KC || j < K) e[j] = have ? __ldg(idx + t * K + j) : -1;

    // everything above overlaps the histogram kernel (programmatic dependent
    // launch); its totals are read only after it has completed
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // ---- bucket bases from the totals (every CTA; tile 0 also writes them out).
    // Conventional order is (p[e], e): per 32-expert chunk and rank, the sum of
    // the chunk's experts on that rank; a scan over chunks per rank; then a
    // prefix among the chunk's own lanes.  All totals are loaded in one round.
    for (int x = tid; x < E; x += kRankThreads) {
        const int he = __ldcg(ws.hist_e + x);
        s_he[x] = he;
        const int d = s_p[x];
        if (d >= 0 && d < R) {
            atomicAdd(&s_cs[(x >> 5) * R + d], he);
            atomicAdd(&s_per_rank[d], 1);
        } else if (tile == 0) {
            md::report(status, MD_ERR_DATA);
        }
    }
    if (dedup)  // column sums of the send matrix: one warp per destination
        for (int dd = w; dd < R; dd += kRankWarps) {
            const int a = __ldcg(ws.send + lane * R + dd);
            const int b = lane + 32 < R ? __ldcg(ws.send + (lane + 32) * R + dd) : 0;
            const int sum = (int)__reduce_add_sync(0xffffffffu, (unsigned)((lane < R ? a : 0) + b));
            if (lane == 0) s_rt[1][dd] = sum;
        }
    __syncthreads();
    const int nchunk = (E + 31) >> 5;
    for (int dd = tid; dd < R; dd += kRankThreads) {  // rank totals (conventional)
        int sum = 0;
        for (int c = 0; c < nchunk; ++c) sum += s_cs[c * R + dd];
        s_rt[0][dd] = sum;
    }
    __syncthreads();
    if (w == 0) {  // exclusive scans over ranks (R <= 64: two values per lane)
        for (int m = 0; m < 2; ++m) {
            const int a = lane < R ? s_rt[m][lane] : 0;
            const int b = lane + 32 < R ? s_rt[m][lane + 32] : 0;
            const int ia = warp_incl_scan(a, lane), ib = warp_incl_scan(b, lane);
            const int tot_a = __shfl_sync(0xffffffffu, ia, 31);
            const int tot = tot_a + __shfl_sync(0xffffffffu, ib, 31);
            __syncwarp();
            if (lane < R) s_rt[m][lane] = ia - a;
            if (lane + 32 < R) s_rt[m][lane + 32] = tot_a + ib - b;
            if (lane == 0) s_rt[m][R] = tot;
            __syncwarp();
        }
        if (!dedup)
            for (int dd = lane; dd <= R; dd += 32) s_rt[1][dd] = s_rt[0][dd];
    }
    __syncthreads();
    for (int dd = tid; dd < R; dd += kRankThreads) {  // chunk starts per rank
        int run = s_rt[0][dd];
        for (int c = 0; c < nchunk; ++c) {
            const int v = s_cs[c * R + dd];
            s_cs[c * R + dd] = run;
            run += v;
        }
    }
    __syncthreads();
    for (int x0 = w * 32; x0 < E; x0 += kRankThreads) {  // one warp per 32-expert chunk
        const int x = x0 + lane;
        const int d = x < E ? s_p[x] : -1;
        const int h = x < E ? s_he[x] : 0;
        int before = 0;
#pragma unroll 8
        for (int q = 0; q < 32; ++q) {
            const int dq = __shfl_sync(0xffffffffu, d, q);
            const int hq = __shfl_sync(0xffffffffu, h, q);
            if (q < lane && dq == d) before += hq;
        }
        if (x < E) s_base[x] = (d >= 0 && d < R) ? s_cs[(x >> 5) * R + d] + before : 0;
    }
    if (dedup)
        for (int dd = tid; dd < R; dd += kRankThreads) s_base[E + dd] = s_rt[1][dd];
    __syncthreads();
    if (tile == 0) {
        for (int x = tid; x < E; x += kRankThreads) {
            expert_counts[x] = s_he[x];
            expert_offsets[x] = s_base[x];
        }
        for (int i = tid; i < R * R; i += kRankThreads) send_counts[i] = __ldcg(ws.send + i);
        for (int d = tid; d <= R; d += kRankThreads) rank_offsets[d] = s_rt[1][d];
        for (int d = tid; d < R; d += kRankThreads)
            if (s_per_rank[d] != E / R) md::report(status, MD_ERR_DATA);
        if (tid == 0) {
            expert_offsets[E] = s_rt[0][R];
            *n_rows = s_rt[1][R];
        }
    }

    // ---- per-token: ranks, which slot carries each dedup row, row masks
    int d[KM];
    int jr[KM];
    unsigned msk[KM];
#pragma unroll
    for (int j = 0; j < KM; ++j) {
        if (!KC && j >= K) break;
        int ee = e[j];
        int dd = (ee >= 0 && ee < E) ? s_p[ee] : -1;
        if (dd >= R) dd = -1;
        if (dd < 0) ee = -1;
        e[j] = ee;
        d[j] = dd;
    }
    if (dedup) {
#pragma unroll
        for (int j = 0; j < KM; ++j) {
            if (!KC && j >= K) break;
            jr[j] = j;
            msk[j] = 0u;
#pragma unroll
            for (int j2 = KM - 1; j2 >= 0; --j2) {
                if (j2 >= K) continue;
                if (d[j2] == d[j] && j2 < j) jr[j] = j2;
                if (d[j2] == d[j]) msk[j] |= 1u << j2;
            }
        }
    }
    // mark this lane in the bucket sets of its warp
    unsigned *wb = s_bits + w * NB;
#pragma unroll
    for (int j = 0; j < KM; ++j) {
        if (!KC && j >= K) break;
        if (d[j] < 0) continue;
        atomicOr(wb + e[j], 1u << lane);
        if (dedup && jr[j] == j) atomicOr(wb + E + d[j], 1u << lane);
    }
    __syncthreads();

    // ---- per-bucket tile totals and rows of earlier warps; the totals are
    // published at once so that later tiles can start their lookback
    for (int b = tid; b < NB; b += kRankThreads) {
        int run = 0;
#pragma unroll
        for (int w2 = 0; w2 < kRankWarps; ++w2) {
            const int c = __popc(s_bits[w2 * NB + b]);
            s_cnt[w2 * NB + b] = run;
            run += c;
        }
        s_pref[b] = run;
        if (tile != ws.skip_tile)
            md::st_relaxed_u64(ws.tiles + (size_t)b * n_tiles + tile,
                               (tile == 0 ? kFlagP : kFlagA) | (unsigned long long)run);
    }
    __syncthreads();
    // tile-local start of each output bucket (the mode's buckets, in order)
    const int ob0 = dedup ? E : 0;
    if (w == 0) {
        int run = 0;
        for (int b0 = ob0; b0 < NB; b0 += 32) {
            const int b = b0 + lane;
            const int c = b < NB ? s_pref[b] : 0;
            const int incl = warp_incl_scan(c, lane);
            if (b < NB) s_toff[b] = run + incl - c;
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) s_nrows = run;
    }
    __syncthreads();

    // ---- tile-local ranks (bucket << 16 | rank inside the tile's bucket run);
    // output rows are staged in shared memory in bucket order
    const unsigned lt = md::lanemask_lt();
    const int *wc = s_cnt + w * NB;
    int ar[KM], rs[KM];
#pragma unroll
    for (int j = 0; j < KM; ++j) {
        if (!KC && j >= K) break;
        ar[j] = -1;
        rs[j] = -1;
        if (d[j] < 0) continue;
        const int x = e[j];
        const int within = wc[x] + __popc(wb[x] & lt);
        ar[j] = (x << 16) | within;
        if (!dedup) {
            rs[j] = ar[j];
            const int o = s_toff[x] + within;
            s_otok[o] = (int)t;
            s_omsk[o] = (int)(1u << j);
            s_opos[o] = ar[j];
        } else if (jr[j] == j) {  // first slot of this token on rank d: owns the row
            const int b = E + d[j];
            const int wd = wc[b] + __popc(wb[b] & lt);
            rs[j] = (b << 16) | wd;
            const int o = s_toff[b] + wd;
            s_otok[o] = (int)t;
            s_omsk[o] = (int)msk[j];
            s_opos[o] = rs[j];
        }
    }
    if (dedup) {  // every slot takes the row of its rank's first slot
#pragma unroll
        for (int j = 0; j < KM; ++j) {
            if (!KC && j >= K) break;
            if (d[j] < 0) continue;
            int r = rs[j];
#pragma unroll
            for (int j2 = 0; j2 < KM; ++j2)
                if (j2 < j && jr[j] == j2) r = rs[j2];
            rs[j] = r;
        }
    }

    // ---- decoupled lookback over earlier tiles.  The words of one bucket are
    // contiguous over tiles.  A warp keeps up to kLookBatch buckets in flight
    // and moves all their windows back together: lane L reads tiles top-2L and
    // top-2L-1, so one round of loads covers 64 earlier tiles of every bucket
    // in the batch.  Counts fit 31 bits, so window sums are one warp reduce.
    for (int b0 = w; b0 < NB; b0 += kRankWarps * kLookBatch) {
        int excl[kLookBatch];
        unsigned pending = 0;  // bit q: bucket b0 + 16 q still looking back
#pragma unroll
        for (int q = 0; q < kLookBatch; ++q) {
            excl[q] = 0;
            if (tile > 0 && b0 + q * kRankWarps < NB) pending |= 1u << q;
        }
        int top = tile - 1;
        long long polls = 0;
        while (pending) {
            unsigned long long v[kLookBatch][2];
#pragma unroll
            for (int q = 0; q < kLookBatch; ++q) {
                const unsigned long long *col = ws.tiles + (size_t)(b0 + q * kRankWarps) * n_tiles;
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int j = top - 2 * lane - u;
                    v[q][u] = ((pending >> q) & 1u) && j >= 0 ? md::ld_relaxed_u64(col + j) : kFlagP;
                }
            }
#pragma unroll
            for (int q = 0; q < kLookBatch; ++q) {
                if (!((pending >> q) & 1u)) continue;
                const unsigned long long *col = ws.tiles + (size_t)(b0 + q * kRankWarps) * n_tiles;
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    // a word not yet published: bounded wait
                    while ((v[q][u] >> 62) == 0ull) {
                        if (++polls > ws.poll_limit) {
                            md::report(status, MD_ERR_TIMEOUT);
                            s_timeout = 1;
                            v[q][u] = kFlagP;
                            break;
                        }
                        __nanosleep(64);
                        v[q][u] = md::ld_relaxed_u64(col + (top - 2 * lane - u));
                    }
                }
                // nearest inclusive prefix: lane order, then u order
                const int fp = (v[q][0] >> 62) == 2ull ? 0 : ((v[q][1] >> 62) == 2ull ? 1 : 2);
                const unsigned pm = __ballot_sync(0xffffffffu, fp < 2);
                const int stop = pm ? __ffs(pm) - 1 : 32;
                unsigned part = 0;
                if (lane < stop) {
                    part = (unsigned)(v[q][0] & kValMask) + (unsigned)(v[q][1] & kValMask);
                } else if (lane == stop) {
                    part = (unsigned)(v[q][0] & kValMask) +
                           (fp == 1 ? (unsigned)(v[q][1] & kValMask) : 0u);
                }
                excl[q] += (int)__reduce_add_sync(0xffffffffu, part);
                if (pm) pending &= ~(1u << q);
            }
            top -= 64;
        }
#pragma unroll
        for (int q = 0; q < kLookBatch; ++q) {
            const int b = b0 + q * kRankWarps;
            if (b < NB && lane == 0) {
                if (tile > 0 && tile != ws.skip_tile)
                    md::st_relaxed_u64(ws.tiles + (size_t)b * n_tiles + tile,
                                       kFlagP | (unsigned long long)(excl[q] + s_pref[b]));
                s_pref[b] = s_base[b] + excl[q];
            }
        }
    }
    __syncthreads();
    if (s_timeout) return;  // positions unknown: leave outputs, status says why

    // ---- global rows: the tile's start in the bucket + the tile-local rank
#pragma unroll
    for (int j = 0; j < KM; ++j) {
        if (!KC && j >= K) break;
        if (ar[j] >= 0) ar[j] = s_pref[ar[j] >> 16] + (ar[j] & 0xffff);
        if (rs[j] >= 0) rs[j] = s_pref[rs[j] >> 16] + (rs[j] & 0xffff);
    }
    if (have) store_row<KC>(assign_row + t * K, ar, K), store_row<KC>(row_of_slot + t * K, rs, K);
    for (int o = tid; o < s_nrows; o += kRankThreads) {
        const int pk = s_opos[o];
        const int pos = s_pref[pk >> 16] + (pk & 0xffff);
        if (pos >= 0 && pos < row_cap) {
            row_token[pos] = s_otok[o];
            row_mask[pos] = (uint32_t)s_omsk[o];
        } else {
            md::report(status, MD_ERR_DATA);
        }
    }
}

size_t rank_smem(int E, int R, int mode)
{
    const int NB = E + (mode == MD_DEDUP ? R : 0);
    return (size_t)(2 * E + (2 * kRankWarps + 3) * NB + 3 * kStageRows + ((E + 31) / 32) * R) *
           sizeof(int);
}

size_t hist_smem(int E, int k, int R)
{
    return (size_t)(2 * E + R * R + kHistThreads * (k | 1)) * sizeof(int);
}

int check_layout_args(int64_t T, int E, int k, int R, int mode)
{
    if (T < 0 || E < 1 || k < 1 || R < 1 || k > E || k > MD_MAX_TOPK) return MD_ERR_ARG;
    if (mode != MD_CONV && mode != MD_DEDUP) return MD_ERR_ARG;
    if (E > MD_MAX_EXPERTS || R > MD_MAX_RANKS) return MD_ERR_UNSUPPORTED;
    if (T % R != 0 || E % R != 0) return MD_ERR_ARG;
    if (T * (int64_t)k >= (int64_t)1 << 31) return MD_ERR_UNSUPPORTED;
    return MD_OK;
}

template <int KC>
void set_attrs()
{
    cudaFuncSetAttribute(k_layout_rank<KC>, cudaFuncAttributeMaxDynamicSharedMemorySize, 220 * 1024);
    cudaFuncSetAttribute(k_layout_hist<KC>, cudaFuncAttributeMaxDynamicSharedMemorySize, 100 * 1024);
}

template <int KC>
void launch_layout(const int32_t *topk_idx, int64_t T, int E, int k, int R,
                   const int32_t *expert_to_rank, int mode, const Plan &pl, const Ws &ws,
                   int32_t *row_of_slot, int32_t *assign_row, int32_t *row_token,
                   uint32_t *row_mask, int64_t cap, int32_t *send_counts,
                   int32_t *expert_counts, int32_t *expert_offsets, int32_t *rank_offsets,
                   int32_t *n_rows, int32_t *dev_status, cudaStream_t s)
{
    // each kernel may start while the previous one drains (programmatic
    // dependent launch); it waits (griddepcontrol.wait) before using its results
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t hc = {};
    hc.gridDim = dim3((unsigned)(T > 0 ? (T + kHistThreads - 1) / kHistThreads : 1));
    hc.blockDim = dim3(kHistThreads);
    hc.dynamicSmemBytes = hist_smem(E, k, R);
    hc.stream = s;
    hc.attrs = attr;
    hc.numAttrs = 1;
    cudaLaunchKernelEx(&hc, k_layout_hist<KC>, topk_idx, T, E, k, R, expert_to_rank, mode, ws,
                       dev_status);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)pl.n_tiles);
    cfg.blockDim = dim3(kRankThreads);
    cfg.dynamicSmemBytes = rank_smem(E, R, mode);
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, k_layout_rank<KC>, topk_idx, T, E, k, R, expert_to_rank, mode,
                       pl.tile_tok, ws, row_of_slot, assign_row, row_token, row_mask, cap,
                       expert_counts, send_counts, expert_offsets, rank_offsets, n_rows,
                       dev_status);
}

}  // namespace

extern "C" size_t md_dispatch_layout_workspace_size(int64_t T, int E, int k, int R, int mode)
{
    if (check_layout_args(T, E, k, R, mode) != MD_OK) return 0;
    return plan(T, E, k, R, mode).total;
}

extern "C" int md_dispatch_layout(const int32_t *topk_idx, int64_t T, int E, int k, int R,
                                  const int32_t *expert_to_rank, int mode, int32_t *row_of_slot,
                                  int32_t *assign_row, int32_t *row_token, uint32_t *row_mask,
                                  int32_t *send_counts, int32_t *expert_counts,
                                  int32_t *expert_offsets, int32_t *rank_offsets, int32_t *n_rows,
                                  void *workspace, size_t workspace_bytes, int32_t *dev_status,
                                  void *stream)
{
    int rc = check_layout_args(T, E, k, R, mode);
    if (rc != MD_OK) return rc;
    if (!expert_to_rank || !send_counts || !expert_counts || !expert_offsets || !rank_offsets ||
        !n_rows)
        return MD_ERR_ARG;
    if (T > 0 && (!topk_idx || !row_of_slot || !assign_row || !row_token || !row_mask))
        return MD_ERR_ARG;
    const Plan pl = plan(T, E, k, R, mode);
    if (!workspace || workspace_bytes < pl.total) return MD_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MD_ERR_ARG;
    cudaStream_t s = md::as_stream(stream);
    const Ws ws = carve(workspace, pl);

    static std::atomic<uint64_t> attr_done{0};
    md::once_per_device(attr_done, [] {
        set_attrs<0>();
        set_attrs<1>();
        set_attrs<2>();
        set_attrs<4>();
        set_attrs<6>();
        set_attrs<8>();
    });
    {
        const size_t n16 = pl.total / 16;
        int zb = (int)((n16 + 255) / 256);
        if (zb > md::sm_count()) zb = md::sm_count();
        k_layout_zero<<<zb < 1 ? 1 : zb, 256, 0, s>>>(static_cast<uint4 *>(workspace), n16,
                                                     dev_status);
        md::count_launches(1);
    }

    const int64_t cap = mode == MD_CONV ? T * k : T * (int64_t)(k < R ? k : R);
#define MD_LAYOUT(KC)                                                                            \
    launch_layout<KC>(topk_idx, T, E, k, R, expert_to_rank, mode, pl, ws, row_of_slot,          \
                      assign_row, row_token, row_mask, cap, send_counts, expert_counts,         \
                      expert_offsets, rank_offsets, n_rows, dev_status, s)
    // the specialised kernels store a token's k outputs as vectors
    const bool vec_ok = md::aligned16(assign_row) && md::aligned16(row_of_slot);
    switch (vec_ok ? k : 0) {
    case 1: MD_LAYOUT(1); break;
    case 2: MD_LAYOUT(2); break;
    case 4: MD_LAYOUT(4); break;
    case 6: MD_LAYOUT(6); break;
    case 8: MD_LAYOUT(8); break;
    default: MD_LAYOUT(0); break;
    }
#undef MD_LAYOUT
    md::count_launches(2);
    return md::launch_status();
}

// ------------------------------------------------------------------------
// md_dispatch_layout_noalloc: the same layout for callers that cannot
// allocate device memory.  Its scratch is the file-scope array below, so the
// library itself allocates nothing at call time.
// ------------------------------------------------------------------------
#include <mutex>

namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)4 << 20;  // MD_NOALLOC_LAYOUT_SCRATCH_BYTES

// Resident on every GPU that loads the library, for the life of the process.
static __device__ __align__(256) unsigned char g_layout_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 256;
std::mutex g_scratch_mutex;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of g_layout_scratch on the current device.  In host code the
// symbol names a host-side stand-in, so the address must be looked up with
// cudaGetSymbolAddress while that device is current; it is cached per device.
int scratch_for_current_device(void **addr)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MD_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_layout_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return MD_ERR_CUDA;
        }
        g_scratch_addr[dev] = p;
    }
    *addr = g_scratch_addr[dev];
    return MD_OK;
}

}  // namespace

extern "C" size_t md_dispatch_layout_noalloc_max_scratch(void) { return kNoAllocScratchBytes; }

extern "C" int md_dispatch_layout_noalloc(const int32_t *topk_idx, int64_t T, int E, int k, int R,
                                          const int32_t *expert_to_rank, int mode,
                                          int32_t *row_of_slot, int32_t *assign_row,
                                          int32_t *row_token, uint32_t *row_mask,
                                          int32_t *send_counts, int32_t *expert_counts,
                                          int32_t *expert_offsets, int32_t *rank_offsets,
                                          int32_t *n_rows, int32_t *dev_status, void *stream)
{
    int rc = check_layout_args(T, E, k, R, mode);
    if (rc != MD_OK) return rc;
    if (plan(T, E, k, R, mode).total > kNoAllocScratchBytes) return MD_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    if ((rc = scratch_for_current_device(&scratch)) != MD_OK) return rc;
    // The shared array keeps the previous call's contents; md_dispatch_layout
    // clears the part that must start at zero on the stream before using it.
    return md_dispatch_layout(topk_idx, T, E, k, R, expert_to_rank, mode, row_of_slot, assign_row,
                              row_token, row_mask, send_counts, expert_counts, expert_offsets,
                              rank_offsets, n_rows, scratch, kNoAllocScratchBytes, dev_status,
                              stream);
}
