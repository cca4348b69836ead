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
// rows by (d, t).  One cooperative kernel, k_layout, one token per thread
// (the token's k experts in registers; k is a template parameter for the
// common values).  CTA c owns a contiguous run of tiles (512 tokens each,
// fewer when k > 8).
//   A. Every CTA counts its tokens per bucket (shared-memory histograms) and
//      the send-matrix rows of the source ranks it covers, writes them to the
//      workspace and stamps its arrival word (cleared to 0 before the launch).
//   B. After every stamp is seen (a bounded wait), each CTA reads the count
//      table: bucket totals give the bucket bases, the counts of CTAs before
//      it give its start inside each bucket.  Each CTA also sums a slice of
//      the send matrix.
//   C. Tile by tile, each warp marks which of its lanes hit each bucket (a
//      32-bit set per bucket, built with shared atomicOr), so a pair's rank
//      among the warp's earlier tokens is a popcount; rows are staged in
//      shared memory in bucket order and written out in runs.
// When a cooperative launch is refused (its CTAs cannot all be resident, e.g.
// while other work holds SMs), the same kernel runs split in two launches:
// A, then B and C; the second launch starts after every CTA's counts, so no
// arrival wait is needed.
// Nothing in the workspace has to start at zero: every call first clears the
// arrival words on its stream (a 1 KiB memset, recorded too when the stream is
// capturing), so a word left over from an earlier call, or from whatever the
// memory held before, can never pass for this call's arrival; every count is
// written before it is read.
#include "common.cuh"

namespace {

// one token per thread; 256-thread CTAs, two per SM, measured no faster
constexpr int kRankThreads = 512;
constexpr int kRankWarps = kRankThreads / 32;
constexpr int kStageRows = 4096;   // output rows a tile can stage
constexpr int kMaxCtas = 256;      // CTAs of one launch; the workspace is sized for it
constexpr long long kPollLimit = 1ll << 22;
constexpr int kPhaseCounts = 1, kPhaseWait = 2, kPhaseRanks = 4;

struct Ws {
    long long poll_limit;         // bound of the arrival wait
    int skip_cta;                 // test hook: this CTA never stamps its arrival (-1: none)
    unsigned epoch;               // the arrival stamp (the words are cleared to 0 first)
    unsigned *flags;              // [kMaxCtas] arrival words
    int *cnt;                     // [NB][kMaxCtas] bucket counts per CTA
    int *part;                    // [(kMaxCtas + R) * R] send rows: CTA c, source s at row c + s
};

// tokens per tile: one per thread, fewer when k is large so that the tile's
// rows fit the staging area
int tile_tokens(int k)
{
    if (k <= kStageRows / kRankThreads) return kRankThreads;
    int t = kStageRows / k, p = 1;
    while (p * 2 <= t) p *= 2;
    return p;
}

struct Plan {
    size_t off_flags, off_cnt, off_part, total;
    int tile_tok, n_tiles, nb;
};

Plan plan(int64_t T, int E, int k, int R, int mode)
{
    Plan p;
    p.tile_tok = tile_tokens(k);
    p.n_tiles = (int)((T + p.tile_tok - 1) / p.tile_tok);
    if (p.n_tiles < 1) p.n_tiles = 1;  // CTA 0 also writes the count outputs
    p.nb = E + (mode == MD_DEDUP ? R : 0);
    size_t o = 0;
    p.off_flags = o;
    o += md::align_up((size_t)kMaxCtas * 4, 256);
    p.off_cnt = o;
    o += md::align_up((size_t)kMaxCtas * p.nb * 4, 256);
    p.off_part = o;
    o += md::align_up((size_t)(kMaxCtas + R) * R * 4, 256);
    p.total = o;
    return p;
}

Ws carve(void *ws, const Plan &p)
{
    char *b = static_cast<char *>(ws);
    Ws w;
    w.poll_limit = md::hook_poll_limit(kPollLimit);
    w.skip_cta = md::hook_layout_skip_tile();
    w.epoch = 1u;
    w.flags = reinterpret_cast<unsigned *>(b + p.off_flags);
    w.cnt = reinterpret_cast<int *>(b + p.off_cnt);
    w.part = reinterpret_cast<int *>(b + p.off_part);
    return w;
}

__device__ __forceinline__ uint4 ld_relaxed_v4(const unsigned *p)
{
    uint4 v;
    asm volatile("ld.relaxed.gpu.global.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p)
                 : "memory");
    return v;
}

__device__ __forceinline__ void st_relaxed_u32(unsigned *p, unsigned v)
{
    asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
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
    k_layout(const int32_t *__restrict__ idx, int64_t T, int E, int k, int R,
             const int32_t *__restrict__ p_g, int mode, int tile_tok, int n_tiles, int tpc, Ws ws,
             int32_t *__restrict__ row_of_slot, int32_t *__restrict__ assign_row,
             int32_t *__restrict__ row_token, uint32_t *__restrict__ row_mask, int64_t row_cap,
             int32_t *__restrict__ expert_counts, int32_t *__restrict__ send_counts,
             int32_t *__restrict__ expert_offsets, int32_t *__restrict__ rank_offsets,
             int32_t *__restrict__ n_rows, int32_t *status, int phases)
{
    // phases: kPhaseCounts (A, publish the counts), kPhaseWait (the arrival
    // wait: all CTAs resident), kPhaseRanks (B, bases, C).  One cooperative
    // launch runs all three; the split form runs counts, then ranks in a
    // second launch whose start orders it after every CTA's counts.
    const bool do_counts = phases & kPhaseCounts, do_wait = phases & kPhaseWait;
    const bool do_ranks = phases & kPhaseRanks;
    constexpr int KM = KC ? KC : MD_MAX_TOPK;
    const int K = KC ? KC : k;
    extern __shared__ int smem[];
    const bool dedup = mode == MD_DEDUP;
    const int NB = E + (dedup ? R : 0);
    const int G = gridDim.x, cta = blockIdx.x;
    int *s_p = smem;                        // [E] placement
    int *s_he = s_p + E;                    // [E] assignments per expert (all CTAs)
    int *s_base = s_he + E;                 // [NB] first row of each bucket
    int *s_run = s_base + NB;               // [NB] this CTA's next row in each bucket
    int *s_tcnt = s_run + NB;               // [NB] bucket totals, then the tile's bucket counts
    int *s_toff = s_tcnt + NB;              // [NB] tile-local start of each output bucket
    int *s_cnt = s_toff + NB;               // [16][NB] rows of earlier warps in the tile
    unsigned *s_bits = reinterpret_cast<unsigned *>(s_cnt + kRankWarps * NB);  // [16][NB]
    int *s_otok = reinterpret_cast<int *>(s_bits + kRankWarps * NB);           // [kStageRows]
    int *s_omsk = s_otok + kStageRows;
    int *s_opos = s_omsk + kStageRows;
    int *s_cs = s_opos + kStageRows;        // [E/32][R] per chunk and rank: sum, then start
    int *s_acnt = s_cnt;                    // phase A: [NB] this CTA's bucket counts
    int *s_send = s_otok;                   // phase A: [R*R] this CTA's send counts
    __shared__ int s_rt[2][MD_MAX_RANKS + 1];  // rank totals -> offsets: conventional, dedup
    __shared__ int s_per_rank[MD_MAX_RANKS];
    __shared__ int s_timeout, s_nrows;

    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int tile_lo = cta * tpc;
    const int tile_hi = tile_lo + tpc < n_tiles ? tile_lo + tpc : n_tiles;
    const int64_t Tr = R > 0 && T > 0 ? T / R : 1;
    if (tid == 0) s_timeout = 0;
    for (int e = tid; e < E; e += kRankThreads) s_p[e] = p_g[e];
    for (int i = tid; i < NB; i += kRankThreads) s_acnt[i] = 0;
    for (int i = tid; i < R * R; i += kRankThreads) s_send[i] = 0;
    for (int i = tid; i < 2 * (MD_MAX_RANKS + 1); i += kRankThreads) (&s_rt[0][0])[i] = 0;
    for (int d = tid; d < R; d += kRankThreads) s_per_rank[d] = 0;
    for (int i = tid; i < ((E + 31) >> 5) * R; i += kRankThreads) s_cs[i] = 0;
    // the first tile's experts: used in A and again in C
    int e0[KM];
    {
        const int64_t t = (int64_t)tile_lo * tile_tok + tid;
        const bool have = tile_lo < tile_hi && tid < tile_tok && t < T;
#pragma unroll
        for (int j = 0; j < KM; ++j)
            if (KC || j < K) e0[j] = have ? __ldg(idx + t * K + j) : -1;
    }
    // tokens t_first .. t_last; when they all come from one source rank, its
    // send row follows from the bucket counts
    const int64_t t_first = (int64_t)tile_lo * tile_tok;
    const int64_t t_last = ((int64_t)tile_hi * tile_tok < T ? (int64_t)tile_hi * tile_tok : T) - 1;
    const int s_lo = t_first <= t_last ? (int)(t_first / Tr) : 0;
    const int s_hi = t_first <= t_last ? (int)(t_last / Tr) : -1;
    const bool one_src = s_lo == s_hi;
    __syncthreads();

    // ---- A. bucket counts and send rows of this CTA's tokens
    bool bad = false;
    for (int tile = tile_lo; do_counts && tile < tile_hi; ++tile) {
        const int64_t t = (int64_t)tile * tile_tok + tid;
        if (tid >= tile_tok || t >= T) continue;
        int e[KM], d[KM];
#pragma unroll
        for (int j = 0; j < KM; ++j)
            if (KC || j < K) e[j] = tile == tile_lo ? e0[j] : __ldg(idx + t * K + j);
        const int src = (int)(t / Tr);
#pragma unroll
        for (int j = 0; j < KM; ++j) {
            if (!KC && j >= K) break;
            int ee = e[j];
            int dd = (ee >= 0 && ee < E) ? s_p[ee] : -1;
            if (dd >= R) dd = -1;
            if (dd < 0) { bad = true; ee = -1; }
            e[j] = ee;
            d[j] = dd;
            bool rep = true;  // the token's first slot on rank dd
#pragma unroll
            for (int j2 = 0; j2 < KM; ++j2) {
                if (j2 >= j) break;
                if (ee >= 0 && e[j2] == ee) bad = true;  // expert twice in one token
                if (d[j2] == dd) rep = false;
            }
            if (ee >= 0) {
                atomicAdd(&s_acnt[ee], 1);
                if (dedup && rep) atomicAdd(&s_acnt[E + dd], 1);
                if (!one_src && (!dedup || rep)) atomicAdd(&s_send[src * R + dd], 1);
            }
        }
    }
    __syncthreads();
    if (do_counts && one_src) {
        if (dedup) {
            for (int dd = tid; dd < R; dd += kRankThreads) s_send[s_lo * R + dd] = s_acnt[E + dd];
        } else {
            for (int x = tid; x < E; x += kRankThreads) {
                const int dd = s_p[x];
                if (dd >= 0 && dd < R && s_acnt[x]) atomicAdd(&s_send[s_lo * R + dd], s_acnt[x]);
            }
        }
        __syncthreads();
    }
    if (do_counts) {
        for (int b = tid; b < NB; b += kRankThreads) ws.cnt[(size_t)b * kMaxCtas + cta] = s_acnt[b];
        for (int i = tid; i < (s_hi - s_lo + 1) * R; i += kRankThreads) {
            const int s = s_lo + i / R, dd = i % R;
            ws.part[(size_t)(cta + s) * R + dd] = s_send[s * R + dd];
        }
        __syncthreads();
        if (do_wait && tid == 0 && cta != ws.skip_cta) {
            __threadfence();
            st_relaxed_u32(ws.flags + cta, ws.epoch);
        }
    }
    if (!do_ranks) {  // the split form's first launch ends here
        if (bad) md::report(status, MD_ERR_DATA);
        return;
    }
    // every CTA's counts are in once its arrival word is stamped; one
    // warp reads all stamps, four per 16-byte load
    if (do_wait && w == 0) {
        long long polls = 0;
        for (;;) {
            bool ok = true;
            for (int i = lane * 4; i < G; i += 128) {
                const uint4 v = ld_relaxed_v4(ws.flags + i);
                ok = ok && v.x == ws.epoch && (i + 1 >= G || v.y == ws.epoch) &&
                     (i + 2 >= G || v.z == ws.epoch) && (i + 3 >= G || v.w == ws.epoch);
            }
            if (__all_sync(0xffffffffu, ok)) break;
            if (++polls > ws.poll_limit) {
                if (lane == 0) s_timeout = 1;
                break;
            }
            if (polls > 16) __nanosleep(32);
        }
        __threadfence();
    }
    __syncthreads();
    if (s_timeout) {  // positions unknown: leave outputs, status says why
        if (tid == 0) md::report(status, MD_ERR_TIMEOUT);
        return;
    }
    if (bad) md::report(status, MD_ERR_DATA);

    // ---- B. bucket totals and this CTA's start in each bucket: a bucket's
    // counts of all CTAs are contiguous, one warp reads them in one pass, for
    // 4 buckets at a time
    for (int b0 = w * 4; b0 < NB; b0 += kRankWarps * 4) {
        int v[4][kMaxCtas / 32];
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int i = 0; i < kMaxCtas / 32; ++i) {
                const int c2 = lane + 32 * i;
                v[q][i] = b0 + q < NB && c2 < G ? __ldcg(ws.cnt + (size_t)(b0 + q) * kMaxCtas + c2) : 0;
            }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            int tot = 0, pre = 0;
#pragma unroll
            for (int i = 0; i < kMaxCtas / 32; ++i) {
                tot += v[q][i];
                pre += lane + 32 * i < cta ? v[q][i] : 0;
            }
            tot = (int)__reduce_add_sync(0xffffffffu, (unsigned)tot);
            pre = (int)__reduce_add_sync(0xffffffffu, (unsigned)pre);
            if (lane == 0 && b0 + q < NB) {
                s_tcnt[b0 + q] = tot;
                s_run[b0 + q] = pre;
            }
        }
    }
    __syncthreads();

    // bucket bases from the totals.  Conventional order is (p[e], e): per
    // 32-expert chunk and rank, the sum of the chunk's experts on that rank; a
    // scan over chunks per rank; then a prefix among the chunk's own lanes.
    for (int x = tid; x < E; x += kRankThreads) {
        const int he = s_tcnt[x];
        s_he[x] = he;
        const int d = s_p[x];
        if (d >= 0 && d < R) {
            atomicAdd(&s_cs[(x >> 5) * R + d], he);
            atomicAdd(&s_per_rank[d], 1);
        } else if (cta == 0) {
            md::report(status, MD_ERR_DATA);
        }
    }
    if (dedup)
        for (int dd = tid; dd < R; dd += kRankThreads) s_rt[1][dd] = s_tcnt[E + dd];
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
    for (int b = tid; b < NB; b += kRankThreads) s_run[b] += s_base[b];
    if (cta == 0) {
        for (int x = tid; x < E; x += kRankThreads) {
            expert_counts[x] = s_he[x];
            expert_offsets[x] = s_base[x];
        }
        for (int d = tid; d <= R; d += kRankThreads) rank_offsets[d] = s_rt[1][d];
        for (int d = tid; d < R; d += kRankThreads)
            if (s_per_rank[d] != E / R) md::report(status, MD_ERR_DATA);
        if (tid == 0) {
            expert_offsets[E] = s_rt[0][R];
            *n_rows = s_rt[1][R];
        }
    }
    // entries cta, cta + G, ... of the send matrix: source s was counted by the
    // CTAs that own tokens s*T/R .. (s+1)*T/R - 1
    for (int i = cta + G * tid; i < R * R; i += G * kRankThreads) {
        int sum = 0;
        if (T > 0) {
            const int s = i / R, dd = i % R;
            const int c_lo = (int)((int64_t)s * Tr / tile_tok) / tpc;
            const int c_hi = (int)(((int64_t)s + 1) * Tr - 1) / tile_tok / tpc;
            for (int c2 = c_lo; c2 <= c_hi; ++c2) sum += __ldcg(ws.part + (size_t)(c2 + s) * R + dd);
        }
        send_counts[i] = sum;
    }
    __syncthreads();

    // ---- C. rows, tile by tile
    const unsigned lt = md::lanemask_lt();
    unsigned *wb = s_bits + w * NB;
    const int *wc = s_cnt + w * NB;
    const int ob0 = dedup ? E : 0;
    for (int tile = tile_lo; tile < tile_hi; ++tile) {
        for (int i = tid; i < kRankWarps * NB; i += kRankThreads) s_bits[i] = 0u;
        const int64_t t = (int64_t)tile * tile_tok + tid;
        const bool have = tid < tile_tok && t < T;
        int e[KM];
#pragma unroll
        for (int j = 0; j < KM; ++j)
            if (KC || j < K) e[j] = e0[j];
        if (tile + 1 < tile_hi) {  // the next tile's experts load while this one is ranked
            const int64_t tn = t + tile_tok;
            const bool hn = tid < tile_tok && tn < T;
#pragma unroll
            for (int j = 0; j < KM; ++j)
                if (KC || j < K) e0[j] = hn ? __ldg(idx + tn * K + j) : -1;
        }
        __syncthreads();

        // per-token: ranks, which slot carries each dedup row, row masks
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
#pragma unroll
        for (int j = 0; j < KM; ++j) {
            if (!KC && j >= K) break;
            if (d[j] < 0) continue;
            atomicOr(wb + e[j], 1u << lane);
            if (dedup && jr[j] == j) atomicOr(wb + E + d[j], 1u << lane);
        }
        __syncthreads();

        // per-bucket tile counts and rows of earlier warps
        for (int b = tid; b < NB; b += kRankThreads) {
            int run = 0;
#pragma unroll
            for (int w2 = 0; w2 < kRankWarps; ++w2) {
                const int c = __popc(s_bits[w2 * NB + b]);
                s_cnt[w2 * NB + b] = run;
                run += c;
            }
            s_tcnt[b] = run;
        }
        __syncthreads();
        // tile-local start of each output bucket (the mode's buckets, in order)
        if (w == 0) {
            int run = 0;
            for (int b0 = ob0; b0 < NB; b0 += 32) {
                const int b = b0 + lane;
                const int c = b < NB ? s_tcnt[b] : 0;
                const int incl = warp_incl_scan(c, lane);
                if (b < NB) s_toff[b] = run + incl - c;
                run += __shfl_sync(0xffffffffu, incl, 31);
            }
            if (lane == 0) s_nrows = run;
        }
        __syncthreads();

        // global rows: this CTA's next row in the bucket + the rank inside the
        // tile; output rows are staged in shared memory in bucket order
        int ar[KM], rs[KM];
#pragma unroll
        for (int j = 0; j < KM; ++j) {
            if (!KC && j >= K) break;
            ar[j] = -1;
            rs[j] = -1;
            if (d[j] < 0) continue;
            const int x = e[j];
            const int within = wc[x] + __popc(wb[x] & lt);
            ar[j] = s_run[x] + within;
            if (!dedup) {
                rs[j] = ar[j];
                const int o = s_toff[x] + within;
                s_otok[o] = (int)t;
                s_omsk[o] = (int)(1u << j);
                s_opos[o] = ar[j];
            } else if (jr[j] == j) {  // first slot of this token on rank d: owns the row
                const int b = E + d[j];
                const int wd = wc[b] + __popc(wb[b] & lt);
                rs[j] = s_run[b] + wd;
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
        if (have) store_row<KC>(assign_row + t * K, ar, K), store_row<KC>(row_of_slot + t * K, rs, K);
        __syncthreads();
        for (int o = tid; o < s_nrows; o += kRankThreads) {
            const int pos = s_opos[o];
            if (pos >= 0 && pos < row_cap) {
                row_token[pos] = s_otok[o];
                row_mask[pos] = (uint32_t)s_omsk[o];
            } else {
                md::report(status, MD_ERR_DATA);
            }
        }
        for (int b = tid; b < NB; b += kRankThreads) s_run[b] += s_tcnt[b];
        __syncthreads();
    }
}

size_t layout_smem(int E, int R, int mode)
{
    const int NB = E + (mode == MD_DEDUP ? R : 0);
    return (size_t)(2 * E + (2 * kRankWarps + 4) * NB + 3 * kStageRows + ((E + 31) / 32) * R) *
           sizeof(int);
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

constexpr size_t kLayoutSmemMax = (size_t)(2 * 1024 + (2 * kRankWarps + 4) * (1024 + 64) +
                                           3 * kStageRows + 32 * 64) * sizeof(int);

// CTAs of k_layout<KC> resident per SM with `smem` bytes of dynamic shared
// memory (the limit is raised to the largest size once per device; the
// occupancy query is host arithmetic, so it runs per call)
template <int KC>
int layout_per_sm(size_t smem)
{
    static std::atomic<uint64_t> done{0};
    static std::atomic<int> attr_ok[64];
    md::once_per_device(done, [] {
        int dev = 0;
        cudaGetDevice(&dev);
        const bool ok = cudaFuncSetAttribute(k_layout<KC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kLayoutSmemMax) == cudaSuccess;
        if (!ok) cudaGetLastError();
        attr_ok[dev & 63].store(ok ? 1 : 0);
    });
    int dev = 0;
    cudaGetDevice(&dev);
    if (!attr_ok[dev & 63].load()) return 0;
    int nb = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, k_layout<KC>, kRankThreads, smem) != cudaSuccess) {
        cudaGetLastError();
        nb = 0;
    }
    return nb;
}

template <int KC>
int launch_layout(const int32_t *topk_idx, int64_t T, int E, int k, int R,
                  const int32_t *expert_to_rank, int mode, const Plan &pl, const Ws &ws,
                  int32_t *row_of_slot, int32_t *assign_row, int32_t *row_token,
                  uint32_t *row_mask, int64_t cap, int32_t *send_counts, int32_t *expert_counts,
                  int32_t *expert_offsets, int32_t *rank_offsets, int32_t *n_rows,
                  int32_t *dev_status, cudaStream_t s)
{
    const size_t smem = layout_smem(E, R, mode);
    const int per_sm = layout_per_sm<KC>(smem);
    if (per_sm < 1 || smem > kLayoutSmemMax) return MD_ERR_UNSUPPORTED;
    // every CTA waits for all the others: the grid must be resident at once
    int resident = md::sm_count() * per_sm;
    if (resident > kMaxCtas) resident = kMaxCtas;
    const int tpc = (pl.n_tiles + resident - 1) / resident;
    const int G = (pl.n_tiles + tpc - 1) / tpc;
    int tile_tok = pl.tile_tok, n_tiles = pl.n_tiles, mode_ = mode, k_ = k, E_ = E, R_ = R;
    int64_t T_ = T, cap_ = cap;
    Ws ws_ = ws;
    const int path = md::layout_path();
    if (path != MD_LAYOUT_SPLIT) {
        int phases = kPhaseCounts | kPhaseWait | kPhaseRanks;
        void *args[] = {(void *)&topk_idx, &T_,          &E_,         &k_,          &R_,
                        (void *)&expert_to_rank, &mode_, &tile_tok,  &n_tiles,     (void *)&tpc,
                        &ws_,        (void *)&row_of_slot, (void *)&assign_row, (void *)&row_token,
                        (void *)&row_mask, &cap_, (void *)&expert_counts, (void *)&send_counts,
                        (void *)&expert_offsets, (void *)&rank_offsets, (void *)&n_rows,
                        (void *)&dev_status, &phases};
        md::count_launches(1);
        if (cudaLaunchCooperativeKernel((const void *)k_layout<KC>, dim3((unsigned)G), dim3(kRankThreads),
                                        args, smem, s) == cudaSuccess)
            return MD_OK;
        cudaGetLastError();  // refused (e.g. SMs held by other work): split, unless forbidden
        if (path == MD_LAYOUT_COOPERATIVE) return MD_ERR_CUDA;
    }
    // split form: the counts of every CTA, then the ranks in a second launch;
    // no CTA waits on another, so the grid need not be resident at once
    md::count_launches(2);
    k_layout<KC><<<(unsigned)G, kRankThreads, smem, s>>>(
        topk_idx, T, E, k, R, expert_to_rank, mode, tile_tok, n_tiles, tpc, ws, row_of_slot,
        assign_row, row_token, row_mask, cap, expert_counts, send_counts, expert_offsets, rank_offsets,
        n_rows, dev_status, kPhaseCounts);
    k_layout<KC><<<(unsigned)G, kRankThreads, smem, s>>>(
        topk_idx, T, E, k, R, expert_to_rank, mode, tile_tok, n_tiles, tpc, ws, row_of_slot,
        assign_row, row_token, row_mask, cap, expert_counts, send_counts, expert_offsets, rank_offsets,
        n_rows, dev_status, kPhaseRanks);
    return md::launch_status();
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
    Ws ws = carve(workspace, pl);
    // The status word and the arrival words are cleared on the stream before
    // the kernel, eagerly and under capture alike (a graph records both
    // memsets, so every replay waits for its own counts).  Stale arrival words
    // can therefore never let a CTA pass the wait early.
    if ((rc = md::clear_status(dev_status, s)) != MD_OK) return rc;
    if (md::layout_path() != MD_LAYOUT_SPLIT) {  // the split form has no arrival wait
        md::count_memsets(1);
        if (cudaMemsetAsync(ws.flags, 0, (size_t)kMaxCtas * 4, s) != cudaSuccess) {
            cudaGetLastError();
            return MD_ERR_CUDA;
        }
    }

    const int64_t cap = mode == MD_CONV ? T * k : T * (int64_t)(k < R ? k : R);
#define MD_LAYOUT(KC)                                                                            \
    rc = launch_layout<KC>(topk_idx, T, E, k, R, expert_to_rank, mode, pl, ws, row_of_slot,     \
                           assign_row, row_token, row_mask, cap, send_counts, expert_counts,    \
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
    return rc;
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
    // The shared array keeps the previous call's contents; nothing in it has to
    // start at zero (md_dispatch_layout clears the arrival words on the stream
    // before its kernel).
    return md_dispatch_layout(topk_idx, T, E, k, R, expert_to_rank, mode, row_of_slot, assign_row,
                              row_token, row_mask, send_counts, expert_counts, expert_offsets,
                              rank_offsets, n_rows, scratch, kNoAllocScratchBytes, dev_status,
                              stream);
}
