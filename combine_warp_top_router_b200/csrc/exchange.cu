// exchange.cu -- the dispatch and combine exchange between real EP ranks
// (md_exchange_plan, md_dispatch_exchange, md_combine_partials,
// md_combine_exchange).
//
// "Expert Coupling in MoE Pretraining" (PicX summary), The Communication
// Bottleneck: each MoE layer runs two all-to-alls, dispatch and combine;
// Method 1: the deduplicating dispatcher sends one row per (token,
// destination rank) carrying the token's expert IDs and routing
// probabilities for that rank.  "DODOCO: MoE AlltoAll Traffic Matrices on
// Real Text", send_matrices.csv: source s sends send_counts[s][d] rows to
// rank d; combine returns the same volumes transposed.
//
// With one process per GPU, every rank lays out its own tokens
// (md_dispatch_layout over its T_r tokens: rows ordered (d, t) for dedup),
// so its send row is the size of each destination block.  After an
// all-gather of those R counts, md_exchange_plan gives each source the first
// row of its block in every destination's receive buffer: rank d receives
// the blocks of sources 0, 1, ... in order, which is the (d, global token)
// order of the single-GPU layout.  The data then moves in one kernel per
// direction that writes or reads the peers' buffers directly (P2P stores and
// loads over NVLink, or local memory for a rank's own block); no staging
// copy and no library collective sit on the data path.
//   dispatch  one warp per token: the token's distinct rows, each written
//             once into its destination rank's buffer with 16-byte stores,
//             with the token's global id and, per slot carried by the row,
//             the expert ID (-1 for slots of other ranks) and its gate; the
//             next token's row and slot data load while the current token's
//             rows are stored.
//   partials  on the receiver, one warp per received row: the gate-weighted
//             sum of its slots' expert outputs in ascending expert order,
//             fp32 FMA, one bf16 rounding -- the row that travels back.
//   combine   one warp per token: the bf16 partial rows of the token's
//             ranks, read from the peers in ascending rank, summed in fp32,
//             one bf16 rounding.
// The combine issues all of a token's return rows before it adds (a token
// has several), so about 8 16-byte loads per lane are in flight; the partials
// take the few slots of a received row one after another.
// No load or store here uses multicast; peers are plain pointers.
#include <climits>

#include "common.cuh"

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kU = 8;  // 16-byte chunks per lane in flight per pass over a row

struct PeerTable {
    md_peer_rows p[MD_MAX_RANKS];
};

// CTAs of kernel K (kThreads threads, no dynamic shared memory) resident per
// SM, queried once per device (8 if the query fails).  A grid of at most that
// many per SM runs in one wave: every CTA walks its share of the units from the
// start, with no second wave left to finish alone.  The dispatch (over 100
// registers, two CTAs per SM) gained from it (391 -> 374 us for the 16 calls
// of the E=128 exchange row); the partials and the combine, four CTAs per SM,
// did better with 8 CTAs per SM launched (783 against 833 us for the partials).
template <auto K>
int resident_per_sm()
{
    static std::atomic<uint64_t> done{0};
    static std::atomic<int> per[64];
    md::once_per_device(done, [] {
        int dev = 0, n = 0;
        cudaGetDevice(&dev);
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, K, kThreads, 0) != cudaSuccess || n < 1) {
            cudaGetLastError();
            n = 8;
        }
        per[dev & 63].store(n);
    });
    int dev = 0;
    cudaGetDevice(&dev);
    return per[dev & 63].load();
}

int grid_warps(int64_t units, int per_sm)
{
    int64_t b = (units + kWarps - 1) / kWarps;
    const int64_t cap = (int64_t)md::sm_count() * per_sm;
    if (b > cap) b = cap;
    return b < 1 ? 1 : (int)b;
}

// --------------------------------------------------------------- dispatch
// One warp per token, the vector permute's pipeline: a pass moves kU 16-byte
// chunks per lane (4 KiB of the row); while the current token's rows are
// stored, the next token's chunks and slot data are already in flight.  Rows
// longer than 4 KiB take one pass over the warp's tokens per 4 KiB block;
// the metadata is written in the first.
template <int KC>
__global__ void __launch_bounds__(kThreads)
    k_dispatch_exchange(const uint4 *__restrict__ x, int64_t T, int C, int k,
                        const int32_t *__restrict__ idx, const float *__restrict__ w,
                        const int32_t *__restrict__ p_g, int E, int R,
                        const int32_t *__restrict__ row_of_slot,
                        const int32_t *__restrict__ rank_offsets, int64_t token_base, PeerTable pt,
                        int32_t *status)
{
    const int K = KC ? KC : k;
    const int lane = threadIdx.x & 31;
    const int64_t w0 = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * kThreads) >> 5;
    if (w0 >= T) return;
    auto slot = [&](int64_t t, int &r, int &e, float &ww) {
        r = -1;
        e = -1;
        ww = 0.0f;
        if (t < T && lane < K) {
            r = __ldg(row_of_slot + t * K + lane);
            e = __ldg(idx + t * K + lane);
            ww = w ? __ldg(w + t * K + lane) : 0.0f;
        }
    };
    for (int c0 = 0; c0 < C; c0 += 32 * kU) {
        int64_t t = w0;
        uint4 cur[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int c = c0 + u * 32 + lane;
            if (c < C) cur[u] = md::ld_stream(x + t * C + c);
        }
        int r, e;
        float ww;
        slot(t, r, e, ww);
        for (; t < T; t += nw) {
            const int64_t tn = t + nw;
            uint4 nxt[kU];
            int rn, en;
            float wn;
            if (tn < T) {
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    const int c = c0 + u * 32 + lane;
                    if (c < C) nxt[u] = md::ld_stream(x + tn * C + c);
                }
            }
            slot(tn, rn, en, wn);
            int d = (lane < K && e >= 0 && e < E) ? __ldg(p_g + e) : -1;
            if (d >= R) d = -1;
            // slots sharing a row travel in it once; the row's slot mask is the group
            const unsigned g = __match_any_sync(0xffffffffu, lane < K ? (unsigned)r : (0x80000000u | lane));
            const bool first = lane < K && (g & md::lanemask_lt()) == 0u;
            int64_t dst = -1;
            if (first && d >= 0) {
                const int lo = __ldg(rank_offsets + d), hi = __ldg(rank_offsets + d + 1);
                if (r >= lo && r < hi) {
                    dst = pt.p[d].row_base + (r - lo);
                    if (dst < 0 || dst >= pt.p[d].rows_cap) dst = -1;
                }
            }
            if (first && dst < 0 && c0 == 0) md::report(status, MD_ERR_DATA);
            const unsigned rows = __ballot_sync(0xffffffffu, first && dst >= 0);
            unsigned todo = rows;
            while (todo) {
                const int j = __ffs(todo) - 1;
                todo &= todo - 1;
                const int dd = __shfl_sync(0xffffffffu, d, j);
                const int64_t drow = __shfl_sync(0xffffffffu, dst, j);
                uint4 *out = static_cast<uint4 *>(pt.p[dd].rows) + drow * C;
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    const int c = c0 + u * 32 + lane;
                    if (c < C) out[c] = cur[u];
                }
                if (c0 == 0) {  // metadata: global token id, expert and gate per slot
                    const unsigned gm = __shfl_sync(0xffffffffu, g, j);
                    const md_peer_rows &q = pt.p[dd];
                    if (lane == 0 && q.token) q.token[drow] = (int32_t)(token_base + t);
                    if (lane < K) {
                        const bool mine = (gm >> lane) & 1u;
                        if (q.slot_idx) q.slot_idx[drow * K + lane] = mine ? e : -1;
                        if (q.slot_w) q.slot_w[drow * K + lane] = mine ? ww : 0.0f;
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < kU; ++u) cur[u] = nxt[u];
            r = rn;
            e = en;
            ww = wn;
        }
    }
}

__device__ __forceinline__ void fma_row8(float (&acc)[8], float wt, const uint4 &v)
{
    acc[0] = fmaf(wt, md::bf16lo(v.x), acc[0]);
    acc[1] = fmaf(wt, md::bf16hi(v.x), acc[1]);
    acc[2] = fmaf(wt, md::bf16lo(v.y), acc[2]);
    acc[3] = fmaf(wt, md::bf16hi(v.y), acc[3]);
    acc[4] = fmaf(wt, md::bf16lo(v.z), acc[4]);
    acc[5] = fmaf(wt, md::bf16hi(v.z), acc[5]);
    acc[6] = fmaf(wt, md::bf16lo(v.w), acc[6]);
    acc[7] = fmaf(wt, md::bf16hi(v.w), acc[7]);
}

__device__ __forceinline__ void add_row8(float (&acc)[8], const uint4 &v)
{
    acc[0] += md::bf16lo(v.x);
    acc[1] += md::bf16hi(v.x);
    acc[2] += md::bf16lo(v.y);
    acc[3] += md::bf16hi(v.y);
    acc[4] += md::bf16lo(v.z);
    acc[5] += md::bf16hi(v.z);
    acc[6] += md::bf16lo(v.w);
    acc[7] += md::bf16hi(v.w);
}

__device__ __forceinline__ uint4 pack8(const float (&a)[8])
{
    return make_uint4(md::pack_bf16x2(a[0], a[1]), md::pack_bf16x2(a[2], a[3]),
                      md::pack_bf16x2(a[4], a[5]), md::pack_bf16x2(a[6], a[7]));
}

// Place of this lane's key among the live lanes (< n) in ascending order,
// ties by lane: 0 for the smallest.
__device__ __forceinline__ int rank_among(bool live, int key, int n)
{
    const int lane = threadIdx.x & 31;
    const unsigned lv = __ballot_sync(0xffffffffu, live);
    int rank = 0;
    for (int j = 0; j < n; ++j) {
        const int kj = __shfl_sync(0xffffffffu, key, j);
        rank += (((lv >> j) & 1u) && (kj < key || (kj == key && j < lane))) ? 1 : 0;
    }
    return rank;
}

// --------------------------------------------------------------- partials
// z[i] = bf16(sum over slots j carried by received row i, ascending expert,
// of slot_w[i][j] * y[y_row[i][j]]), fp32 FMA from +0.0f.  A received dedup
// row carries few slots (k / rows per token, about 1.2 for top-8 over 16
// ranks), so the warp takes them one after another, 4 16-byte chunks per
// lane of each at a time (8 measured slower: twice the registers, half the
// resident warps; so did a compile-time k, 930 against 780 us).
__global__ void __launch_bounds__(kThreads)
    k_combine_partials(const uint4 *__restrict__ y, int64_t y_rows, const int32_t *__restrict__ y_row,
                       const int32_t *__restrict__ slot_idx, const float *__restrict__ slot_w,
                       int64_t n, int k, int C, uint4 *__restrict__ z, int32_t *status)
{
    constexpr int U = 4;
    const int K = k;
    const int lane = threadIdx.x & 31;
    const int64_t nw = ((int64_t)gridDim.x * kThreads) >> 5;
    for (int64_t i = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5; i < n; i += nw) {
        int yr = -1, e = INT_MAX;
        float ww = 0.0f;
        if (lane < K) {
            yr = __ldg(y_row + i * K + lane);
            e = __ldg(slot_idx + i * K + lane);
            ww = __ldg(slot_w + i * K + lane);
            if (yr >= y_rows) {
                md::report(status, MD_ERR_DATA);
                yr = -1;
            }
        }
        const bool live = yr >= 0;
        const int nv = __popc(__ballot_sync(0xffffffffu, live));
        const int rank = rank_among(live, e, K);
        for (int c0 = 0; c0 < C; c0 += 32 * U) {
            float acc[U][8];
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int q = 0; q < 8; ++q) acc[u][q] = 0.0f;
            for (int q = 0; q < nv; ++q) {
                const int j = __ffs(__ballot_sync(0xffffffffu, live && rank == q)) - 1;
                const int64_t r = __shfl_sync(0xffffffffu, yr, j);
                const float wt = __shfl_sync(0xffffffffu, ww, j);
                uint4 v[U];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int c = c0 + u * 32 + lane;
                    v[u] = c < C ? md::ld_stream(y + r * C + c) : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int u = 0; u < U; ++u) fma_row8(acc[u], wt, v[u]);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int c = c0 + u * 32 + lane;
                if (c < C) md::st_stream(z + i * C + c, pack8(acc[u]));
            }
        }
    }
}

// ---------------------------------------------------------------- combine
// out[t] = bf16(fp32 sum over t's distinct rows, in ascending destination
// rank, of the bf16 return row held by that rank).  With a compile-time k the
// warp issues the loads of all the token's return rows before the adds.
template <int KC>
__global__ void __launch_bounds__(kThreads)
    k_combine_exchange(int64_t T, int C, int k, const int32_t *__restrict__ idx,
                       const int32_t *__restrict__ p_g, int E, int R,
                       const int32_t *__restrict__ row_of_slot,
                       const int32_t *__restrict__ rank_offsets, PeerTable pt,
                       uint4 *__restrict__ out, int32_t *status)
{
    constexpr int KB = KC ? KC : 1;
    constexpr int U = KC ? (KC >= 8 ? 1 : 8 / KC) : 4;
    const int K = KC ? KC : k;
    const int lane = threadIdx.x & 31;
    const int64_t nw = ((int64_t)gridDim.x * kThreads) >> 5;
    for (int64_t t = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5; t < T; t += nw) {
        int r = -1, d = -1;
        if (lane < K) {
            r = __ldg(row_of_slot + t * K + lane);
            const int e = __ldg(idx + t * K + lane);
            d = (e >= 0 && e < E) ? __ldg(p_g + e) : -1;
            if (d >= R) d = -1;
        }
        const unsigned g = __match_any_sync(0xffffffffu, lane < K ? (unsigned)r : (0x80000000u | lane));
        const bool first = lane < K && (g & md::lanemask_lt()) == 0u;
        int64_t src = -1;
        if (first && d >= 0) {
            const int lo = __ldg(rank_offsets + d), hi = __ldg(rank_offsets + d + 1);
            if (r >= lo && r < hi) {
                src = pt.p[d].row_base + (r - lo);
                if (src < 0 || src >= pt.p[d].rows_cap) src = -1;
            }
        }
        if (first && src < 0) md::report(status, MD_ERR_DATA);
        const bool live = first && src >= 0;
        const int nv = __popc(__ballot_sync(0xffffffffu, live));
        const int rank = rank_among(live, d, K);
        // the token's return rows in ascending rank
        const uint4 *zr[KB];
#pragma unroll
        for (int q = 0; q < KB; ++q) {
            const unsigned bal = KC ? __ballot_sync(0xffffffffu, live && rank == q) : 0u;
            const int j = bal ? __ffs(bal) - 1 : 0;
            const int dd = __shfl_sync(0xffffffffu, d, j);
            const int64_t sr = __shfl_sync(0xffffffffu, src, j);
            zr[q] = bal ? static_cast<const uint4 *>(pt.p[dd].rows) + sr * C : nullptr;
        }
        for (int c0 = 0; c0 < C; c0 += 32 * U) {
            float acc[U][8];
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int q = 0; q < 8; ++q) acc[u][q] = 0.0f;
            if (KC) {
                uint4 v[KB][U];
#pragma unroll
                for (int q = 0; q < KB; ++q)
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const int c = c0 + u * 32 + lane;
                        v[q][u] = (zr[q] && c < C) ? __ldcg(zr[q] + c) : make_uint4(0, 0, 0, 0);
                    }
#pragma unroll
                for (int q = 0; q < KB; ++q)
                    if (zr[q]) {
#pragma unroll
                        for (int u = 0; u < U; ++u) add_row8(acc[u], v[q][u]);
                    }
            } else {
                for (int q = 0; q < nv; ++q) {
                    const int j = __ffs(__ballot_sync(0xffffffffu, live && rank == q)) - 1;
                    const int dd = __shfl_sync(0xffffffffu, d, j);
                    const int64_t sr = __shfl_sync(0xffffffffu, src, j);
                    const uint4 *row = static_cast<const uint4 *>(pt.p[dd].rows) + sr * C;
                    uint4 v[U];
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const int c = c0 + u * 32 + lane;
                        v[u] = c < C ? __ldcg(row + c) : make_uint4(0, 0, 0, 0);
                    }
#pragma unroll
                    for (int u = 0; u < U; ++u) add_row8(acc[u], v[u]);
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int c = c0 + u * 32 + lane;
                if (c < C) md::st_stream(out + t * C + c, pack8(acc[u]));
            }
        }
    }
}

int load_peers(const md_peer_rows *peers, int R, int H, bool need_rows, PeerTable *pt)
{
    if (!peers) return MD_ERR_ARG;
    for (int d = 0; d < R; ++d) {
        const md_peer_rows &q = peers[d];
        if (q.rows_cap < 0 || q.row_base < 0) return MD_ERR_ARG;
        if (q.rows_cap > 0 && need_rows && (!q.rows || !md::aligned16(q.rows))) return MD_ERR_ARG;
        pt->p[d] = q;
    }
    for (int d = R; d < MD_MAX_RANKS; ++d) pt->p[d] = md_peer_rows{};
    (void)H;
    return MD_OK;
}

int check_common(int64_t T, int H, int k, int E, int R)
{
    if (T < 0 || H < 8 || H % 8 != 0 || k < 1 || k > MD_MAX_TOPK || k > E || R < 1) return MD_ERR_ARG;
    if (E > MD_MAX_EXPERTS || R > MD_MAX_RANKS) return MD_ERR_UNSUPPORTED;
    return MD_OK;
}

}  // namespace

extern "C" int md_exchange_plan(const int64_t *src_rank_offsets, int R, int me,
                                int64_t *dst_row_base, int64_t *recv_offsets)
{
    if (!src_rank_offsets || !dst_row_base || !recv_offsets || R < 1 || R > MD_MAX_RANKS ||
        me < 0 || me >= R)
        return MD_ERR_ARG;
    // source s sends S[s][d] = its rank_offsets[d+1] - rank_offsets[d] rows to d
    auto S = [&](int s, int d) {
        return src_rank_offsets[(int64_t)s * (R + 1) + d + 1] - src_rank_offsets[(int64_t)s * (R + 1) + d];
    };
    for (int s = 0; s < R; ++s) {
        if (src_rank_offsets[(int64_t)s * (R + 1)] != 0) return MD_ERR_DATA;
        for (int d = 0; d < R; ++d)
            if (S(s, d) < 0) return MD_ERR_DATA;
    }
    // first row of my block on destination d: the rows of sources before me
    for (int d = 0; d < R; ++d) {
        int64_t base = 0;
        for (int s = 0; s < me; ++s) base += S(s, d);
        dst_row_base[d] = base;
    }
    // blocks of my receive buffer, one per source in order
    int64_t run = 0;
    for (int s = 0; s < R; ++s) {
        recv_offsets[s] = run;
        run += S(s, me);
    }
    recv_offsets[R] = run;
    return MD_OK;
}

extern "C" int md_dispatch_exchange(const void *x, int64_t T, int H, int k, const int32_t *topk_idx,
                                    const float *topk_w, const int32_t *expert_to_rank, int E, int R,
                                    const int32_t *row_of_slot, const int32_t *rank_offsets,
                                    int64_t token_base, const md_peer_rows *peers,
                                    int32_t *dev_status, void *stream)
{
    int rc = check_common(T, H, k, E, R);
    if (rc != MD_OK) return rc;
    if (T > 0 && (!x || !md::aligned16(x) || !topk_idx || !expert_to_rank || !row_of_slot ||
                  !rank_offsets))
        return MD_ERR_ARG;
    if (token_base < 0 || token_base + T > INT32_MAX) return MD_ERR_ARG;
    PeerTable pt;
    if ((rc = load_peers(peers, R, H, true, &pt)) != MD_OK) return rc;
    cudaStream_t s = md::as_stream(stream);
    if ((rc = md::clear_status(dev_status, s)) != MD_OK || T == 0) return rc;
    const int C = H / 8;
#define MD_DX(KC)                                                                                  \
    k_dispatch_exchange<KC><<<(unsigned)grid_warps(T, resident_per_sm<k_dispatch_exchange<KC>>()),  \
                              kThreads, 0, s>>>(                                                    \
        static_cast<const uint4 *>(x), T, C, k, topk_idx, topk_w, expert_to_rank, E, R, row_of_slot, \
        rank_offsets, token_base, pt, dev_status)
    switch (k) {
    case 2: MD_DX(2); break;
    case 4: MD_DX(4); break;
    case 6: MD_DX(6); break;
    case 8: MD_DX(8); break;
    default: MD_DX(0); break;
    }
#undef MD_DX
    md::count_launches(1);
    return md::launch_status();
}

extern "C" int md_combine_partials(const void *y, int64_t y_rows, const int32_t *y_row,
                                   const int32_t *slot_idx, const float *slot_w, int64_t n, int k,
                                   int H, void *z, int32_t *dev_status, void *stream)
{
    if (n < 0 || y_rows < 0 || H < 8 || H % 8 != 0 || k < 1 || k > MD_MAX_TOPK) return MD_ERR_ARG;
    if (n > 0 && (!y_row || !slot_idx || !slot_w || !z || !md::aligned16(z))) return MD_ERR_ARG;
    if (y_rows > 0 && (!y || !md::aligned16(y))) return MD_ERR_ARG;
    cudaStream_t s = md::as_stream(stream);
    int rc = md::clear_status(dev_status, s);
    if (rc != MD_OK || n == 0) return rc;
    k_combine_partials<<<(unsigned)grid_warps(n, 8), kThreads, 0, s>>>(
        static_cast<const uint4 *>(y), y_rows, y_row, slot_idx, slot_w, n, k, H / 8,
        static_cast<uint4 *>(z), dev_status);
    md::count_launches(1);
    return md::launch_status();
}

extern "C" int md_combine_exchange(const md_peer_rows *peers, int64_t T, int H, int k,
                                   const int32_t *topk_idx, const int32_t *expert_to_rank, int E,
                                   int R, const int32_t *row_of_slot, const int32_t *rank_offsets,
                                   void *out, int32_t *dev_status, void *stream)
{
    int rc = check_common(T, H, k, E, R);
    if (rc != MD_OK) return rc;
    if (T > 0 && (!out || !md::aligned16(out) || !topk_idx || !expert_to_rank || !row_of_slot ||
                  !rank_offsets))
        return MD_ERR_ARG;
    PeerTable pt;
    if ((rc = load_peers(peers, R, H, true, &pt)) != MD_OK) return rc;
    cudaStream_t s = md::as_stream(stream);
    if ((rc = md::clear_status(dev_status, s)) != MD_OK || T == 0) return rc;
    const int C = H / 8;
#define MD_CX(KC)                                                                                  \
    k_combine_exchange<KC><<<(unsigned)grid_warps(T, 8), kThreads, 0, s>>>(                        \
        T, C, k, topk_idx, expert_to_rank, E, R, row_of_slot, rank_offsets, pt,                     \
        static_cast<uint4 *>(out), dev_status)
    switch (k) {
    case 2: MD_CX(2); break;
    case 4: MD_CX(4); break;
    case 6: MD_CX(6); break;
    case 8: MD_CX(8); break;
    default: MD_CX(0); break;
    }
#undef MD_CX
    md::count_launches(1);
    return md::launch_status();
}
