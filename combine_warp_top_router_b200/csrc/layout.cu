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
// rows by (d, t).  Two kernels:
//   k_layout_hist  per-bucket totals (expert counts, send matrix) with
//                  shared-memory histograms; the last block to finish turns
//                  them into bucket bases, offsets and n_rows.
//   k_layout_rank  one tile of tokens per CTA (tile order from an atomic
//                  ticket).  Each warp ranks its run of (t, j) pairs with
//                  __match_any_sync; the CTA publishes its per-bucket counts
//                  and finds the counts of all earlier tiles by a single-pass
//                  decoupled lookback (bounded waits), then writes positions.
#include "common.cuh"

namespace {

constexpr int kHistThreads = 512;
constexpr int kHistTok = 1024;
constexpr int kRankThreads = 256;
constexpr int kRankWarps = kRankThreads / 32;
constexpr unsigned long long kFlagA = 1ull << 62;  // tile aggregate published
constexpr unsigned long long kFlagP = 2ull << 62;  // tile inclusive prefix published
constexpr unsigned long long kValMask = (1ull << 62) - 1;
constexpr int kLookWindow = 8;
constexpr long long kPollLimit = 1ll << 22;

struct Ws {
    unsigned int *ctrl;           // [0] finished hist blocks, [1] rank tile ticket
    int *hist_e;                  // [E]   assignments per expert
    int *send;                    // [R*R] rows per (source, destination)
    unsigned long long *tiles;    // [n_tiles * NB] lookback words
    int *base;                    // [E + R] first row of each bucket
};

int tile_tokens(int k)
{
    int t = 2048 / k, p = 1;
    while (p * 2 <= t) p *= 2;
    return p < 64 ? 64 : (p > 2048 ? 2048 : p);
}

struct Plan {
    size_t off_hist, off_send, off_tiles, off_base, zero_bytes, total;
    int tile_tok, n_tiles, nb;
};

Plan plan(int64_t T, int E, int k, int R, int mode)
{
    Plan p;
    p.tile_tok = tile_tokens(k);
    p.n_tiles = (int)((T + p.tile_tok - 1) / p.tile_tok);
    p.nb = E + (mode == MD_DEDUP ? R : 0);
    size_t o = 256;
    p.off_hist = o;
    o += md::align_up((size_t)E * 4, 256);
    p.off_send = o;
    o += md::align_up((size_t)R * R * 4, 256);
    p.off_tiles = o;
    o += md::align_up((size_t)p.n_tiles * p.nb * 8, 256);
    p.zero_bytes = o;
    p.off_base = o;
    o += md::align_up((size_t)(E + R) * 4, 256);
    p.total = o;
    return p;
}

Ws carve(void *ws, const Plan &p)
{
    char *b = static_cast<char *>(ws);
    Ws w;
    w.ctrl = reinterpret_cast<unsigned int *>(b);
    w.hist_e = reinterpret_cast<int *>(b + p.off_hist);
    w.send = reinterpret_cast<int *>(b + p.off_send);
    w.tiles = reinterpret_cast<unsigned long long *>(b + p.off_tiles);
    w.base = reinterpret_cast<int *>(b + p.off_base);
    return w;
}

// Is slot j of token row `row` the first slot of that token on rank d?
__device__ __forceinline__ bool first_on_rank(const int32_t *row, int j, int d, const int *s_p,
                                              int E)
{
    for (int j2 = 0; j2 < j; ++j2) {
        int e2 = row[j2];
        if (e2 >= 0 && e2 < E && s_p[e2] == d) return false;
    }
    return true;
}

__global__ void __launch_bounds__(kHistThreads)
    k_layout_hist(const int32_t *__restrict__ idx, int64_t T, int E, int k, int R,
                  const int32_t *__restrict__ p_g, int mode, Ws ws, int32_t *expert_counts,
                  int32_t *send_counts, int32_t *expert_offsets, int32_t *rank_offsets,
                  int32_t *n_rows, int32_t *status)
{
    extern __shared__ int smem[];
    int *s_p = smem;           // [E]
    int *s_hist = s_p + E;     // [E]
    int *s_send = s_hist + E;  // [R*R]
    __shared__ int s_last;
    __shared__ int s_rt[2][MD_MAX_RANKS + 1];  // rank totals: conventional, this mode

    const int tid = threadIdx.x;
    for (int e = tid; e < E; e += blockDim.x) {
        s_p[e] = p_g[e];
        s_hist[e] = 0;
    }
    for (int i = tid; i < R * R; i += blockDim.x) s_send[i] = 0;
    __syncthreads();

    const int64_t Tr = T / R;
    const int64_t t0 = (int64_t)blockIdx.x * kHistTok;
    const int64_t t1 = t0 + kHistTok < T ? t0 + kHistTok : T;
    for (int64_t f = t0 * k + tid; f < t1 * k; f += blockDim.x) {
        const int64_t t = f / k;
        const int j = (int)(f - t * k);
        const int e = idx[f];
        if (e < 0 || e >= E) { md::report(status, MD_ERR_DATA); continue; }
        const int d = s_p[e];
        if (d < 0 || d >= R) { md::report(status, MD_ERR_DATA); continue; }
        const int32_t *row = idx + t * k;
        bool rep = true;
        for (int j2 = 0; j2 < j; ++j2) {
            const int e2 = __ldg(row + j2);
            if (e2 == e) md::report(status, MD_ERR_DATA);  // expert twice in one token
            if (e2 >= 0 && e2 < E && s_p[e2] == d) rep = false;
        }
        atomicAdd(&s_hist[e], 1);
        if (mode == MD_CONV || rep) atomicAdd(&s_send[(int)(t / Tr) * R + d], 1);
    }
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x)
        if (s_hist[e]) atomicAdd(&ws.hist_e[e], s_hist[e]);
    for (int i = tid; i < R * R; i += blockDim.x)
        if (s_send[i]) atomicAdd(&ws.send[i], s_send[i]);
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(&ws.ctrl[0], 1u) == gridDim.x - 1;
    __syncthreads();
    if (!s_last) return;

    // ---- last block: totals -> bases, offsets, counts
    __threadfence();
    for (int e = tid; e < E; e += blockDim.x) s_hist[e] = __ldcg(&ws.hist_e[e]);
    for (int i = tid; i < R * R; i += blockDim.x) s_send[i] = __ldcg(&ws.send[i]);
    for (int i = tid; i < 2 * (MD_MAX_RANKS + 1); i += blockDim.x) (&s_rt[0][0])[i] = 0;
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x) {
        const int d = s_p[e];
        if (d >= 0 && d < R) {
            atomicAdd(&s_rt[0][d], s_hist[e]);
        } else {
            md::report(status, MD_ERR_DATA);
        }
        expert_counts[e] = s_hist[e];
    }
    for (int i = tid; i < R * R; i += blockDim.x) send_counts[i] = s_send[i];
    if (mode == MD_DEDUP)
        for (int d = tid; d < R; d += blockDim.x) {
            int s = 0;
            for (int src = 0; src < R; ++src) s += s_send[src * R + d];
            s_rt[1][d] = s;
        }
    __syncthreads();
    if (tid == 0) {
        // placement must give every rank E/R experts
        int cnt[MD_MAX_RANKS];
        for (int d = 0; d < R; ++d) cnt[d] = 0;
        for (int e = 0; e < E; ++e)
            if (s_p[e] >= 0 && s_p[e] < R) cnt[s_p[e]] += 1;
        for (int d = 0; d < R; ++d)
            if (cnt[d] != E / R) md::report(status, MD_ERR_DATA);
        // exclusive scans over ranks (in place)
        for (int m = 0; m < 2; ++m) {
            int run = 0;
            for (int d = 0; d < R; ++d) {
                int c = s_rt[m][d];
                s_rt[m][d] = run;
                run += c;
            }
            s_rt[m][R] = run;
        }
        if (mode == MD_CONV)
            for (int d = 0; d <= R; ++d) s_rt[1][d] = s_rt[0][d];
    }
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x) {
        const int d = s_p[e];
        int b = 0;
        if (d >= 0 && d < R) {
            b = s_rt[0][d];
            for (int e2 = 0; e2 < e; ++e2)
                if (s_p[e2] == d) b += s_hist[e2];
        }
        expert_offsets[e] = b;
        ws.base[e] = b;
    }
    for (int d = tid; d <= R; d += blockDim.x) {
        rank_offsets[d] = s_rt[1][d];
        if (d < R) ws.base[E + d] = s_rt[1][d];
    }
    if (tid == 0) {
        expert_offsets[E] = s_rt[0][R];
        *n_rows = s_rt[1][R];
    }
}

__global__ void __launch_bounds__(kRankThreads)
    k_layout_rank(const int32_t *__restrict__ idx, int64_t T, int E, int k, int R,
                  const int32_t *__restrict__ p_g, int mode, int tile_tok, Ws ws,
                  int32_t *__restrict__ row_of_slot, int32_t *__restrict__ assign_row,
                  int32_t *__restrict__ row_token, uint32_t *__restrict__ row_mask,
                  int64_t row_cap, int32_t *status)
{
    extern __shared__ int smem[];
    const int NB = E + (mode == MD_DEDUP ? R : 0);
    const int P = tile_tok * k;
    int *s_p = smem;                   // [E]
    int *s_idx = s_p + E;              // [P]  the tile's experts, pair order
    int *s_loc = s_idx + P;            // [P]  rank within the warp run, expert bucket
    int *s_aux = s_loc + P;            // [P]  same for the rank bucket; then the wire row
    int *s_cnt = s_aux + P;            // [8][NB] per-warp counts, then exclusive prefix
    int *s_pref = s_cnt + kRankWarps * NB;  // [NB] tile total, then first row of the tile
    __shared__ int s_tile, s_timeout;

    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    if (tid == 0) {
        s_tile = (int)atomicAdd(&ws.ctrl[1], 1u);
        s_timeout = 0;
    }
    for (int e = tid; e < E; e += kRankThreads) s_p[e] = p_g[e];
    for (int i = tid; i < kRankWarps * NB; i += kRankThreads) s_cnt[i] = 0;
    __syncthreads();
    const int tile = s_tile;
    const int64_t t0 = (int64_t)tile * tile_tok;
    const int ntok = (int)(T - t0 < tile_tok ? T - t0 : tile_tok);
    const int np = ntok * k;
    for (int i = tid; i < P; i += kRankThreads) s_idx[i] = i < np ? idx[t0 * k + i] : -1;
    __syncthreads();

    // ---- rank each pair within its warp's run of the tile
    const int seg = P / kRankWarps;
    const int f_end = (w + 1) * seg;
    for (int c0 = w * seg; c0 < f_end; c0 += 32) {
        const int f = c0 + lane;
        const int e = (f < f_end && f < np) ? s_idx[f] : -1;
        const int d = (e >= 0 && e < E) ? s_p[e] : -1;
        const bool valid = e >= 0 && e < E && d >= 0 && d < R;
        const unsigned g = __match_any_sync(0xffffffffu, valid ? (unsigned)e : (0x80000000u | lane));
        const int cb = valid ? s_cnt[w * NB + e] : 0;
        if (valid) s_loc[f] = cb + __popc(g & md::lanemask_lt());
        bool rep = false;
        unsigned gd = 0;
        int cbd = 0;
        if (mode == MD_DEDUP) {
            if (valid) {
                const int tl = f / k;
                rep = first_on_rank(s_idx + tl * k, f - tl * k, d, s_p, E);
            }
            gd = __match_any_sync(0xffffffffu, rep ? (unsigned)d : (0x80000000u | lane));
            cbd = rep ? s_cnt[w * NB + E + d] : 0;
            if (rep) s_aux[f] = cbd + __popc(gd & md::lanemask_lt());
        }
        __syncwarp();
        if (valid && (g >> lane) == 1u) s_cnt[w * NB + e] = cb + __popc(g);
        if (rep && (gd >> lane) == 1u) s_cnt[w * NB + E + d] = cbd + __popc(gd);
        __syncwarp();
    }
    __syncthreads();

    // ---- per-bucket tile totals; exclusive prefix over the warps
    for (int b = tid; b < NB; b += kRankThreads) {
        int run = 0;
        for (int w2 = 0; w2 < kRankWarps; ++w2) {
            const int c = s_cnt[w2 * NB + b];
            s_cnt[w2 * NB + b] = run;
            run += c;
        }
        s_pref[b] = run;
    }
    __syncthreads();

    // ---- publish, then decoupled lookback over earlier tiles
    unsigned long long *mine = ws.tiles + (size_t)tile * NB;
    for (int b = tid; b < NB; b += kRankThreads)
        md::st_relaxed_u64(mine + b, (tile == 0 ? kFlagP : kFlagA) | (unsigned long long)s_pref[b]);
    for (int b = tid; b < NB; b += kRankThreads) {
        const int total = s_pref[b];
        long long excl = 0;
        if (tile > 0) {
            int j = tile - 1;
            bool done = false;
            long long polls = 0;
            while (!done) {
                unsigned long long v[kLookWindow];
#pragma unroll
                for (int q = 0; q < kLookWindow; ++q)
                    v[q] = (j - q >= 0) ? md::ld_relaxed_u64(ws.tiles + (size_t)(j - q) * NB + b)
                                        : kFlagP;
#pragma unroll
                for (int q = 0; q < kLookWindow; ++q) {
                    if (done) break;
                    unsigned long long x = v[q];
                    while ((x >> 62) == 0ull) {  // not published yet: bounded wait
                        if (++polls > kPollLimit) {
                            md::report(status, MD_ERR_TIMEOUT);
                            s_timeout = 1;
                            x = kFlagP;
                            break;
                        }
                        __nanosleep(64);
                        x = md::ld_relaxed_u64(ws.tiles + (size_t)(j - q) * NB + b);
                    }
                    excl += (long long)(x & kValMask);
                    if ((x >> 62) == 2ull) done = true;
                }
                j -= kLookWindow;
            }
            md::st_relaxed_u64(mine + b, kFlagP | (unsigned long long)(excl + total));
        }
        s_pref[b] = ws.base[b] + (int)excl;
    }
    __syncthreads();
    if (s_timeout) return;  // positions unknown: leave outputs, status says why

    // ---- positions
    for (int f = tid; f < np; f += kRankThreads) {
        const int tl = f / k, j = f - tl * k;
        const int64_t t = t0 + tl;
        const int e = s_idx[f];
        const int d = (e >= 0 && e < E) ? s_p[e] : -1;
        if (!(e >= 0 && e < E && d >= 0 && d < R)) {
            assign_row[t * k + j] = -1;
            row_of_slot[t * k + j] = -1;
            continue;
        }
        const int wf = f / seg;
        const int pos = s_pref[e] + s_cnt[wf * NB + e] + s_loc[f];
        assign_row[t * k + j] = pos;
        if (mode == MD_CONV) {
            row_of_slot[t * k + j] = pos;
            if (pos >= 0 && pos < row_cap) {
                row_token[pos] = (int32_t)t;
                row_mask[pos] = 1u << j;
            } else {
                md::report(status, MD_ERR_DATA);
            }
        } else if (first_on_rank(s_idx + tl * k, j, d, s_p, E)) {
            const int pw = s_pref[E + d] + s_cnt[wf * NB + E + d] + s_aux[f];
            s_aux[f] = pw;
            uint32_t mask = 0;
            for (int j2 = 0; j2 < k; ++j2) {
                const int e2 = s_idx[tl * k + j2];
                if (e2 >= 0 && e2 < E && s_p[e2] == d) mask |= 1u << j2;
            }
            if (pw >= 0 && pw < row_cap) {
                row_token[pw] = (int32_t)t;
                row_mask[pw] = mask;
            } else {
                md::report(status, MD_ERR_DATA);
            }
        }
    }
    if (mode == MD_DEDUP) {
        __syncthreads();
        for (int f = tid; f < np; f += kRankThreads) {
            const int tl = f / k, j = f - tl * k;
            const int e = s_idx[f];
            const int d = (e >= 0 && e < E) ? s_p[e] : -1;
            if (!(e >= 0 && e < E && d >= 0 && d < R)) continue;
            int jr = 0;
            while (jr < j) {
                const int e2 = s_idx[tl * k + jr];
                if (e2 >= 0 && e2 < E && s_p[e2] == d) break;
                ++jr;
            }
            row_of_slot[(t0 + tl) * k + j] = s_aux[tl * k + jr];
        }
    }
}

size_t rank_smem(int E, int k, int R, int mode)
{
    const int P = tile_tokens(k) * k;
    const int NB = E + (mode == MD_DEDUP ? R : 0);
    return (size_t)(E + 3 * P + (kRankWarps + 1) * NB) * sizeof(int);
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

    static bool attr_set = false;
    if (!attr_set) {
        cudaFuncSetAttribute(k_layout_rank, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             160 * 1024);
        attr_set = true;
    }
    if ((rc = md::clear_status(dev_status, s)) != MD_OK) return rc;
    md::count_launches(1);
    if (cudaMemsetAsync(workspace, 0, pl.zero_bytes, s) != cudaSuccess) return MD_ERR_CUDA;

    const int hist_blocks = T > 0 ? (int)((T + kHistTok - 1) / kHistTok) : 1;
    const size_t hsm = (size_t)(2 * E + R * R) * sizeof(int);
    k_layout_hist<<<hist_blocks, kHistThreads, hsm, s>>>(topk_idx, T, E, k, R, expert_to_rank, mode,
                                                         ws, expert_counts, send_counts,
                                                         expert_offsets, rank_offsets, n_rows,
                                                         dev_status);
    md::count_launches(1);
    if ((rc = md::launch_status()) != MD_OK) return rc;
    if (T == 0) return MD_OK;
    const int64_t cap = mode == MD_CONV ? T * k : T * (int64_t)(k < R ? k : R);
    k_layout_rank<<<pl.n_tiles, kRankThreads, rank_smem(E, k, R, mode), s>>>(
        topk_idx, T, E, k, R, expert_to_rank, mode, pl.tile_tok, ws, row_of_slot, assign_row,
        row_token, row_mask, cap, dev_status);
    md::count_launches(1);
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
