// movement.cu -- row movement on HBM: dispatch permute, combine, row gather
// (md_dispatch_permute, md_combine, md_gather_rows).
//
// All three are bound by HBM bandwidth and move rows as 16-byte vectors, so
// every warp instruction reads or writes 512 contiguous bytes of a row.
//   permute  rows of 1 KiB and more: TMA bulk copies through a per-warp
//            ring of shared-memory slots (one bulk load per row piece, one
//            bulk store per destination row).  Shorter rows: one warp per
//            token, 16-byte vectors, the next token's x row and row indices
//            loaded while the current token's stores drain.
//   combine  a CTA takes kGroup tokens at a time: one warp per token orders
//            its slots and stages (row, gate) in shared memory, then each
//            thread issues the k 16-byte loads of its column chunk before the
//            FMAs, so k loads per thread are in flight.
//   gather   one 16-byte (or 4-byte) chunk per thread, grid-stride.
// Grids are sized from the SM count and loop over their work.
#include <climits>

#include "common.cuh"

namespace {

constexpr int kThreads = 256;
constexpr int kGroup = 8;  // tokens per CTA iteration: one of the 8 warps sorts each token's slots

int grid_for(int64_t units, int per_block)
{
    int64_t b = (units + per_block - 1) / per_block;
    const int64_t cap = (int64_t)md::sm_count() * 8;
    if (b > cap) b = cap;
    return b < 1 ? 1 : (int)b;
}

// ----------------------------------------------------------------- permute
// out[row_of_slot[t][j]] = x[t] for every distinct row of token t.
// One warp per token, no block barriers.  A pass moves kPermU 16-byte chunks
// per lane (4 KiB per warp); while the stores of token t drain, the x chunks
// and row indices of the warp's next token are already in flight.
constexpr int kPermU = 8;

template <int KC>
__global__ void __launch_bounds__(kThreads)
    k_permute(const uint4 *__restrict__ x, int64_t T, int C, int k,
              const int32_t *__restrict__ row_of_slot, int64_t out_rows, uint4 *__restrict__ out,
              int32_t *status)
{
    const int K = KC ? KC : k;
    const int lane = threadIdx.x & 31;
    const int64_t w0 = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * kThreads) >> 5;
    if (w0 >= T) return;
    for (int c0 = 0; c0 < C; c0 += 32 * kPermU) {
        int64_t t = w0;
        uint4 cur[kPermU];
        int rows = -1;
#pragma unroll
        for (int u = 0; u < kPermU; ++u) {
            const int c = c0 + u * 32 + lane;
            if (c < C) cur[u] = md::ld_stream(x + t * C + c);
        }
        if (lane < K) rows = __ldg(row_of_slot + t * K + lane);
        for (; t < T; t += nw) {
            const int64_t tn = t + nw;
            uint4 nxt[kPermU];
            int nrows = -1;
            if (tn < T) {
#pragma unroll
                for (int u = 0; u < kPermU; ++u) {
                    const int c = c0 + u * 32 + lane;
                    if (c < C) nxt[u] = md::ld_stream(x + tn * C + c);
                }
                if (lane < K) nrows = __ldg(row_of_slot + tn * K + lane);
            }
            // distinct, in-range rows of this token (slots sharing a row write once)
            const unsigned g = __match_any_sync(0xffffffffu, lane < K ? (unsigned)rows : (0x80000000u | lane));
            const bool first = lane < K && (g & md::lanemask_lt()) == 0u;
            const bool ok = rows >= 0 && rows < out_rows;
            if (first && !ok && c0 == 0) md::report(status, MD_ERR_DATA);
            unsigned todo = __ballot_sync(0xffffffffu, first && ok);
            while (todo) {
                const int j = __ffs(todo) - 1;
                todo &= todo - 1;
                const int64_t r = __shfl_sync(0xffffffffu, rows, j);
                uint4 *dst = out + r * C;
#pragma unroll
                for (int u = 0; u < kPermU; ++u) {
                    const int c = c0 + u * 32 + lane;
                    if (c < C) md::st_stream(dst + c, cur[u]);
                }
            }
#pragma unroll
            for (int u = 0; u < kPermU; ++u) cur[u] = nxt[u];
            rows = nrows;
        }
    }
}

// Rows of 1 KiB and more move by TMA bulk copies instead: each warp runs its
// own ring of kTmaStages 4 KiB shared-memory slots.  Lane 0 loads a piece of
// x (up to 4 KiB of one row) into a slot with one bulk copy, kTmaAhead pieces
// ahead, and writes it to each distinct destination row with one bulk store
// per row; the other lanes resolve the token's distinct rows.  A slot is
// reloaded only after the stores that read it have finished reading.
constexpr int kTmaWarps = 4;
constexpr int kTmaStages = 4;
constexpr int kTmaAhead = 2;
constexpr int kTmaPiece = 4096;
constexpr int kTmaMinRowBytes = 1024;
constexpr long long kTmaPolls = 1ll << 22;
static_assert(kTmaAhead >= 1 && kTmaAhead < kTmaStages, "ring: loads ahead < stages");

template <int KC>
__global__ void __launch_bounds__(kTmaWarps * 32)
    k_permute_tma(const char *__restrict__ x, int64_t T, int rowbytes, int pieces, int k,
                  const int32_t *__restrict__ row_of_slot, int64_t out_rows, char *__restrict__ out,
                  int32_t *status)
{
    extern __shared__ __align__(128) unsigned char tma_ring[];
    __shared__ uint64_t bars[kTmaWarps][kTmaStages];
    const int K = KC ? KC : k;
    const int lane = threadIdx.x & 31, wl = threadIdx.x >> 5;
    unsigned char *ring = tma_ring + (size_t)wl * kTmaStages * kTmaPiece;
    uint64_t *bar = bars[wl];
    const int64_t U = T * pieces;  // units: (token, piece)
    const int64_t gw = (int64_t)blockIdx.x * kTmaWarps + wl;
    const int64_t nw = (int64_t)gridDim.x * kTmaWarps;
    if (lane == 0) {
        for (int st = 0; st < kTmaStages; ++st) md::mbar_init(&bar[st], 1);
        md::fence_mbar_init();
    }
    __syncwarp();
    if (gw >= U) return;

    auto token_of = [&](int64_t u) { return pieces == 1 ? u : u / pieces; };
    auto piece_of = [&](int64_t u) { return pieces == 1 ? 0 : (int)(u - (u / pieces) * pieces); };
    auto bytes_of = [&](int64_t u) {
        const int b = rowbytes - piece_of(u) * kTmaPiece;
        return (uint32_t)(b < kTmaPiece ? b : kTmaPiece);
    };
    auto issue_load = [&](int64_t u, int st) {
        const uint32_t nb = bytes_of(u);
        md::mbar_expect_tx(&bar[st], nb);
        md::bulk_load(ring + (size_t)st * kTmaPiece,
                      x + token_of(u) * (int64_t)rowbytes + (int64_t)piece_of(u) * kTmaPiece, nb,
                      &bar[st]);
    };

    if (lane == 0)
        for (int j = 0; j < kTmaAhead; ++j)
            if (gw + j * nw < U) issue_load(gw + j * nw, j % kTmaStages);
    int rows = lane < K ? __ldg(row_of_slot + token_of(gw) * K + lane) : -1;

    int64_t i = 0;
    for (int64_t u = gw; u < U; u += nw, ++i) {
        const int st = (int)(i % kTmaStages);
        const int64_t ua = u + (int64_t)kTmaAhead * nw;
        if (lane == 0 && ua < U) {
            // slot of unit i + kTmaAhead was last read by the stores of unit
            // i + kTmaAhead - kTmaStages
            md::bulk_wait_read<kTmaStages - kTmaAhead - 1>();
            issue_load(ua, (int)((i + kTmaAhead) % kTmaStages));
        }
        const int64_t un = u + nw;
        const int nrows = (un < U && lane < K) ? __ldg(row_of_slot + token_of(un) * K + lane) : -1;

        int ok = 1;
        if (lane == 0) ok = md::mbar_wait_bounded(&bar[st], (uint32_t)((i / kTmaStages) & 1), kTmaPolls);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
            md::report(status, MD_ERR_TIMEOUT);
            if (lane == 0) {
                // wait, again bounded, for the loads still in flight: the one
                // that timed out and the ones issued after it.  A load that
                // is merely late beyond both bounds can still land in shared
                // memory after the block has exited.
                for (int j = 0; j <= kTmaAhead; ++j)
                    if (u + j * nw < U)
                        md::mbar_wait_bounded(&bar[(i + j) % kTmaStages],
                                              (uint32_t)(((i + j) / kTmaStages) & 1), kTmaPolls);
            }
            break;
        }
        // distinct, in-range rows of this token (slots sharing a row write once)
        const unsigned g = __match_any_sync(0xffffffffu, lane < K ? (unsigned)rows : (0x80000000u | lane));
        const bool first = lane < K && (g & md::lanemask_lt()) == 0u;
        const bool valid = rows >= 0 && rows < out_rows;
        const int pc = piece_of(u);
        if (first && !valid && pc == 0) md::report(status, MD_ERR_DATA);
        unsigned todo = __ballot_sync(0xffffffffu, first && valid);
        const uint32_t nb = bytes_of(u);
        while (todo) {
            const int j = __ffs(todo) - 1;
            todo &= todo - 1;
            const int64_t r = __shfl_sync(0xffffffffu, rows, j);
            if (lane == 0)
                md::bulk_store(out + r * rowbytes + (int64_t)pc * kTmaPiece,
                               ring + (size_t)st * kTmaPiece, nb);
        }
        if (lane == 0) md::bulk_commit();
        rows = nrows;
    }
    if (lane == 0) md::bulk_wait_all();
}

// ----------------------------------------------------------------- combine
__device__ __forceinline__ void fma_row(float (&acc)[8], float w, const uint4 &v)
{
    acc[0] = fmaf(w, md::bf16lo(v.x), acc[0]);
    acc[1] = fmaf(w, md::bf16hi(v.x), acc[1]);
    acc[2] = fmaf(w, md::bf16lo(v.y), acc[2]);
    acc[3] = fmaf(w, md::bf16hi(v.y), acc[3]);
    acc[4] = fmaf(w, md::bf16lo(v.z), acc[4]);
    acc[5] = fmaf(w, md::bf16hi(v.z), acc[5]);
    acc[6] = fmaf(w, md::bf16lo(v.w), acc[6]);
    acc[7] = fmaf(w, md::bf16hi(v.w), acc[7]);
}

__device__ __forceinline__ uint4 pack_row(const float (&a)[8])
{
    return make_uint4(md::pack_bf16x2(a[0], a[1]), md::pack_bf16x2(a[2], a[3]),
                      md::pack_bf16x2(a[4], a[5]), md::pack_bf16x2(a[6], a[7]));
}

// FUSED: out[t] = bf16(sum over slots by ascending expert of w * y), fp32 FMA.
// WIRE:  slots sorted by (wire row, expert); each run of one wire row is
//        summed, rounded to bf16 and stored in z; out[t] = bf16(fp32 sum of
//        those bf16 partials in wire-row order).
template <int KC, bool WIRE>
__global__ void __launch_bounds__(kThreads)
    k_combine(const uint4 *__restrict__ y, int64_t y_rows, const int32_t *__restrict__ assign_row,
              const int32_t *__restrict__ idx, const float *__restrict__ w, int64_t T, int k, int C,
              const int32_t *__restrict__ row_of_slot, int64_t z_rows, uint4 *__restrict__ z,
              uint4 *__restrict__ out, int32_t *status)
{
    __shared__ int s_r[kGroup][MD_MAX_TOPK];
    __shared__ float s_w[kGroup][MD_MAX_TOPK];
    __shared__ int s_z[kGroup][WIRE ? MD_MAX_TOPK : 1];
    const int K = KC ? KC : k;
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;

    for (int64_t g0 = (int64_t)blockIdx.x * kGroup; g0 < T; g0 += (int64_t)gridDim.x * kGroup) {
        const int ng = (int)(T - g0 < kGroup ? T - g0 : kGroup);
        // warp wp orders the slots of token g0 + wp
        if (wp < ng) {
            const int64_t t = g0 + wp;
            const bool live = lane < K;
            const int e = live ? idx[t * K + lane] : INT_MAX;
            int r = live ? assign_row[t * K + lane] : -1;
            const float ww = live ? w[t * K + lane] : 0.0f;
            int zr = (WIRE && live) ? row_of_slot[t * K + lane] : 0;
            int rank = 0;
            for (int j = 0; j < K; ++j) {
                const int ej = __shfl_sync(0xffffffffu, e, j);
                const int zj = WIRE ? __shfl_sync(0xffffffffu, zr, j) : 0;
                bool before = ej < e || (ej == e && j < lane);
                if (WIRE) before = zj < zr || (zj == zr && before);
                rank += before ? 1 : 0;
            }
            if (live) {
                if (r < 0 || r >= y_rows) {
                    md::report(status, MD_ERR_DATA);
                    r = -1;
                }
                if (WIRE && (zr < 0 || zr >= z_rows)) {
                    md::report(status, MD_ERR_DATA);
                    zr = -1;
                }
                s_r[wp][rank] = r;
                s_w[wp][rank] = ww;
                if (WIRE) s_z[wp][rank] = zr;
            }
        }
        __syncthreads();
        for (int g = 0; g < ng; ++g) {
            const int64_t t = g0 + g;
            for (int c = threadIdx.x; c < C; c += kThreads) {
                float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                float tot[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                constexpr int B = KC ? KC : 4;  // loads issued together
                for (int j0 = 0; j0 < K; j0 += B) {
                    uint4 v[B];
#pragma unroll
                    for (int q = 0; q < B; ++q) {
                        const int j = j0 + q;
                        const int r = j < K ? s_r[g][j] : -1;
                        v[q] = r >= 0 ? md::ld_stream(y + (int64_t)r * C + c) : make_uint4(0, 0, 0, 0);
                    }
#pragma unroll
                    for (int q = 0; q < B; ++q) {
                        const int j = j0 + q;
                        if (j >= K) break;
                        if (s_r[g][j] >= 0) fma_row(acc, s_w[g][j], v[q]);
                        if (WIRE && (j == K - 1 || s_z[g][j + 1] != s_z[g][j])) {
                            const uint4 zb = pack_row(acc);
                            const int zr = s_z[g][j];
                            if (zr >= 0) md::st_stream(z + (int64_t)zr * C + c, zb);
                            tot[0] += md::bf16lo(zb.x);
                            tot[1] += md::bf16hi(zb.x);
                            tot[2] += md::bf16lo(zb.y);
                            tot[3] += md::bf16hi(zb.y);
                            tot[4] += md::bf16lo(zb.z);
                            tot[5] += md::bf16hi(zb.z);
                            tot[6] += md::bf16lo(zb.w);
                            tot[7] += md::bf16hi(zb.w);
#pragma unroll
                            for (int i = 0; i < 8; ++i) acc[i] = 0.f;
                        }
                    }
                }
                md::st_stream(out + t * C + c, pack_row(WIRE ? tot : acc));
            }
        }
        __syncthreads();
    }
}

// FUSED with a compile-time k: the same slot order and arithmetic as
// k_combine<KC, false>, but for small k each thread works on U (token,
// 16-byte column) items at once and issues all U*KC row loads before the
// first FMA, so that 8 loads are in flight per thread (with k = 2 a single
// item keeps only two in flight, and the kernel waits on latency).  From
// k = 4 on one item per thread measured best.  Items of a group are
// q = c + g*C for its ng tokens.
template <int KC>
constexpr int combine_items() { return KC >= 4 ? 1 : (8 + KC - 1) / KC; }

template <int KC>
__global__ void __launch_bounds__(kThreads)
    k_combine_fused(const uint4 *__restrict__ y, int64_t y_rows, const int32_t *__restrict__ assign_row,
                    const int32_t *__restrict__ idx, const float *__restrict__ w, int64_t T, int C,
                    uint4 *__restrict__ out, int32_t *status)
{
    constexpr int U = combine_items<KC>();
    __shared__ int s_r[kGroup][KC];
    __shared__ float s_w[kGroup][KC];
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;

    for (int64_t g0 = (int64_t)blockIdx.x * kGroup; g0 < T; g0 += (int64_t)gridDim.x * kGroup) {
        const int ng = (int)(T - g0 < kGroup ? T - g0 : kGroup);
        // warp wp orders the slots of token g0 + wp by ascending expert
        if (wp < ng) {
            const int64_t t = g0 + wp;
            const bool live = lane < KC;
            const int e = live ? idx[t * KC + lane] : INT_MAX;
            int r = live ? assign_row[t * KC + lane] : -1;
            const float ww = live ? w[t * KC + lane] : 0.0f;
            int rank = 0;
#pragma unroll
            for (int j = 0; j < KC; ++j) {
                const int ej = __shfl_sync(0xffffffffu, e, j);
                rank += (ej < e || (ej == e && j < lane)) ? 1 : 0;
            }
            if (live) {
                if (r < 0 || r >= y_rows) {
                    md::report(status, MD_ERR_DATA);
                    r = -1;
                }
                s_r[wp][rank] = r;
                s_w[wp][rank] = ww;
            }
        }
        __syncthreads();
        const int nq = ng * C;
        for (int q0 = threadIdx.x; q0 < nq; q0 += kThreads * U) {
            uint4 v[U][KC];
            int gq[U], cq[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int q = q0 + u * kThreads;
                gq[u] = q < nq ? q / C : -1;
                cq[u] = q < nq ? q - gq[u] * C : 0;
#pragma unroll
                for (int j = 0; j < KC; ++j) {
                    const int r = gq[u] >= 0 ? s_r[gq[u]][j] : -1;
                    v[u][j] = r >= 0 ? md::ld_stream(y + (int64_t)r * C + cq[u]) : make_uint4(0, 0, 0, 0);
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (gq[u] < 0) continue;
                float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int j = 0; j < KC; ++j)
                    if (s_r[gq[u]][j] >= 0) fma_row(acc, s_w[gq[u]][j], v[u][j]);
                md::st_stream(out + (g0 + gq[u]) * C + cq[u], pack_row(acc));
            }
        }
        __syncthreads();
    }
}

// ------------------------------------------------------------------ gather
__global__ void __launch_bounds__(kThreads)
    k_gather16(const uint4 *__restrict__ src, int64_t src_rows, int C,
               const int32_t *__restrict__ index, int64_t n_out, uint4 *__restrict__ dst,
               int32_t *status)
{
    const int64_t n = n_out * C;
    for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * kThreads) {
        const int64_t row = i / C;
        const int c = (int)(i - row * C);
        const int s = __ldg(index + row);
        if (s < 0 || s >= src_rows) {
            if (c == 0) md::report(status, MD_ERR_DATA);
            continue;
        }
        md::st_stream(dst + i, md::ld_stream(src + (int64_t)s * C + c));
    }
}

__global__ void __launch_bounds__(kThreads)
    k_gather4(const uint32_t *__restrict__ src, int64_t src_rows, int C,
              const int32_t *__restrict__ index, int64_t n_out, uint32_t *__restrict__ dst,
              int32_t *status)
{
    const int64_t n = n_out * C;
    for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * kThreads) {
        const int64_t row = i / C;
        const int c = (int)(i - row * C);
        const int s = __ldg(index + row);
        if (s < 0 || s >= src_rows) {
            if (c == 0) md::report(status, MD_ERR_DATA);
            continue;
        }
        dst[i] = __ldg(src + (int64_t)s * C + c);
    }
}

template <int KC>
void launch_permute(const void *x, int64_t T, int C, int k, const int32_t *rs, int64_t rows,
                    void *out, int32_t *st, cudaStream_t s)
{
    const int rowbytes = C * 16;
    const int pieces = (rowbytes + kTmaPiece - 1) / kTmaPiece;
    const int64_t units = T * pieces;
    // Which kernel: bulk copies need rows of 1 KiB and more.  By shape (the
    // default), they take the write-heavy calls -- k > 4 slots per token and
    // at least 8 row pieces per warp of the bulk-copy grid -- where one ring
    // of 4 warps per SM gave the best write bandwidth.  With k <= 4 a larger
    // share of the bytes are reads and the ring waits on its loads; with few
    // pieces per warp its start and drain dominate.  There the vector kernel,
    // with one warp per token in flight across the whole GPU, measured faster.
    const int path = md::permute_path();
    bool bulk = rowbytes >= kTmaMinRowBytes && path != MD_PERMUTE_VECTOR;
    if (bulk && path == MD_PERMUTE_AUTO)
        bulk = k > 4 && units >= (int64_t)8 * md::sm_count() * kTmaWarps;
    // once per device: the ring's shared-memory limit and the vector
    // kernel's resident CTAs per SM
    static std::atomic<uint64_t> setup{0};
    static std::atomic<int> vec_per_sm[64];
    const size_t smem = (size_t)kTmaWarps * kTmaStages * kTmaPiece;
    md::once_per_device(setup, [smem] {
        int dev = 0, nb = 0;
        cudaGetDevice(&dev);
        if (cudaFuncSetAttribute(k_permute_tma<KC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem) != cudaSuccess)
            cudaGetLastError();  // the launch then fails and reports MD_ERR_CUDA
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, k_permute<KC>, kThreads, 0) != cudaSuccess) {
            cudaGetLastError();
            nb = 1;
        }
        vec_per_sm[dev & 63].store(nb < 1 ? 1 : nb);
    });
    if (bulk) {
        int64_t blocks = (units + kTmaWarps - 1) / kTmaWarps;
        const int64_t cap = md::sm_count();
        if (blocks > cap) blocks = cap;
        k_permute_tma<KC><<<(unsigned)(blocks < 1 ? 1 : blocks), kTmaWarps * 32, smem, s>>>(
            static_cast<const char *>(x), T, rowbytes, pieces, k, rs, rows, static_cast<char *>(out),
            st);
        return;
    }
    int dev = 0;
    cudaGetDevice(&dev);
    const int per_sm = vec_per_sm[dev & 63].load();
    int64_t blocks = (T + kThreads / 32 - 1) / (kThreads / 32);
    const int64_t cap = (int64_t)md::sm_count() * per_sm;
    if (blocks > cap) blocks = cap;
    k_permute<KC><<<(unsigned)(blocks < 1 ? 1 : blocks), kThreads, 0, s>>>(
        static_cast<const uint4 *>(x), T, C, k, rs, rows, static_cast<uint4 *>(out), st);
}

template <int KC, bool WIRE>
void launch_combine(const void *y, int64_t y_rows, const int32_t *ar, const int32_t *idx,
                    const float *w, int64_t T, int k, int C, const int32_t *rs, int64_t z_rows,
                    void *z, void *out, int32_t *st, cudaStream_t s)
{
    if (KC > 0 && !WIRE) {  // 4, 6 or 16 CTAs per SM measured no better than 8
        k_combine_fused<KC ? KC : 1><<<grid_for(T, kGroup), kThreads, 0, s>>>(
            static_cast<const uint4 *>(y), y_rows, ar, idx, w, T, C, static_cast<uint4 *>(out), st);
        return;
    }
    k_combine<KC, WIRE><<<grid_for(T, kGroup), kThreads, 0, s>>>(
        static_cast<const uint4 *>(y), y_rows, ar, idx, w, T, k, C, rs, z_rows,
        static_cast<uint4 *>(z), static_cast<uint4 *>(out), st);
}

template <bool WIRE>
void dispatch_combine(const void *y, int64_t y_rows, const int32_t *ar, const int32_t *idx,
                      const float *w, int64_t T, int k, int C, const int32_t *rs, int64_t z_rows,
                      void *z, void *out, int32_t *st, cudaStream_t s)
{
    switch (k) {
    case 1: launch_combine<1, WIRE>(y, y_rows, ar, idx, w, T, k, C, rs, z_rows, z, out, st, s); break;
    case 2: launch_combine<2, WIRE>(y, y_rows, ar, idx, w, T, k, C, rs, z_rows, z, out, st, s); break;
    case 4: launch_combine<4, WIRE>(y, y_rows, ar, idx, w, T, k, C, rs, z_rows, z, out, st, s); break;
    case 6: launch_combine<6, WIRE>(y, y_rows, ar, idx, w, T, k, C, rs, z_rows, z, out, st, s); break;
    case 8: launch_combine<8, WIRE>(y, y_rows, ar, idx, w, T, k, C, rs, z_rows, z, out, st, s); break;
    default: launch_combine<0, WIRE>(y, y_rows, ar, idx, w, T, k, C, rs, z_rows, z, out, st, s); break;
    }
}

}  // namespace

extern "C" int md_dispatch_permute(const void *x, int64_t T, int H, int k,
                                   const int32_t *row_of_slot, int64_t out_rows, void *out,
                                   int32_t *dev_status, void *stream)
{
    if (T < 0 || H < 8 || H % 8 != 0 || k < 1 || k > MD_MAX_TOPK || out_rows < 0) return MD_ERR_ARG;
    if (T > 0 && (!x || !row_of_slot || !md::aligned16(x))) return MD_ERR_ARG;
    if (out_rows > 0 && (!out || !md::aligned16(out))) return MD_ERR_ARG;
    cudaStream_t s = md::as_stream(stream);
    int rc = md::clear_status(dev_status, s);
    if (rc != MD_OK || T == 0) return rc;
    const int C = H / 8;
    switch (k) {
    case 1: launch_permute<1>(x, T, C, k, row_of_slot, out_rows, out, dev_status, s); break;
    case 2: launch_permute<2>(x, T, C, k, row_of_slot, out_rows, out, dev_status, s); break;
    case 4: launch_permute<4>(x, T, C, k, row_of_slot, out_rows, out, dev_status, s); break;
    case 6: launch_permute<6>(x, T, C, k, row_of_slot, out_rows, out, dev_status, s); break;
    case 8: launch_permute<8>(x, T, C, k, row_of_slot, out_rows, out, dev_status, s); break;
    default: launch_permute<0>(x, T, C, k, row_of_slot, out_rows, out, dev_status, s); break;
    }
    md::count_launches(1);
    return md::launch_status();
}

extern "C" int md_combine(const void *y, int64_t y_rows, const int32_t *assign_row,
                          const int32_t *topk_idx, const float *topk_w, int64_t T, int k, int H,
                          int combine_mode, const int32_t *row_of_slot, int64_t z_rows, void *z,
                          void *out, int32_t *dev_status, void *stream)
{
    if (T < 0 || H < 8 || H % 8 != 0 || k < 1 || k > MD_MAX_TOPK || y_rows < 0) return MD_ERR_ARG;
    if (combine_mode != MD_COMBINE_FUSED && combine_mode != MD_COMBINE_WIRE) return MD_ERR_ARG;
    if (T > 0 && (!assign_row || !topk_idx || !topk_w || !out || !md::aligned16(out)))
        return MD_ERR_ARG;
    if (y_rows > 0 && (!y || !md::aligned16(y))) return MD_ERR_ARG;
    const bool wire = combine_mode == MD_COMBINE_WIRE;
    if (wire && T > 0 && (!row_of_slot || z_rows < 0 || (z_rows > 0 && (!z || !md::aligned16(z)))))
        return MD_ERR_ARG;
    cudaStream_t s = md::as_stream(stream);
    int rc = md::clear_status(dev_status, s);
    if (rc != MD_OK || T == 0) return rc;
    const int C = H / 8;
    if (wire)
        dispatch_combine<true>(y, y_rows, assign_row, topk_idx, topk_w, T, k, C, row_of_slot,
                               z_rows, z, out, dev_status, s);
    else
        dispatch_combine<false>(y, y_rows, assign_row, topk_idx, topk_w, T, k, C, nullptr, 0,
                                nullptr, out, dev_status, s);
    md::count_launches(1);
    return md::launch_status();
}

extern "C" int md_gather_rows(const void *src, int64_t src_rows, int64_t row_bytes,
                              const int32_t *index, int64_t n_out, void *dst, int32_t *dev_status,
                              void *stream)
{
    if (src_rows < 0 || n_out < 0 || row_bytes < 4 || row_bytes % 4 != 0) return MD_ERR_ARG;
    if (n_out > 0 && (!index || !dst)) return MD_ERR_ARG;
    if (src_rows > 0 && !src) return MD_ERR_ARG;
    cudaStream_t s = md::as_stream(stream);
    int rc = md::clear_status(dev_status, s);
    if (rc != MD_OK || n_out == 0) return rc;
    if (row_bytes % 16 == 0 && md::aligned16(src) && md::aligned16(dst)) {
        const int C = (int)(row_bytes / 16);
        k_gather16<<<grid_for(n_out * C, kThreads * 4), kThreads, 0, s>>>(
            static_cast<const uint4 *>(src), src_rows, C, index, n_out, static_cast<uint4 *>(dst),
            dev_status);
    } else {
        const int C = (int)(row_bytes / 4);
        k_gather4<<<grid_for(n_out * C, kThreads * 4), kThreads, 0, s>>>(
            static_cast<const uint32_t *>(src), src_rows, C, index, n_out,
            static_cast<uint32_t *>(dst), dev_status);
    }
    md::count_launches(1);
    return md::launch_status();
}
