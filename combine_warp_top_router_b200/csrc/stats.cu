// stats.cu -- routing statistics (md_rank_stats, md_successor_share,
// md_count_sums).
//
// "Expert Coupling in MoE Pretraining" (PicX summary):
//   Offline Placement and Prediction Statistics, Table I: "Same GPU" (tokens
//   whose experts all sit on one rank), "GPUs" (distinct ranks per token) and
//   "Dedup" (1 - GPUs / k) come from hist[D], the number of tokens with D
//   distinct destination ranks.  A token's ranks are a 64-bit mask, so D is
//   one popcount.
//   Cross-layer correlation: the share of expert e's tokens that select e'
//   at the next layer is C[e][e'] / W[e][e]; one warp per row finds the
//   largest C[e][e'].
//   Correlation Formation and Stability: the Pearson correlation of two count
//   tables follows from five exact sums, accumulated in 128 bits by one CTA.
#include <cmath>

#include "common.cuh"

namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
    k_rank_stats(const int32_t *__restrict__ idx, int64_t T, int E, int k, int R,
                 const int32_t *__restrict__ p, unsigned long long *__restrict__ hist,
                 int32_t *status)
{
    __shared__ unsigned int h[MD_MAX_TOPK + 1];
    for (int d = threadIdx.x; d <= k; d += kThreads) h[d] = 0u;
    __syncthreads();
    for (int64_t t = (int64_t)blockIdx.x * kThreads + threadIdx.x; t < T;
         t += (int64_t)gridDim.x * kThreads) {
        unsigned long long mask = 0ull;
        bool bad = false;
        for (int j = 0; j < k; ++j) {
            const int e = __ldg(idx + t * k + j);
            const int d = (e >= 0 && e < E) ? __ldg(p + e) : -1;
            if (d < 0 || d >= R) {
                bad = true;
                continue;
            }
            mask |= 1ull << d;
        }
        if (bad) md::report(status, MD_ERR_DATA);
        atomicAdd(&h[__popcll(mask)], 1u);
    }
    __syncthreads();
    for (int d = threadIdx.x; d <= k; d += kThreads)
        if (h[d]) atomicAdd(hist + d, (unsigned long long)h[d]);
}

__global__ void __launch_bounds__(kThreads)
    k_successor_share(const uint32_t *__restrict__ C, const uint32_t *__restrict__ W, int E,
                      uint32_t *__restrict__ num, uint32_t *__restrict__ den)
{
    const int lane = threadIdx.x & 31;
    const int64_t w0 = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * kThreads) >> 5;
    for (int64_t e = w0; e < E; e += nw) {
        uint32_t m = 0u;
        for (int e2 = lane; e2 < E; e2 += 32) m = max(m, __ldg(C + e * E + e2));
        m = __reduce_max_sync(0xffffffffu, m);
        if (lane == 0) {
            num[e] = m;
            den[e] = __ldg(W + e * E + e);
        }
    }
}

// One CTA of 1024 threads; each thread keeps 128-bit partial sums.
__global__ void __launch_bounds__(1024)
    k_count_sums(const uint32_t *__restrict__ x, const uint32_t *__restrict__ y, int64_t n,
                 unsigned long long *__restrict__ out)
{
    __shared__ unsigned long long s_part[32][10];
    unsigned __int128 s[5] = {0, 0, 0, 0, 0};
    for (int64_t i = threadIdx.x; i < n; i += 1024) {
        const unsigned long long a = __ldg(x + i), b = __ldg(y + i);
        s[0] += a;
        s[1] += b;
        s[2] += (unsigned __int128)(a * a);
        s[3] += (unsigned __int128)(b * b);
        s[4] += (unsigned __int128)(a * b);
    }
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
#pragma unroll
    for (int q = 0; q < 5; ++q) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const unsigned long long lo = __shfl_xor_sync(0xffffffffu, (unsigned long long)s[q], o);
            const unsigned long long hi =
                __shfl_xor_sync(0xffffffffu, (unsigned long long)(s[q] >> 64), o);
            s[q] += ((unsigned __int128)hi << 64) | lo;
        }
    }
    if (lane == 0)
        for (int q = 0; q < 5; ++q) {
            s_part[wp][2 * q] = (unsigned long long)s[q];
            s_part[wp][2 * q + 1] = (unsigned long long)(s[q] >> 64);
        }
    __syncthreads();
    if (threadIdx.x < 5) {
        const int q = threadIdx.x;
        unsigned __int128 t = 0;
        for (int w = 0; w < 32; ++w)
            t += ((unsigned __int128)s_part[w][2 * q + 1] << 64) | s_part[w][2 * q];
        out[2 * q] = (unsigned long long)t;
        out[2 * q + 1] = (unsigned long long)(t >> 64);
    }
}

}  // namespace

extern "C" int md_rank_stats(const int32_t *topk_idx, int64_t T, int E, int k, int R,
                             const int32_t *expert_to_rank, int64_t *hist, int32_t *dev_status,
                             void *stream)
{
    if (T < 0 || E < 1 || k < 1 || k > MD_MAX_TOPK || R < 1 || !hist || !expert_to_rank)
        return MD_ERR_ARG;
    if (R > MD_MAX_RANKS || E > MD_MAX_EXPERTS) return MD_ERR_UNSUPPORTED;
    if (T > 0 && !topk_idx) return MD_ERR_ARG;
    cudaStream_t s = md::as_stream(stream);
    int rc = md::clear_status(dev_status, s);
    if (rc != MD_OK) return rc;
    md::count_memsets(1);
    if (cudaMemsetAsync(hist, 0, sizeof(int64_t) * (size_t)(k + 1), s) != cudaSuccess)
        return MD_ERR_CUDA;
    if (T == 0) return MD_OK;
    int64_t blocks = (T + kThreads - 1) / kThreads;
    const int64_t cap = (int64_t)md::sm_count() * 8;
    if (blocks > cap) blocks = cap;
    k_rank_stats<<<(unsigned)blocks, kThreads, 0, s>>>(topk_idx, T, E, k, R, expert_to_rank,
                                                       reinterpret_cast<unsigned long long *>(hist),
                                                       dev_status);
    md::count_launches(1);
    return md::launch_status();
}

extern "C" int md_successor_share(const uint32_t *C, const uint32_t *W, int E, uint32_t *num,
                                  uint32_t *den, void *stream)
{
    if (E < 1 || !C || !W || !num || !den) return MD_ERR_ARG;
    if (E > MD_MAX_EXPERTS) return MD_ERR_UNSUPPORTED;
    cudaStream_t s = md::as_stream(stream);
    const int blocks = (E * 32 + kThreads - 1) / kThreads;
    k_successor_share<<<blocks, kThreads, 0, s>>>(C, W, E, num, den);
    md::count_launches(1);
    return md::launch_status();
}

extern "C" int md_count_sums(const uint32_t *x, const uint32_t *y, int64_t n, uint64_t *sums,
                             void *stream)
{
    if (n < 0 || !sums || (n > 0 && (!x || !y))) return MD_ERR_ARG;
    if (n >= ((int64_t)1 << 31)) return MD_ERR_UNSUPPORTED;
    cudaStream_t s = md::as_stream(stream);
    k_count_sums<<<1, 1024, 0, s>>>(x, y, n, reinterpret_cast<unsigned long long *>(sums));
    md::count_launches(1);
    return md::launch_status();
}

// ------------------------------------------------------------------------
// Host helpers: the finished statistics from the device counts above.
// ------------------------------------------------------------------------

// Table I columns ("Expert Coupling ...", Offline Placement and Prediction
// Statistics) from hist[D] = tokens on exactly D distinct ranks:
//   out[0] "Same GPU" %  = 100 * hist[1] / T
//   out[1] "GPUs"        = sum_D D * hist[D] / T   (mean distinct ranks)
//   out[2] "Dedup" %     = 100 * (1 - GPUs / k)
// The token count T = sum_D hist[D] and the weighted sum are exact integers.
extern "C" int md_table1_row(const int64_t *hist, int k, double *out)
{
    if (!hist || !out || k < 1 || k > MD_MAX_TOPK) return MD_ERR_ARG;
    int64_t T = 0, ranks = 0;
    for (int d = 0; d <= k; ++d) {
        if (hist[d] < 0) return MD_ERR_ARG;
        T += hist[d];
        ranks += (int64_t)d * hist[d];
    }
    if (T == 0) return MD_ERR_ARG;
    const double gpus = (double)ranks / (double)T;
    out[0] = 100.0 * (double)hist[1] / (double)T;
    out[1] = gpus;
    out[2] = 100.0 * (1.0 - gpus / (double)k);
    return MD_OK;
}

// Pearson correlation of two count tables of n entries ("Expert Coupling
// ...", Correlation Formation and Stability) from md_count_sums' exact sums
// (sx, sy, sxx, syy, sxy as 128-bit (low, high) word pairs):
//   r = (n sxy - sx sy) / sqrt((n sxx - sx^2) (n syy - sy^2)).
// With n < 2^31 and 32-bit counts, sx < 2^63 and sxx, sxy < 2^95, so every
// product and each of the three differences is exact in signed 128 bits; the
// quotient is taken in long double.  A table with zero variance gives MD_ERR_DATA (r undefined).
extern "C" int md_pearson_from_sums(const uint64_t *sums, int64_t n, double *r)
{
    if (!sums || !r || n < 1) return MD_ERR_ARG;
    if (n >= ((int64_t)1 << 31)) return MD_ERR_UNSUPPORTED;
    // n < 2^31 entries below 2^32: sums below 2^63, sums of products below 2^95
    unsigned __int128 v[5];
    for (int q = 0; q < 5; ++q) {
        v[q] = ((unsigned __int128)sums[2 * q + 1] << 64) | sums[2 * q];
        if (v[q] >> (q < 2 ? 63 : 95)) return MD_ERR_DATA;  // not sums of such counts
    }
    const __int128 N = n, sx = (__int128)v[0], sy = (__int128)v[1];
    const __int128 sxx = (__int128)v[2], syy = (__int128)v[3], sxy = (__int128)v[4];
    const __int128 cov = N * sxy - sx * sy;
    const __int128 vx = N * sxx - sx * sx;
    const __int128 vy = N * syy - sy * sy;
    if (vx <= 0 || vy <= 0) return MD_ERR_DATA;
    const long double den = sqrtl((long double)vx) * sqrtl((long double)vy);
    *r = (double)((long double)cov / den);
    return MD_OK;
}
