// coselect.cu -- within-layer co-selection and cross-layer transition counts
// (md_coselect_stats).
//
// "Expert Coupling in MoE Pretraining" (PicX summary), Correlated Placement:
// W[e, e'] counts tokens selecting both e and e'; Cross-layer correlation:
// the experts a token selects at layer l predict its layer-l+1 experts.
//
// The counters are privatised in shared memory.  The E x E tables do not fit
// in one CTA's shared memory for E = 256 (W's upper triangle plus C is 98,432
// counters), so the counter space [W upper triangle | C] is cut into
// segments of at most kSegEntries; blockIdx.y picks the segment and
// blockIdx.x a chunk of tokens.  Each CTA counts the increments that fall in
// its segment with shared-memory atomics and adds its non-zero counters to
// W / C in global memory (both W[a][b] and W[b][a] for a != b).
//
// Pair counts (md_coselect_pair_stats), "Expert Coupling ...", Method 2,
// Prediction (pair-based lookup over the two preceding layers):
// C2[a][b][e'] counts every (a in S_{l-1}(t), b in S_l(t), e' in S_{l+1}(t))
// triple.  The E^3 table lives in global memory; one thread per (token, a, b)
// adds its k increments with global atomics.
#include "common.cuh"

namespace {

constexpr int kThreads = 1024;
constexpr int kSegEntries = 48 * 1024;  // 192 KiB of uint32 counters

__device__ __forceinline__ int64_t tri_id(int a, int b, int E)  // a <= b
{
    return (int64_t)a * E - (int64_t)a * (a - 1) / 2 + (b - a);
}

__global__ void __launch_bounds__(kThreads)
    k_coselect(const int32_t *__restrict__ idx_l, const int32_t *__restrict__ idx_n, int64_t T_fit,
               int E, int k, int64_t tok_per_block, uint32_t *__restrict__ W,
               uint32_t *__restrict__ C, int64_t n_tri, int64_t seg_len, int32_t *status)
{
    extern __shared__ uint32_t cnt[];
    const int64_t lo = (int64_t)blockIdx.y * seg_len;
    const int64_t n_total = (W ? n_tri : 0) + (C ? (int64_t)E * E : 0);
    const int64_t hi = lo + seg_len < n_total ? lo + seg_len : n_total;
    const int64_t c_base = W ? n_tri : 0;  // id of C[0][0]
    for (int64_t i = threadIdx.x; i < hi - lo; i += kThreads) cnt[i] = 0u;
    __syncthreads();

    const int64_t t0 = (int64_t)blockIdx.x * tok_per_block;
    const int64_t t1 = t0 + tok_per_block < T_fit ? t0 + tok_per_block : T_fit;
    // one thread per (token, slot i); loops over the token's slots j
    for (int64_t f = t0 * k + threadIdx.x; f < t1 * k; f += kThreads) {
        const int64_t t = f / k;
        const int i = (int)(f - t * k);
        const int a = idx_l[f];
        if (a < 0 || a >= E) {
            if (blockIdx.y == 0) md::report(status, MD_ERR_DATA);
            continue;
        }
        for (int j = 0; j < k; ++j) {
            if (W && j >= i) {
                const int b = __ldg(idx_l + t * k + j);
                if (b >= 0 && b < E) {
                    const int64_t id = a <= b ? tri_id(a, b, E) : tri_id(b, a, E);
                    if (id >= lo && id < hi) atomicAdd(&cnt[id - lo], 1u);
                }
            }
            if (C) {
                const int b = __ldg(idx_n + t * k + j);
                if (b < 0 || b >= E) {
                    if (i == 0 && blockIdx.y == 0) md::report(status, MD_ERR_DATA);
                    continue;
                }
                const int64_t id = c_base + (int64_t)a * E + b;
                if (id >= lo && id < hi) atomicAdd(&cnt[id - lo], 1u);
            }
        }
    }
    __syncthreads();

    // flush the segment: walk (a, b) over all cells whose id lands here
    if (W && lo < n_tri) {
        for (int64_t cell = threadIdx.x; cell < (int64_t)E * E; cell += kThreads) {
            const int a = (int)(cell / E), b = (int)(cell - (int64_t)a * E);
            if (b < a) continue;
            const int64_t id = tri_id(a, b, E);
            if (id < lo || id >= hi) continue;
            const uint32_t v = cnt[id - lo];
            if (!v) continue;
            atomicAdd(&W[(int64_t)a * E + b], v);
            if (a != b) atomicAdd(&W[(int64_t)b * E + a], v);
        }
    }
    if (C && hi > c_base) {
        const int64_t from = lo > c_base ? lo : c_base;
        for (int64_t id = from + threadIdx.x; id < hi; id += kThreads) {
            const uint32_t v = cnt[id - lo];
            if (v) atomicAdd(&C[id - c_base], v);
        }
    }
}

__global__ void __launch_bounds__(256)
    k_coselect_pair(const int32_t *__restrict__ idx_p, const int32_t *__restrict__ idx_l,
                    const int32_t *__restrict__ idx_n, int64_t T_fit, int E, int k,
                    uint32_t *__restrict__ C2, int32_t *status)
{
    const int kk = k * k;
    const int64_t n = T_fit * kk;
    for (int64_t f = (int64_t)blockIdx.x * 256 + threadIdx.x; f < n; f += (int64_t)gridDim.x * 256) {
        const int64_t t = f / kk;
        const int r = (int)(f - t * kk);
        const int i = r / k, j = r - i * k;
        const int a = __ldg(idx_p + t * k + i), b = __ldg(idx_l + t * k + j);
        if (a < 0 || a >= E || b < 0 || b >= E) {
            md::report(status, MD_ERR_DATA);
            continue;
        }
        uint32_t *row = C2 + ((int64_t)a * E + b) * E;
        for (int m = 0; m < k; ++m) {
            const int c = __ldg(idx_n + t * k + m);
            if (c >= 0 && c < E) atomicAdd(row + c, 1u);
            else md::report(status, MD_ERR_DATA);
        }
    }
}

}  // namespace

extern "C" int md_coselect_stats(const int32_t *idx_l, const int32_t *idx_next, int64_t T_fit,
                                 int E, int k, uint32_t *W, uint32_t *C, int accumulate,
                                 int32_t *dev_status, void *stream)
{
    if (T_fit < 0 || E < 1 || k < 1 || k > MD_MAX_TOPK) return MD_ERR_ARG;
    if (E > MD_MAX_EXPERTS) return MD_ERR_UNSUPPORTED;
    if (!W && !C) return MD_ERR_ARG;
    if (T_fit > 0 && (!idx_l || (C && !idx_next))) return MD_ERR_ARG;
    cudaStream_t s = md::as_stream(stream);
    int rc = md::clear_status(dev_status, s);
    if (rc != MD_OK) return rc;
    const size_t table = (size_t)E * E * sizeof(uint32_t);
    if (!accumulate) {
        if (W) {
            md::count_memsets(1);
            if (cudaMemsetAsync(W, 0, table, s) != cudaSuccess) return MD_ERR_CUDA;
        }
        if (C) {
            md::count_memsets(1);
            if (cudaMemsetAsync(C, 0, table, s) != cudaSuccess) return MD_ERR_CUDA;
        }
    }
    if (T_fit == 0) return MD_OK;

    static std::atomic<uint64_t> attr_done{0};
    md::once_per_device(attr_done, [] {
        cudaFuncSetAttribute(k_coselect, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSegEntries * (int)sizeof(uint32_t));
    });
    const int64_t n_tri = (int64_t)E * (E + 1) / 2;
    const int64_t n_total = (W ? n_tri : 0) + (C ? (int64_t)E * E : 0);
    const int64_t n_seg = (n_total + kSegEntries - 1) / kSegEntries;
    const int64_t seg_len = (n_total + n_seg - 1) / n_seg;
    // about two CTAs per SM in total, at least 256 tokens per CTA
    int64_t nx = (2 * md::sm_count()) / n_seg;
    if (nx < 1) nx = 1;
    int64_t max_nx = (T_fit + 255) / 256;
    if (nx > max_nx) nx = max_nx;
    const int64_t tpb = (T_fit + nx - 1) / nx;
    nx = (T_fit + tpb - 1) / tpb;
    dim3 grid((unsigned)nx, (unsigned)n_seg);
    k_coselect<<<grid, kThreads, (size_t)seg_len * sizeof(uint32_t), s>>>(
        idx_l, idx_next, T_fit, E, k, tpb, W, C, n_tri, seg_len, dev_status);
    md::count_launches(1);
    return md::launch_status();
}

extern "C" int md_coselect_pair_stats(const int32_t *idx_prev, const int32_t *idx_l,
                                      const int32_t *idx_next, int64_t T_fit, int E, int k,
                                      uint32_t *C2, int accumulate, int32_t *dev_status,
                                      void *stream)
{
    if (T_fit < 0 || E < 1 || k < 1 || k > MD_MAX_TOPK || !C2) return MD_ERR_ARG;
    if (E > MD_MAX_PAIR_EXPERTS) return MD_ERR_UNSUPPORTED;
    if (T_fit > 0 && (!idx_prev || !idx_l || !idx_next)) return MD_ERR_ARG;
    cudaStream_t s = md::as_stream(stream);
    int rc = md::clear_status(dev_status, s);
    if (rc != MD_OK) return rc;
    if (!accumulate) {
        md::count_memsets(1);
        if (cudaMemsetAsync(C2, 0, (size_t)E * E * E * sizeof(uint32_t), s) != cudaSuccess)
            return MD_ERR_CUDA;
    }
    if (T_fit == 0) return MD_OK;
    int64_t blocks = (T_fit * k * k + 255) / 256;
    const int64_t cap = (int64_t)md::sm_count() * 16;
    if (blocks > cap) blocks = cap;
    k_coselect_pair<<<(unsigned)blocks, 256, 0, s>>>(idx_prev, idx_l, idx_next, T_fit, E, k, C2,
                                                     dev_status);
    md::count_launches(1);
    return md::launch_status();
}
