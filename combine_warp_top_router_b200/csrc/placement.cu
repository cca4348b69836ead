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
// One CTA of 1024 threads does the whole search.  Each step evaluates every
// candidate pair in parallel and picks the best with a block arg-max (gain
// descending, then lowest expert pair), so the result is deterministic.
//   Greedy seed: the scan of pairs by weight places a pair only while it is
//   eligible, and eligibility never comes back once lost (ranks only fill
//   up), so "take the heaviest pair that is still eligible" repeated until
//   none is left places the same pairs as the ordered scan.
//   Refinement: A[e][d] = sum of W[e][e'] over e' != e on rank d is kept in
//   the workspace; swapping a (rank P) with b (rank Q) gains
//   A[a][Q] - A[a][P] + A[b][P] - A[b][Q] - 2 W[a][b], and only columns P
//   and Q of A change.
#include "common.cuh"

namespace {

constexpr int kThreads = 1024;

struct Cand {
    long long g;
    int a, b;
};

__device__ __forceinline__ bool better(const Cand &x, const Cand &y)
{
    if (x.a < 0) return false;
    if (y.a < 0) return true;
    if (x.g != y.g) return x.g > y.g;
    if (x.a != y.a) return x.a < y.a;
    return x.b < y.b;
}

// Block-wide best candidate; every thread gets the result.
__device__ Cand block_best(Cand v, Cand *s_red, Cand *s_out)
{
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        Cand u;
        u.g = __shfl_xor_sync(0xffffffffu, v.g, o);
        u.a = __shfl_xor_sync(0xffffffffu, v.a, o);
        u.b = __shfl_xor_sync(0xffffffffu, v.b, o);
        if (better(u, v)) v = u;
    }
    if (lane == 0) s_red[w] = v;
    __syncthreads();
    if (w == 0) {
        v = s_red[lane];  // kThreads / 32 == 32 warps
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            Cand u;
            u.g = __shfl_xor_sync(0xffffffffu, v.g, o);
            u.a = __shfl_xor_sync(0xffffffffu, v.a, o);
            u.b = __shfl_xor_sync(0xffffffffu, v.b, o);
            if (better(u, v)) v = u;
        }
        if (lane == 0) *s_out = v;
    }
    __syncthreads();
    Cand r = *s_out;
    __syncthreads();
    return r;
}

__global__ void __launch_bounds__(kThreads)
    k_place(const uint32_t *__restrict__ W, int E, int R, int seed_mode, int refine,
            int32_t *__restrict__ p_out, long long *__restrict__ A)
{
    extern __shared__ int sm[];
    int *s_p = sm;          // [E] rank of each expert (-1: not placed yet)
    int *s_fill = s_p + E;  // [R] experts on each rank
    __shared__ Cand s_red[32], s_out;
    __shared__ int s_roomiest;
    const int tid = threadIdx.x;
    const int cap = E / R;
    const int64_t cells = (int64_t)E * E;

    if (seed_mode == MD_SEED_CONTIGUOUS) {
        for (int e = tid; e < E; e += kThreads) s_p[e] = e / cap;
        __syncthreads();
    } else {
        for (int e = tid; e < E; e += kThreads) s_p[e] = -1;
        for (int d = tid; d < R; d += kThreads) s_fill[d] = 0;
        __syncthreads();
        for (int it = 0; it < E; ++it) {
            if (tid == 0) {
                int b = 0;
                for (int d = 1; d < R; ++d)
                    if (s_fill[d] < s_fill[b]) b = d;
                s_roomiest = b;
            }
            __syncthreads();
            const int roomiest = s_roomiest;
            const int maxfree = cap - s_fill[roomiest];
            Cand v = {0, -1, -1};
            for (int64_t cell = tid; cell < cells; cell += kThreads) {
                const int a = (int)(cell / E), b = (int)(cell - (int64_t)a * E);
                if (b <= a) continue;
                const uint32_t wv = W[cell];
                if (wv == 0u) continue;
                const int pa = s_p[a], pb = s_p[b];
                bool ok;
                if (pa < 0 && pb < 0) ok = maxfree >= 2;
                else if (pa >= 0 && pb < 0) ok = s_fill[pa] < cap;
                else if (pa < 0 && pb >= 0) ok = s_fill[pb] < cap;
                else ok = false;
                if (ok) {
                    const Cand c = {(long long)wv, a, b};
                    if (better(c, v)) v = c;
                }
            }
            const Cand win = block_best(v, s_red, &s_out);
            if (win.a < 0) break;
            if (tid == 0) {
                const int pa = s_p[win.a], pb = s_p[win.b];
                if (pa < 0 && pb < 0) {
                    s_p[win.a] = roomiest;
                    s_p[win.b] = roomiest;
                    s_fill[roomiest] += 2;
                } else if (pa >= 0) {
                    s_p[win.b] = pa;
                    s_fill[pa] += 1;
                } else {
                    s_p[win.a] = pb;
                    s_fill[pb] += 1;
                }
            }
            __syncthreads();
        }
        if (tid == 0) {
            for (int e = 0; e < E; ++e) {
                if (s_p[e] >= 0) continue;
                for (int d = 0; d < R; ++d)
                    if (s_fill[d] < cap) {
                        s_p[e] = d;
                        s_fill[d] += 1;
                        break;
                    }
            }
        }
        __syncthreads();
    }

    if (refine) {
        for (int e = tid; e < E; e += kThreads) {
            long long *row = A + (int64_t)e * R;
            for (int d = 0; d < R; ++d) row[d] = 0;
            for (int e2 = 0; e2 < E; ++e2)
                if (e2 != e) row[s_p[e2]] += W[(int64_t)e * E + e2];
        }
        __syncthreads();
        for (long long it = 0; it < (long long)E * E; ++it) {
            Cand v = {0, -1, -1};
            for (int64_t cell = tid; cell < cells; cell += kThreads) {
                const int a = (int)(cell / E), b = (int)(cell - (int64_t)a * E);
                if (b <= a) continue;
                const int P = s_p[a], Q = s_p[b];
                if (P == Q) continue;
                const long long g = A[(int64_t)a * R + Q] - A[(int64_t)a * R + P] +
                                    A[(int64_t)b * R + P] - A[(int64_t)b * R + Q] -
                                    2ll * (long long)W[cell];
                if (g > 0) {
                    const Cand c = {g, a, b};
                    if (better(c, v)) v = c;
                }
            }
            const Cand win = block_best(v, s_red, &s_out);
            if (win.a < 0) break;
            const int a = win.a, b = win.b, P = s_p[a], Q = s_p[b];
            for (int e = tid; e < E; e += kThreads) {
                const long long wa = e != a ? (long long)W[(int64_t)e * E + a] : 0;
                const long long wb = e != b ? (long long)W[(int64_t)e * E + b] : 0;
                A[(int64_t)e * R + P] += wb - wa;
                A[(int64_t)e * R + Q] += wa - wb;
            }
            __syncthreads();
            if (tid == 0) {
                s_p[a] = Q;
                s_p[b] = P;
            }
            __syncthreads();
        }
    }
    for (int e = tid; e < E; e += kThreads) p_out[e] = s_p[e];
}

}  // namespace

extern "C" size_t md_place_correlated_workspace_size(int E, int R)
{
    if (E < 1 || R < 1) return 0;
    return md::align_up((size_t)E * R * sizeof(long long), 256);
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
    k_place<<<1, kThreads, (size_t)(E + R) * sizeof(int), s>>>(
        W, E, R, seed_mode, refine ? 1 : 0, expert_to_rank, static_cast<long long *>(workspace));
    md::count_launches(1);
    return md::launch_status();
}
