// route_topk.cu -- router top-k selection and gate weights (md_route_topk).
//
// "Expert Coupling in MoE Pretraining" (PicX summary), Background: every token
// is routed to its top-k of E experts; Method 1: the routing probabilities
// ride with the dispatched rows.
//
// Two kernels.  E in {64, 128, 256} with k in {1, 2, 4, 6, 8} (16-byte
// aligned logits) takes k_route_topk_tpt, one thread per token (described
// below it).  Every other shape takes k_route_topk:
//
// One warp per token.  Lane L holds M of the token's E logits as order-
// preserving 32-bit keys (element index increases with the register slot);
// keys compare exactly like the fp32 logits with -0.0 folded onto +0.0, and
// equal keys go to the lower expert index.
//
// Fast path: the k-th largest of the 32 lane maxima is a lower bound on the
// k-th largest logit (k lane maxima are k distinct logits at or above it), so
// every top-k element is at or above it.  The few candidates that pass
// (typically k to 2k) are compacted one per lane, and k rounds of
// __reduce_max_sync / __reduce_min_sync pick them in order.  If more than 32
// pass (heavy ties), the exact slow path runs instead: k rounds of the same
// warp arg-max over all elements, with the winning lane rescanning its own.
//
// A warp handles G = floor(32/k) tokens back to back and keeps token g's slot
// r in lane g*k + r, so the gates of the whole group are computed at once:
// exp of exact (double) logit differences to the token's largest logit, a
// double sum in slot order, one rounding to float.
#include "common.cuh"

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ uint32_t float_key(float f)
{
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;  // -0.0 compares equal to +0.0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_float(uint32_t k)
{
    uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
    return __uint_as_float(u);
}

// Element held in register slot s of `lane`.
template <bool VEC>
__device__ __forceinline__ int elem_of(int lane, int s)
{
    return VEC ? (s >> 2) * 128 + lane * 4 + (s & 3) : s * 32 + lane;
}

__device__ __forceinline__ double warp_sum_d(double v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

template <int M, bool VEC>
__device__ __forceinline__ void load_row(float (&v)[M], const float *row, int E, int lane)
{
    if (VEC) {
#pragma unroll
        for (int c = 0; c < M / 4; ++c) {
            float4 q = make_float4(0.f, 0.f, 0.f, 0.f);
            if (c * 128 < E) q = __ldcs(reinterpret_cast<const float4 *>(row + c * 128 + lane * 4));
            v[4 * c + 0] = q.x;
            v[4 * c + 1] = q.y;
            v[4 * c + 2] = q.z;
            v[4 * c + 3] = q.w;
        }
    } else {
#pragma unroll
        for (int s = 0; s < M; ++s) {
            const int e = s * 32 + lane;
            v[s] = e < E ? __ldcs(row + e) : 0.0f;
        }
    }
}

template <int M, bool VEC, int KC>
__global__ void __launch_bounds__(kThreads)
    k_route_topk(const float *__restrict__ logits, int64_t T, int E, int k_rt, int gate_mode,
                 int32_t *__restrict__ out_idx, float *__restrict__ out_w)
{
    __shared__ uint32_t s_ck[kWarps][32];
    __shared__ int s_ce[kWarps][32];
    const int k = KC ? KC : k_rt;  // compile-time for the common k
    const int lane = threadIdx.x & 31, wl = threadIdx.x >> 5;
    const int G = 32 / k;  // tokens per warp group
    const int64_t warp0 = (int64_t)blockIdx.x * kWarps + wl;
    const int64_t nwarps = (int64_t)gridDim.x * kWarps;

    // token sequence of this warp: groups tg = (warp0 + i*nwarps)*G, tokens tg .. tg+G-1;
    // the next token's logits are loaded while the current one is processed
    float cur[M];
    const int64_t first = warp0 * G;
    if (first < T) load_row<M, VEC>(cur, logits + first * (int64_t)E, E, lane);
    for (int64_t tg = first; tg < T; tg += nwarps * G) {
        int my_e = -1;          // lane g*k + r: expert of token tg+g, slot r
        uint32_t my_key = 0;
        double my_den = 1.0;    // full-softmax denominator of that token
        const int ng = (int)(T - tg < G ? T - tg : G);
        for (int g = 0; g < ng; ++g) {
            const int64_t tn = g + 1 < ng ? tg + g + 1 : tg + nwarps * G;
            float val[M];
#pragma unroll
            for (int s = 0; s < M; ++s) val[s] = cur[s];
            if (tn < T) load_row<M, VEC>(cur, logits + tn * (int64_t)E, E, lane);
            uint32_t key[M];
            uint32_t best = 0;
            int bs = 0;
#pragma unroll
            for (int s = 0; s < M; ++s) {
                key[s] = elem_of<VEC>(lane, s) < E ? float_key(val[s]) : 0u;
                if (key[s] > best) { best = key[s]; bs = s; }
            }
            if (gate_mode == MD_GATE_FULL_SOFTMAX) {
                const double m = (double)key_float(__reduce_max_sync(0xffffffffu, best));
                double s = 0.0;
#pragma unroll
                for (int q = 0; q < M; ++q)
                    if (elem_of<VEC>(lane, q) < E) s += exp((double)val[q] - m);
                s = warp_sum_d(s);
                if (lane >= g * k && lane < (g + 1) * k) my_den = s;
            }

            // threshold: the k-th largest lane maximum
            uint32_t act = best, th = 0;
#pragma unroll
            for (int r = 0; r < (KC ? KC : MD_MAX_TOPK); ++r) {
                if (!KC && r >= k) break;
                th = __reduce_max_sync(0xffffffffu, act);
                const unsigned b = __ballot_sync(0xffffffffu, act == th);
                if (lane == __ffs(b) - 1) act = 0u;
            }
            int c = 0;
#pragma unroll
            for (int s = 0; s < M; ++s) c += key[s] >= th ? 1 : 0;
            int incl = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const int ncand = __shfl_sync(0xffffffffu, incl, 31);

            if (ncand <= 32) {
                int pos = incl - c;
#pragma unroll
                for (int s = 0; s < M; ++s)
                    if (key[s] >= th) {
                        s_ck[wl][pos] = key[s];
                        s_ce[wl][pos] = elem_of<VEC>(lane, s);
                        ++pos;
                    }
                __syncwarp();
                uint32_t ck = lane < ncand ? s_ck[wl][lane] : 0u;
                const uint32_t ce = lane < ncand ? (uint32_t)s_ce[wl][lane] : 0xffffffffu;
                __syncwarp();
#pragma unroll
                for (int r = 0; r < (KC ? KC : MD_MAX_TOPK); ++r) {
                    if (!KC && r >= k) break;
                    const uint32_t kmax = __reduce_max_sync(0xffffffffu, ck);
                    const uint32_t cand = ck == kmax ? ce : 0xffffffffu;
                    const uint32_t emin = __reduce_min_sync(0xffffffffu, cand);
                    if (cand == emin) ck = 0u;
                    if (lane == g * k + r) { my_e = (int)emin; my_key = kmax; }
                }
            } else {
                // exact fallback over all elements
                for (int r = 0; r < k; ++r) {
                    const uint32_t kmax = __reduce_max_sync(0xffffffffu, best);
                    const uint32_t cand = best == kmax ? (uint32_t)elem_of<VEC>(lane, bs) : 0xffffffffu;
                    const uint32_t emin = __reduce_min_sync(0xffffffffu, cand);
                    if (lane == g * k + r) { my_e = (int)emin; my_key = kmax; }
                    if (cand == emin) {
                        best = 0;
                        bs = 0;
#pragma unroll
                        for (int s = 0; s < M; ++s) {
                            if (elem_of<VEC>(lane, s) == (int)emin) key[s] = 0u;
                            if (key[s] > best) { best = key[s]; bs = s; }
                        }
                    }
                }
            }
        }

        // gates of the whole group: lane g*k + r holds token g's slot r
        const int base = (lane / k) * k;
        const bool live = lane < ng * k;
        const float v = key_float(my_key);
        const float m = __shfl_sync(0xffffffffu, v, base < 32 ? base : 0);
        const double ex = live ? exp((double)v - (double)m) : 0.0;
        double den;
        if (gate_mode == MD_GATE_FULL_SOFTMAX) {
            den = my_den;
        } else {
            den = 0.0;
#pragma unroll
            for (int r = 0; r < (KC ? KC : MD_MAX_TOPK); ++r) {
                if (!KC && r >= k) break;
                const int src = base + r;
                den += __shfl_sync(0xffffffffu, ex, src < 32 ? src : 0);
            }
        }
        if (live) {
            out_idx[tg * k + lane] = my_e;
            out_w[tg * k + lane] = (float)(ex / den);
        }
    }
}

template <int M, bool VEC, int KC>
void launch(const float *logits, int64_t T, int E, int k, int gate_mode, int32_t *idx, float *w,
            cudaStream_t s)
{
    const int64_t G = 32 / k;
    int64_t blocks = (T + kWarps * G - 1) / (kWarps * G);
    const int64_t cap = (int64_t)md::sm_count() * 16;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    k_route_topk<M, VEC, KC><<<(unsigned)blocks, kThreads, 0, s>>>(logits, T, E, k, gate_mode, idx, w);
    md::count_launches(1);
}

// 16-byte loads; the common k are compile-time constants
template <int M>
void launch_k(const float *logits, int64_t T, int E, int k, int gate_mode, int32_t *idx, float *w,
              cudaStream_t s)
{
    switch (k) {
    case 1: launch<M, true, 1>(logits, T, E, k, gate_mode, idx, w, s); break;
    case 2: launch<M, true, 2>(logits, T, E, k, gate_mode, idx, w, s); break;
    case 4: launch<M, true, 4>(logits, T, E, k, gate_mode, idx, w, s); break;
    case 6: launch<M, true, 6>(logits, T, E, k, gate_mode, idx, w, s); break;
    case 8: launch<M, true, 8>(logits, T, E, k, gate_mode, idx, w, s); break;
    default: launch<M, true, 0>(logits, T, E, k, gate_mode, idx, w, s); break;
    }
}

// ---------------------------------------------------------------- thread per token
// E in {64, 128, 256}, k in {1, 2, 4, 6, 8}: one thread per token, so the
// selection needs no cross-lane steps.  A warp stages its 32 consecutive rows
// (contiguous in memory) in shared memory with one bulk copy.  At iteration c
// lane L reads its row's 16-byte chunk c xor (L mod 8), which puts the 8
// lanes of a shared-memory phase on distinct banks.
//   1. Threshold.  Chunk iteration c belongs to group c mod 16; the k-th
//      largest of the 16 group maxima is at or below the k-th largest logit
//      (k group maxima are k distinct elements at or above it).
//   2. Candidates.  Only groups whose maximum reaches the threshold (k or a
//      few more of the 16) are read again; their elements at or above it
//      (about 10 for k = 8) are compacted into a per-lane list of expert
//      indices (64 entries, so a sixth warp fits an SM at E = 256; appends
//      past the end land on the last entry without a branch, and a lane
//      with more candidates ranks them by insertion over its row instead).
//   3. Selection.  Candidates become exact 64-bit keys (order-preserving
//      logit key, then the complement of the expert index, so that equal
//      logits go to the lower index).  Batches of 8 are sorted by a 19-
//      comparator network and merged into the running sorted top 8: the
//      pairwise maxima of two sorted lists, one reversed, are the union's top 8
//      as a bitonic sequence, which a 12-comparator bitonic merge sorts.
// The gates are computed as in the warp kernel, one token per thread.
constexpr int kTptGroups = 16;
constexpr long long kTptPolls = 1ll << 22;

// descending compare-exchange
__device__ __forceinline__ void cx(uint64_t &a, uint64_t &b)
{
    const uint64_t hi = a > b ? a : b;
    b = a > b ? b : a;
    a = hi;
}

__device__ __forceinline__ void cx(float &a, float &b)
{
    const float hi = fmaxf(a, b);
    b = fminf(a, b);
    a = hi;
}

// Batcher's odd-even merge sort of 8, descending
template <typename V>
__device__ __forceinline__ void sort8(V (&a)[8])
{
    cx(a[0], a[1]); cx(a[2], a[3]); cx(a[4], a[5]); cx(a[6], a[7]);
    cx(a[0], a[2]); cx(a[1], a[3]); cx(a[4], a[6]); cx(a[5], a[7]);
    cx(a[1], a[2]); cx(a[5], a[6]); cx(a[0], a[4]); cx(a[3], a[7]);
    cx(a[1], a[5]); cx(a[2], a[6]);
    cx(a[1], a[4]); cx(a[3], a[6]);
    cx(a[2], a[4]); cx(a[3], a[5]);
    cx(a[3], a[4]);
}

// sorts a bitonic sequence of 8, descending
__device__ __forceinline__ void bitonic8(uint64_t (&a)[8])
{
#pragma unroll
    for (int d = 4; d >= 1; d >>= 1)
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if ((i & d) == 0) cx(a[i], a[i + d]);
}

__device__ __forceinline__ uint64_t cand_key(float v, int e)
{
    return ((uint64_t)float_key(v) << 32) | (uint64_t)(0xffffu - (uint32_t)e);
}

template <int E>
constexpr int tpt_cap() { return E > 64 ? 64 : E; }  // candidate list entries per lane
template <int E>
constexpr size_t tpt_smem() { return (size_t)32 * E * 4 + (size_t)32 * tpt_cap<E>(); }

// One warp per CTA, one tile of 32 consecutive tokens (one per lane).
template <int E, int KC>
__global__ void __launch_bounds__(32)
    k_route_topk_tpt(const float *__restrict__ logits, int64_t T, int gate_mode,
                     int32_t *__restrict__ out_idx, float *__restrict__ out_w, int vec_out,
                     long long polls)
{
    constexpr int NCH = E / 4;
    constexpr int NG = kTptGroups;
    constexpr int CAP = tpt_cap<E>();
    __shared__ float s_th[32];
    static_assert(KC >= 1 && KC <= 8 && NCH >= NG && (NCH & (NCH - 1)) == 0, "shape");
    extern __shared__ __align__(16) unsigned char smem[];
    float *rows = reinterpret_cast<float *>(smem);                      // [32][E]
    const int lane = threadIdx.x;
    uint8_t *lst = smem + (size_t)32 * E * 4 + lane;                    // slot s at lst[32 s]
    const int64_t t0 = (int64_t)blockIdx.x * 32;
    const int ntok = (int)(T - t0 < 32 ? T - t0 : 32);
    {
        // the tile's rows are contiguous: one bulk copy, completing on an
        // mbarrier every lane waits on (bounded; if the bound runs out, the
        // lanes copy the same bytes with plain loads, so a late bulk copy can
        // only rewrite identical values)
        __shared__ uint64_t bar;
        const uint32_t bytes = (uint32_t)(ntok * E * 4);
        if (lane == 0) {
            md::mbar_init(&bar, 1);
            md::fence_mbar_init();
        }
        __syncwarp();
        if (lane == 0) {
            md::mbar_expect_tx(&bar, bytes);
            md::bulk_load(rows, logits + t0 * E, bytes, &bar);
        }
        const bool ok = md::mbar_wait_bounded(&bar, 0u, polls);
        if (!__all_sync(0xffffffffu, ok)) {
            const float4 *src = reinterpret_cast<const float4 *>(logits + t0 * E);
            float4 *dst = reinterpret_cast<float4 *>(rows);
            for (int i = lane; i < ntok * NCH; i += 32) dst[i] = __ldg(src + i);
            // let the late copy land (bounded again, at the default limit)
            // before the rows are read, so it cannot arrive after the CTA
            md::mbar_wait_bounded(&bar, 0u, kTptPolls);
        }
        __syncwarp();
    }
    const bool live = lane < ntok;
    const float *row = rows + lane * E;
    const float4 *row4 = reinterpret_cast<const float4 *>(row);

    // 1-2. threshold and candidate list
    int n = 0;
    if (live) {
        // iteration c reads chunk c ^ (lane & 7): the 8 lanes of a shared-
        // memory phase hit distinct banks, and with the 8 row pointers below
        // each read is one load at a constant offset
        const int sw = lane & 7;
        const float4 *rb[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) rb[q] = row4 + (q ^ sw);
        float gm[NG];
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            const float4 q = rb[c & 7][c & ~7];
            const float m = fmaxf(fmaxf(q.x, q.y), fmaxf(q.z, q.w));
            gm[c % NG] = c < NG ? m : fmaxf(gm[c % NG], m);
        }
        float a[8], b[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            a[i] = gm[i];
            b[i] = gm[8 + i];
        }
        sort8(a);
        sort8(b);
        // k-th largest of the union of two descending lists
        float th = fmaxf(a[KC - 1], b[KC - 1]);
#pragma unroll
        for (int i = 1; i < KC; ++i) th = fmaxf(th, fminf(a[i - 1], b[KC - i - 1]));

        // only a group whose maximum reaches the threshold can hold a
        // candidate: k or a few more of the 16, so about half the chunks
        uint32_t gmask = 0u;
#pragma unroll
        for (int g = 0; g < NG; ++g)
            if (gm[g] >= th) gmask |= 1u << g;
        while (gmask) {
            const int g = __ffs(gmask) - 1;
            gmask &= gmask - 1;
#pragma unroll
            for (int j = 0; j < NCH / NG; ++j) {  // iterations g, g + 16, ... of the first pass
                const int ch = (g + NG * j) ^ sw;
                const float4 q = row4[ch];
                const int e0 = ch * 4;
                if (q.x >= th) { lst[32 * min(n, CAP - 1)] = (uint8_t)e0; ++n; }
                if (q.y >= th) { lst[32 * min(n, CAP - 1)] = (uint8_t)(e0 + 1); ++n; }
                if (q.z >= th) { lst[32 * min(n, CAP - 1)] = (uint8_t)(e0 + 2); ++n; }
                if (q.w >= th) { lst[32 * min(n, CAP - 1)] = (uint8_t)(e0 + 3); ++n; }
            }
        }
        s_th[lane] = th;  // for the overflow path below
        if (n < KC) {
            // fewer than k candidates happens only with NaN logits (outside
            // the contract): every element becomes a candidate, through the
            // overflow path, so the indices stay valid and distinct
            n = E + 1;
        }
    }

    // 3. sorted top 8 of the candidates, batches of 8
    const int nb = n > CAP ? 0 : n;
    const int nmax = (int)__reduce_max_sync(0xffffffffu, (unsigned)nb);
    uint64_t best[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) best[i] = 0ull;
    for (int s = 0; s < nmax; s += 8) {
        uint64_t bt[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            uint64_t key = 0ull;  // below every logit's key
            if (s + j < nb) {
                const int e = lst[32 * (s + j)];
                key = cand_key(row[e], e);
            }
            bt[j] = key;
        }
        sort8(bt);
        if (s == 0) {
#pragma unroll
            for (int i = 0; i < 8; ++i) best[i] = bt[i];
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) best[i] = best[i] > bt[7 - i] ? best[i] : bt[7 - i];
            bitonic8(best);
        }
    }
    // a lane with more candidates than its list holds (heavy ties, NaN rows)
    // inserts them into its sorted top 8 straight from the row; the loop is
    // kept compact so that it costs the common path nothing
    if (__any_sync(0xffffffffu, n > CAP) && n > CAP) {
        const float th = s_th[lane];
        const bool all = n > E;  // NaN row: every element
#pragma unroll 1
        for (int e = 0; e < E; ++e) {
            const float v = row[e];
            if (!(all || v >= th)) continue;
            uint64_t key = cand_key(v, e);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint64_t hi = best[i] > key ? best[i] : key;
                key = best[i] > key ? key : best[i];
                best[i] = hi;
            }
        }
    }
    if (!live) return;

    const int64_t t = t0 + lane;
    int sel[KC];
    double ex[KC];
    const double m = (double)key_float((uint32_t)(best[0] >> 32));
    double den = 0.0;
#pragma unroll
    for (int r = 0; r < KC; ++r) {
        sel[r] = (int)(0xffffu - (uint32_t)(best[r] & 0xffffffffu));
        // slot 0 holds the largest logit m itself: exp(0) = 1 exactly
        ex[r] = r == 0 ? 1.0 : exp((double)key_float((uint32_t)(best[r] >> 32)) - m);
        den += ex[r];
    }
    if (gate_mode == MD_GATE_FULL_SOFTMAX) {
        den = 0.0;
#pragma unroll 4
        for (int c = 0; c < NCH; ++c) {
            const float4 q = row4[(c + lane) & (NCH - 1)];
            den += exp((double)q.x - m) + exp((double)q.y - m) + exp((double)q.z - m) +
                   exp((double)q.w - m);
        }
    }
    // one reciprocal; each quotient stays within a double ulp or two of
    // ex / den before its single rounding to float
    const double inv = 1.0 / den;
    float w[KC];
#pragma unroll
    for (int r = 0; r < KC; ++r) w[r] = (float)(ex[r] * inv);
    if (vec_out && KC % 4 == 0) {
#pragma unroll
        for (int q = 0; q < KC / 4; ++q) {
            reinterpret_cast<int4 *>(out_idx + t * KC)[q] =
                make_int4(sel[4 * q], sel[4 * q + 1], sel[4 * q + 2], sel[4 * q + 3]);
            reinterpret_cast<float4 *>(out_w + t * KC)[q] =
                make_float4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
        }
    } else {
#pragma unroll
        for (int r = 0; r < KC; ++r) {
            out_idx[t * KC + r] = sel[r];
            out_w[t * KC + r] = w[r];
        }
    }
}

template <int E, int KC>
void launch_tpt(const float *logits, int64_t T, int gate_mode, int32_t *idx, float *w, cudaStream_t s)
{
    static std::atomic<uint64_t> attr_done{0};
    md::once_per_device(attr_done, [] {
        cudaFuncSetAttribute(k_route_topk_tpt<E, KC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)tpt_smem<E>());
    });
    const int vec = md::aligned16(idx) && md::aligned16(w);
    const int64_t blocks = (T + 31) / 32;
    k_route_topk_tpt<E, KC><<<(unsigned)blocks, 32, tpt_smem<E>(), s>>>(logits, T, gate_mode, idx, w, vec,
                                                                       md::hook_poll_limit(kTptPolls));
    md::count_launches(1);
}

template <int E>
bool try_tpt(const float *logits, int64_t T, int k, int gate_mode, int32_t *idx, float *w, cudaStream_t s)
{
    switch (k) {
    case 1: launch_tpt<E, 1>(logits, T, gate_mode, idx, w, s); return true;
    case 2: launch_tpt<E, 2>(logits, T, gate_mode, idx, w, s); return true;
    case 4: launch_tpt<E, 4>(logits, T, gate_mode, idx, w, s); return true;
    case 6: launch_tpt<E, 6>(logits, T, gate_mode, idx, w, s); return true;
    case 8: launch_tpt<E, 8>(logits, T, gate_mode, idx, w, s); return true;
    default: return false;
    }
}

}  // namespace

extern "C" int md_route_topk(const float *logits, int64_t T, int E, int k, int gate_mode,
                             int32_t *topk_idx, float *topk_w, void *stream)
{
    if (T < 0 || E < 1 || k < 1 || k > E || k > MD_MAX_TOPK) return MD_ERR_ARG;
    if (E > MD_MAX_EXPERTS) return MD_ERR_UNSUPPORTED;
    if (gate_mode != MD_GATE_TOPK_SOFTMAX && gate_mode != MD_GATE_FULL_SOFTMAX) return MD_ERR_ARG;
    if (T == 0) return MD_OK;
    if (!logits || !topk_idx || !topk_w) return MD_ERR_ARG;
    cudaStream_t s = md::as_stream(stream);
    if (md::aligned16(logits)) {
        bool done = false;
        if (E == 64) done = try_tpt<64>(logits, T, k, gate_mode, topk_idx, topk_w, s);
        else if (E == 128) done = try_tpt<128>(logits, T, k, gate_mode, topk_idx, topk_w, s);
        else if (E == 256) done = try_tpt<256>(logits, T, k, gate_mode, topk_idx, topk_w, s);
        if (done) return md::launch_status();
    }
    const bool vec = (E % 128 == 0) && md::aligned16(logits);
    if (vec) {
        switch (E / 128) {
        case 1: launch_k<4>(logits, T, E, k, gate_mode, topk_idx, topk_w, s); break;
        case 2: launch_k<8>(logits, T, E, k, gate_mode, topk_idx, topk_w, s); break;
        case 3:
        case 4: launch_k<16>(logits, T, E, k, gate_mode, topk_idx, topk_w, s); break;
        default: launch_k<32>(logits, T, E, k, gate_mode, topk_idx, topk_w, s); break;
        }
    } else {
        const int m = (E + 31) / 32;
        if (m <= 1) launch<1, false, 0>(logits, T, E, k, gate_mode, topk_idx, topk_w, s);
        else if (m <= 2) launch<2, false, 0>(logits, T, E, k, gate_mode, topk_idx, topk_w, s);
        else if (m <= 4) launch<4, false, 0>(logits, T, E, k, gate_mode, topk_idx, topk_w, s);
        else if (m <= 8) launch<8, false, 0>(logits, T, E, k, gate_mode, topk_idx, topk_w, s);
        else if (m <= 16) launch<16, false, 0>(logits, T, E, k, gate_mode, topk_idx, topk_w, s);
        else launch<32, false, 0>(logits, T, E, k, gate_mode, topk_idx, topk_w, s);
    }
    return md::launch_status();
}
