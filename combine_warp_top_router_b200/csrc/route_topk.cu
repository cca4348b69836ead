// route_topk.cu -- router top-k selection and gate weights (md_route_topk).
//
// "Expert Coupling in MoE Pretraining" (PicX summary), Background: every token
// is routed to its top-k of E experts; Method 1: the routing probabilities
// ride with the dispatched rows.
//
// One warp per token.  Lane L holds M of the token's E logits as order-
// preserving 32-bit keys (element index increases with the register slot).
// k rounds of a warp arg-max pick the experts: __reduce_max_sync finds the
// largest key, __reduce_min_sync the lowest expert holding it, and only the
// winning lane replaces its local best.  Keys compare exactly like the fp32
// logits with -0.0 folded onto +0.0, so ties go to the lower expert index.
// The gates are computed in double from exact logit differences and rounded
// to float once.
#include "common.cuh"

namespace {

constexpr int kThreads = 256;

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
template <int M, bool VEC>
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
__global__ void __launch_bounds__(kThreads)
    k_route_topk(const float *__restrict__ logits, int64_t T, int E, int k, int gate_mode,
                 int32_t *__restrict__ out_idx, float *__restrict__ out_w)
{
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * kThreads) >> 5;

    for (int64_t t = warp0; t < T; t += nwarps) {
        const float *row = logits + t * (int64_t)E;
        float val[M];
        uint32_t key[M];
        if (VEC) {
#pragma unroll
            for (int c = 0; c < M / 4; ++c) {
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (c * 128 < E) v = __ldcs(reinterpret_cast<const float4 *>(row + c * 128 + lane * 4));
                val[4 * c + 0] = v.x;
                val[4 * c + 1] = v.y;
                val[4 * c + 2] = v.z;
                val[4 * c + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int s = 0; s < M; ++s) {
                int e = s * 32 + lane;
                val[s] = e < E ? __ldcs(row + e) : 0.0f;
            }
        }
        uint32_t best = 0;
        int bs = 0;
#pragma unroll
        for (int s = 0; s < M; ++s) {
            key[s] = elem_of<M, VEC>(lane, s) < E ? float_key(val[s]) : 0u;
            if (key[s] > best) { best = key[s]; bs = s; }
        }

        int my_e = -1;
        uint32_t my_key = 0;
        double denom_full = 0.0;
        for (int r = 0; r < k; ++r) {
            const uint32_t kmax = __reduce_max_sync(0xffffffffu, best);
            const uint32_t cand = best == kmax ? (uint32_t)elem_of<M, VEC>(lane, bs) : 0xffffffffu;
            const uint32_t emin = __reduce_min_sync(0xffffffffu, cand);
            if (r == 0 && gate_mode == MD_GATE_FULL_SOFTMAX) {
                const double m = (double)key_float(kmax);
                double s = 0.0;
#pragma unroll
                for (int q = 0; q < M; ++q)
                    if (elem_of<M, VEC>(lane, q) < E) s += exp((double)val[q] - m);
                denom_full = warp_sum_d(s);
            }
            if (lane == r) { my_e = (int)emin; my_key = kmax; }
            if (cand == emin) {  // winning lane: drop the taken element, find the next best
                best = 0;
                bs = 0;
#pragma unroll
                for (int s = 0; s < M; ++s) {
                    if (elem_of<M, VEC>(lane, s) == (int)emin) key[s] = 0u;
                    if (key[s] > best) { best = key[s]; bs = s; }
                }
            }
        }

        // gates: exp of exact (double) differences to the largest logit
        const float m = __shfl_sync(0xffffffffu, key_float(my_key), 0);
        const double ex = lane < k ? exp((double)key_float(my_key) - (double)m) : 0.0;
        const double denom = gate_mode == MD_GATE_FULL_SOFTMAX ? denom_full : warp_sum_d(ex);
        if (lane < k) {
            out_idx[t * k + lane] = my_e;
            out_w[t * k + lane] = (float)(ex / denom);
        }
    }
}

template <int M, bool VEC>
void launch(const float *logits, int64_t T, int E, int k, int gate_mode, int32_t *idx, float *w,
            cudaStream_t s)
{
    int64_t blocks = (T + kThreads / 32 - 1) / (kThreads / 32);
    int64_t cap = (int64_t)md::sm_count() * 16;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    k_route_topk<M, VEC><<<(unsigned)blocks, kThreads, 0, s>>>(logits, T, E, k, gate_mode, idx, w);
    md::count_launches(1);
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
    const bool vec = (E % 128 == 0) && md::aligned16(logits);
    if (vec) {
        switch (E / 128) {
        case 1: launch<4, true>(logits, T, E, k, gate_mode, topk_idx, topk_w, s); break;
        case 2: launch<8, true>(logits, T, E, k, gate_mode, topk_idx, topk_w, s); break;
        case 3:
        case 4: launch<16, true>(logits, T, E, k, gate_mode, topk_idx, topk_w, s); break;
        default: launch<32, true>(logits, T, E, k, gate_mode, topk_idx, topk_w, s); break;
        }
    } else {
        const int m = (E + 31) / 32;
        if (m <= 1) launch<1, false>(logits, T, E, k, gate_mode, topk_idx, topk_w, s);
        else if (m <= 2) launch<2, false>(logits, T, E, k, gate_mode, topk_idx, topk_w, s);
        else if (m <= 4) launch<4, false>(logits, T, E, k, gate_mode, topk_idx, topk_w, s);
        else if (m <= 8) launch<8, false>(logits, T, E, k, gate_mode, topk_idx, topk_w, s);
        else if (m <= 16) launch<16, false>(logits, T, E, k, gate_mode, topk_idx, topk_w, s);
        else launch<32, false>(logits, T, E, k, gate_mode, topk_idx, topk_w, s);
    }
    return md::launch_status();
}
