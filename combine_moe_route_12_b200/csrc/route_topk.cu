// Step 1: router top-k with renormalised softmax weights (LightLLM PR 1687,
// _select_experts with norm_topk_prob; axolotl ExpertParallelArgs: the routing
// top-k is saved state), and its variants: grouped top-k (the experts() path of
// the same page) and a bias that steers the selection only.
//
// Plain top-k: one warp per token.  Lane l holds the biased logits of experts
// l, l+32, ... as 32-bit order keys (the fp32 bits mapped so that unsigned order
// is value order) and tracks its best remaining one (the lowest expert among
// equal values).  A round is two warp reductions in hardware (redux.sync): the
// largest key over the lanes, then the lowest expert among the lanes holding it;
// lane j keeps slot j, and only the winning lane rescans its few values.  The
// next token's logits are loaded while the current token's rounds run.
// Grouped top-k: a group of LPT lanes (8, 16 or 32) per token, 32/LPT tokens per
// warp at a time.  Lane l of a group holds the biased logits of experts l, l+LPT,
// ... as 64-bit rank keys (value descending, lower expert index first among equal
// values).  k rounds of a butterfly max over the lanes' best remaining keys pick
// the experts in rank order; lane j of the group keeps slot j, and only the lane
// whose key won rescans its values.
// The weights w_j = exp(l_j - l_0) / sum_i exp(l_i - l_0) use a fixed fp32
// exponential (Cody & Waite reduction, degree-7 Taylor polynomial, every step
// one IEEE-rounded operation) and a slot-ordered sum, so they are bit-exact
// against any implementation that performs the same operations.
#include "moe_common.cuh"

namespace moe {

// e^r for r <= 0 in fp32.  Derivation:
//   n = rint(r * log2(e)),  f = r - n ln2 (ln2 = hi + lo, hi = 45426 / 2^16 has
//   16 significant bits so n*hi and r - n*hi are exact for |n| <= 127),
//   e^f by Horner on the Taylor series to degree 7 (|f| <= ln2/2 leaves a
//   truncation error near 5e-9), then scaled by 2^n through the exponent field.
__device__ __forceinline__ float det_exp_nonpos(float r) {
    constexpr double kLn2 = 0.69314718055994530941723212145818;
    constexpr float kLog2e = (float)(1.0 / kLn2);
    constexpr float kLn2Hi = 45426.0f / 65536.0f;
    constexpr float kLn2Lo = (float)(kLn2 - 45426.0 / 65536.0);
    constexpr float kC7 = (float)(1.0 / 5040.0), kC6 = (float)(1.0 / 720.0),
                    kC5 = (float)(1.0 / 120.0), kC4 = (float)(1.0 / 24.0),
                    kC3 = (float)(1.0 / 6.0), kC2 = 0.5f, kC1 = 1.0f, kC0 = 1.0f;
    if (r < -87.0f) return 0.0f;
    const float n = rintf(__fmul_rn(r, kLog2e));
    float f = __fmaf_rn(-n, kLn2Hi, r);
    f = __fmaf_rn(-n, kLn2Lo, f);
    float p = kC7;
    p = __fmaf_rn(p, f, kC6);
    p = __fmaf_rn(p, f, kC5);
    p = __fmaf_rn(p, f, kC4);
    p = __fmaf_rn(p, f, kC3);
    p = __fmaf_rn(p, f, kC2);
    p = __fmaf_rn(p, f, kC1);
    p = __fmaf_rn(p, f, kC0);
    const float two_n = __int_as_float(((int)n + 127) << 23);
    return __fmul_rn(p, two_n);
}


// Rank key of (biased logit l, expert e): larger l first, lower e among equal
// l.  The fp32 bits are mapped to an unsigned order (negatives flipped) in the
// high word and the complemented expert index fills the low word, so one 64-bit
// comparison ranks two candidates; 0 is below every real key (empty slot).
__device__ __forceinline__ uint64_t rank_key(float l, int e) {
    const uint32_t u = __float_as_uint(l);
    const uint32_t ord = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ((uint64_t)ord << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)e);
}
__device__ __forceinline__ float key_value(uint64_t key) {
    const uint32_t ord = (uint32_t)(key >> 32);
    return __uint_as_float((ord & 0x80000000u) ? (ord & 0x7FFFFFFFu) : ~ord);
}
__device__ __forceinline__ int key_expert(uint64_t key) {
    return (int)(0xFFFFFFFFu - (uint32_t)key);
}
__device__ __forceinline__ uint64_t max_u64(uint64_t a, uint64_t b) { return a > b ? a : b; }

// Routing variants: grouped top-k and a bias that steers the selection only.
struct RouteVariant {
    int n_group;          // <= 1: no grouping
    int topk_group;
    int group_score;      // 0: best biased logit of the group; 1: sum of its two best
    int bias_select_only;
};

// Top two keys of the union of (a1 >= a2) and (b1 >= b2); keys are distinct or 0.
__device__ __forceinline__ void merge_top2(uint64_t &a1, uint64_t &a2, uint64_t b1, uint64_t b2) {
    if (a1 > b1) {
        a2 = max_u64(a2, b1);
    } else {
        a2 = max_u64(a1, b2);
        a1 = b1;
    }
}

// Unsigned order key of a (finite or infinite) fp32 value: larger value, larger
// key; every real key is > 0, which marks a taken or missing expert.
__device__ __forceinline__ uint32_t order_key(float l) {
    const uint32_t u = __float_as_uint(l);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float order_value(uint32_t ord) {
    return __uint_as_float((ord & 0x80000000u) ? (ord & 0x7FFFFFFFu) : ~ord);
}

// The lane's best remaining key and its index (the first among equal keys: the
// lowest expert, since the lane's experts ascend with i).
template <int VPL>
__device__ __forceinline__ void lane_best(const uint32_t (&ord)[VPL], uint32_t &best, int &bi) {
    best = ord[0];
    bi = 0;
#pragma unroll
    for (int i = 1; i < VPL; ++i)
        if (ord[i] > best) { best = ord[i]; bi = i; }
}

template <int VPL>
__global__ void __launch_bounds__(256) route_topk_warp_kernel(
    int T, int E, int k, const float *__restrict__ logits, const float *__restrict__ bias,
    int bias_select_only, int32_t *__restrict__ topk_idx, float *__restrict__ topk_w,
    int32_t *__restrict__ counts, uint32_t *__restrict__ status) {
    grid_dependency_wait();
    grid_dependents_launch();
    extern __shared__ int32_t s_hist[];  // [E]
    for (int e = threadIdx.x; e < E; e += blockDim.x) s_hist[e] = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const long long warps_total = (long long)gridDim.x * (blockDim.x >> 5);
    long long t = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    float bv[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        const int e = lane + 32 * i;
        bv[i] = (bias && e < E) ? __ldg(bias + e) : 0.0f;
    }
    float nxt[VPL];
    auto load_row = [&](long long tt) {
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            const int e = lane + 32 * i;
            nxt[i] = (tt < T && e < E) ? __ldg(logits + (size_t)tt * E + e) : 0.0f;
        }
    };
    load_row(t);
    bool nonfinite = false;
    for (; t < T; t += warps_total) {
        uint32_t ord[VPL];
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            // the add also turns -0 into +0, so the key order matches IEEE ==
            float l = __fadd_rn(nxt[i], bv[i]);
            if (!isfinite(l)) {
                if (lane + 32 * i < E) nonfinite = true;
                if (isnan(l)) l = -INFINITY;  // keep the ranking a total order
            }
            ord[i] = lane + 32 * i < E ? order_key(l) : 0u;
        }
        load_row(t + warps_total);   // the next token's logits, in flight during the rounds
        uint32_t best;
        int bi;
        lane_best(ord, best, bi);
        uint32_t my_ord = 0;
        int my_e = -1;
        for (int j = 0; j < k; ++j) {
            const uint32_t top = __reduce_max_sync(0xffffffffu, best);
            const uint32_t cand = (best == top) ? (uint32_t)(lane + 32 * bi) : 0xFFFFFFFFu;
            const uint32_t e_top = __reduce_min_sync(0xffffffffu, cand);
            if (lane == j) { my_ord = top; my_e = (int)e_top; }
            if (cand == e_top) {
#pragma unroll
                for (int i = 0; i < VPL; ++i)
                    if (i == bi) ord[i] = 0u;
                lane_best(ord, best, bi);
            }
        }
        // the weights' logit: biased, or the unbiased logit when the bias only selects
        float my_v = order_value(my_ord);
        if (bias_select_only && lane < k) my_v = __fadd_rn(__ldg(logits + (size_t)t * E + my_e), 0.0f);
        float m = lane < k ? my_v : -INFINITY;   // the largest of the k
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        const float ex = (lane < k) ? det_exp_nonpos(__fsub_rn(my_v, m)) : 0.0f;
        float S = 0.0f;
        for (int j = 0; j < k; ++j) S = __fadd_rn(S, __shfl_sync(0xffffffffu, ex, j));
        if (lane < k) {
            topk_idx[(size_t)t * k + lane] = my_e;
            topk_w[(size_t)t * k + lane] = __fdiv_rn(ex, S);
            if (my_e >= 0 && my_e < E) atomicAdd(&s_hist[my_e], 1);   // always, as k <= E
        }
    }
    if (nonfinite) raise_status(status, MOE_DEV_NONFINITE_LOGIT);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        if (s_hist[e]) atomicAdd(&counts[e], s_hist[e]);
}

template <int LPT, int VPL>
__global__ void __launch_bounds__(256) route_topk_grouped_kernel(
    int T, int E, int k, const float *__restrict__ logits, const float *__restrict__ bias,
    RouteVariant rv,
    int32_t *__restrict__ topk_idx, float *__restrict__ topk_w, int32_t *__restrict__ counts,
    uint32_t *__restrict__ status) {
    grid_dependency_wait();
    grid_dependents_launch();
    extern __shared__ int32_t s_hist[];  // [E]
    for (int e = threadIdx.x; e < E; e += blockDim.x) s_hist[e] = 0;
    __syncthreads();

    constexpr int kGroups = 32 / LPT;
    const int lane = threadIdx.x & 31;
    const int gl = lane % LPT, g = lane / LPT;
    const int glane0 = g * LPT;
    const long long warps_total = (long long)gridDim.x * (blockDim.x >> 5);
    bool nonfinite = false;

    for (long long t0 = ((long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * kGroups;
         t0 < T; t0 += warps_total * kGroups) {
        const long long t = t0 + g;
        const bool valid = t < T;
        const float *row = logits + (size_t)(valid ? t : 0) * E;
        uint64_t key[VPL];
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            const int e = gl + LPT * i;
            key[i] = 0;
            if (valid && e < E) {
                // the add also turns -0 into +0, so the key order matches IEEE ==
                float l = __fadd_rn(__ldg(row + e), bias ? __ldg(bias + e) : 0.0f);
                if (!isfinite(l)) {
                    nonfinite = true;
                    if (isnan(l)) l = -INFINITY;  // keep the ranking a total order
                }
                key[i] = rank_key(l, e);
            }
        }
        {
            // grouped top-k: the score of every expert group (in-group butterfly per
            // group), kept as rank keys (score, group) spread over the lanes like the
            // experts (lane l holds groups l, l + LPT, ...); the topk_group best groups
            // are taken with the same rounds as the experts, and the experts of the
            // other groups drop out
            const int gsz = E / rv.n_group;
            constexpr int kGPL = (kMaxGroups + LPT - 1) / LPT;   // group keys per lane
            int eg[VPL];                                          // group of each held expert
#pragma unroll
            for (int i = 0; i < VPL; ++i) eg[i] = (gl + LPT * i) / gsz;
            uint64_t gkey[kGPL];
#pragma unroll
            for (int i = 0; i < kGPL; ++i) gkey[i] = 0;
            for (int grp = 0; grp < rv.n_group; ++grp) {
                uint64_t b1 = 0, b2 = 0;   // this lane's two best keys in the group
#pragma unroll
                for (int i = 0; i < VPL; ++i) {
                    if (key[i] != 0 && eg[i] == grp) {
                        if (key[i] > b1) { b2 = b1; b1 = key[i]; }
                        else b2 = max_u64(b2, key[i]);
                    }
                }
#pragma unroll
                for (int off = LPT / 2; off > 0; off >>= 1) {
                    const uint64_t o1 = __shfl_xor_sync(0xffffffffu, b1, off);
                    const uint64_t o2 = __shfl_xor_sync(0xffffffffu, b2, off);
                    merge_top2(b1, b2, o1, o2);
                }
                const float score = rv.group_score == 0 ? key_value(b1)
                                                        : __fadd_rn(key_value(b1), key_value(b2));
                if (grp % LPT == gl) {
#pragma unroll
                    for (int i = 0; i < kGPL; ++i)
                        if (i == grp / LPT) gkey[i] = rank_key(score, grp);
                }
            }
            uint64_t gbest = 0;
#pragma unroll
            for (int i = 0; i < kGPL; ++i) gbest = max_u64(gbest, gkey[i]);
            uint32_t kept = 0;   // bit g: group g kept
            for (int j = 0; j < rv.topk_group; ++j) {
                uint64_t top = gbest;
#pragma unroll
                for (int off = LPT / 2; off > 0; off >>= 1)
                    top = max_u64(top, __shfl_xor_sync(0xffffffffu, top, off));
                kept |= 1u << key_expert(top);
                if (gbest == top && top != 0) {
                    gbest = 0;
#pragma unroll
                    for (int i = 0; i < kGPL; ++i) {
                        if (gkey[i] == top) gkey[i] = 0;
                        gbest = max_u64(gbest, gkey[i]);
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < VPL; ++i)
                if (key[i] != 0 && !((kept >> eg[i]) & 1u)) key[i] = 0;
        }
        // each lane keeps its best remaining key; a round takes the group's best
        // and only the lane that held it looks for its next one
        uint64_t best = 0;
#pragma unroll
        for (int i = 0; i < VPL; ++i) best = max_u64(best, key[i]);
        uint64_t my_key = 0;  // slot `gl`'s key
        for (int j = 0; j < k; ++j) {
            uint64_t top = best;
#pragma unroll
            for (int off = LPT / 2; off > 0; off >>= 1)
                top = max_u64(top, __shfl_xor_sync(0xffffffffu, top, off));
            if (gl == j) my_key = top;
            if (best == top && top != 0) {
                best = 0;
#pragma unroll
                for (int i = 0; i < VPL; ++i) {
                    if (key[i] == top) key[i] = 0;
                    best = max_u64(best, key[i]);
                }
            }
        }
        const int my_e = key_expert(my_key);
        // the weights' logit: biased, or the unbiased logit when the bias only selects
        float my_v = key_value(my_key);
        if (rv.bias_select_only && valid && gl < k) my_v = __fadd_rn(__ldg(row + my_e), 0.0f);
        float m = gl < k ? my_v : -INFINITY;   // the largest of the k (slot 0's when biased)
#pragma unroll
        for (int off = LPT / 2; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        const float ex = (gl < k) ? det_exp_nonpos(__fsub_rn(my_v, m)) : 0.0f;
        float S = 0.0f;
        for (int j = 0; j < k; ++j) S = __fadd_rn(S, __shfl_sync(0xffffffffu, ex, glane0 + j));
        if (valid && gl < k) {
            topk_idx[(size_t)t * k + gl] = my_e;
            topk_w[(size_t)t * k + gl] = __fdiv_rn(ex, S);
            atomicAdd(&s_hist[my_e], 1);
        }
    }
    if (nonfinite) raise_status(status, MOE_DEV_NONFINITE_LOGIT);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        if (s_hist[e]) atomicAdd(&counts[e], s_hist[e]);
}

cudaError_t launch_route_topk(const moe_config &c, const float *logits, const float *bias,
                              int32_t *topk_idx, float *topk_w, int32_t *counts,
                              uint32_t *status, cudaStream_t s, int num_sms) {
    cudaError_t err = cudaMemsetAsync(counts, 0, sizeof(int32_t) * (size_t)c.E, s);
    if (err != cudaSuccess || c.T == 0) return err;
    const int warps_per_block = 8;
    int blocks = (c.T + warps_per_block - 1) / warps_per_block;
    const int cap = num_sms * 4;   // one global atomic per CTA and expert
    if (blocks > cap) blocks = cap;
    const size_t smem = sizeof(int32_t) * (size_t)c.E;
    const RouteVariant rv{c.n_group, c.topk_group, c.group_score, c.bias_select_only};
    if (rv.n_group <= 1) {
        // one warp per token, up to 8 CTAs of 8 warps per SM
        int wb = (c.T + warps_per_block - 1) / warps_per_block;
        if (wb > num_sms * 8) wb = num_sms * 8;
        const int v = (c.E + 31) / 32;
#define MOE_ROUTE_WARP(V)                                                                                 \
    return launch_dependent(route_topk_warp_kernel<V>, wb, 256, smem, s, c.T, c.E, c.k, logits, bias,     \
                            c.bias_select_only, topk_idx, topk_w, counts, status)
        if (v <= 1) MOE_ROUTE_WARP(1);
        if (v <= 2) MOE_ROUTE_WARP(2);
        if (v <= 4) MOE_ROUTE_WARP(4);
        if (v <= 8) MOE_ROUTE_WARP(8);
        if (v <= 16) MOE_ROUTE_WARP(16);
        MOE_ROUTE_WARP(32);
#undef MOE_ROUTE_WARP
    }
    // grouped: lanes per token: at least k (slot j lives in group lane j), at most 32,
    // aiming at 16 values per lane
    int lpt = 8;
    while (lpt < 32 && (lpt < c.k || (c.E + lpt - 1) / lpt > 16)) lpt *= 2;
    const int vpl = (c.E + lpt - 1) / lpt;
    blocks = (int)(((long long)c.T * lpt / 32 + warps_per_block - 1) / warps_per_block);
    if (blocks < 1) blocks = 1;
    if (blocks > cap) blocks = cap;
#define MOE_ROUTE_CASE(L, V)                                                                                 \
    return launch_dependent(route_topk_grouped_kernel<L, V>, blocks, 256, smem, s, c.T, c.E, c.k, logits, bias, \
                            rv, topk_idx, topk_w, counts, status)
    if (lpt == 8) {
        if (vpl <= 1) MOE_ROUTE_CASE(8, 1);
        else if (vpl <= 2) MOE_ROUTE_CASE(8, 2);
        else if (vpl <= 4) MOE_ROUTE_CASE(8, 4);
        else if (vpl <= 8) MOE_ROUTE_CASE(8, 8);
        else MOE_ROUTE_CASE(8, 16);
    } else if (lpt == 16) {
        if (vpl <= 1) MOE_ROUTE_CASE(16, 1);
        else if (vpl <= 2) MOE_ROUTE_CASE(16, 2);
        else if (vpl <= 4) MOE_ROUTE_CASE(16, 4);
        else if (vpl <= 8) MOE_ROUTE_CASE(16, 8);
        else MOE_ROUTE_CASE(16, 16);
    } else {
        if (vpl <= 1) MOE_ROUTE_CASE(32, 1);
        else if (vpl <= 2) MOE_ROUTE_CASE(32, 2);
        else if (vpl <= 4) MOE_ROUTE_CASE(32, 4);
        else if (vpl <= 8) MOE_ROUTE_CASE(32, 8);
        else if (vpl <= 16) MOE_ROUTE_CASE(32, 16);
        else MOE_ROUTE_CASE(32, 32);
    }
#undef MOE_ROUTE_CASE
}

}  // namespace moe
