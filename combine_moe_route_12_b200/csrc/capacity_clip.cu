// Step 2: per-expert token capacity (axolotl ExpertParallelArgs,
// expert_parallel_token_capacity): an expert holding more than C assignments
// keeps the C with the largest weight; the lowest-weight excess is dropped,
// and among equal weights the higher token index goes first.
//
// Every assignment (t, j) of expert e gets the 64-bit key
//     (bits(w[t, j]) << 32) | (2^32 - 1 - t),
// which orders by weight descending then token ascending (weights are >= 0,
// so their bit patterns order like their values; keys of one expert are
// distinct because a token picks an expert at most once).  For each
// over-capacity expert one CTA finds the C-th largest key by an MSB-first
// radix select (8 passes of 8-bit digits); an assignment is kept iff its key
// is >= that threshold, which keeps exactly C.
#include "moe_common.cuh"

namespace moe {

constexpr int kClipThreads = 1024;
constexpr int kClipMaxSmemKeys = 24576;  // 192 KiB of keys; larger segments stream from global

__device__ __forceinline__ uint64_t clip_key(float w, int t) {
    return ((uint64_t)__float_as_uint(w) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)t);
}

// Radix select of the rank-`want` (1-based, descending) key among the keys that
// `visit` produces.  visit(f) calls f(key) for every key of the segment; it is
// called once per pass by every thread of the CTA.
template <typename Visit>
__device__ uint64_t radix_select_desc(Visit visit, uint32_t want, uint32_t *s_hist,
                                      uint32_t *s_sel) {
    uint64_t prefix = 0, mask = 0;
    for (int pass = 0; pass < 8; ++pass) {
        const int shift = 56 - 8 * pass;
        for (int i = threadIdx.x; i < 256; i += blockDim.x) s_hist[i] = 0;
        __syncthreads();
        visit([&](uint64_t key) {
            // warp-aggregated: keys of one expert share their leading digits, so
            // plain per-key shared atomics would serialise on one bin
            const unsigned active = __activemask();
            const int d = ((key & mask) == prefix) ? (int)((key >> shift) & 255u) : -1;
            const unsigned peers = __match_any_sync(active, d);
            if (d >= 0 && (int)(threadIdx.x & 31) == __ffs(peers) - 1)
                atomicAdd(&s_hist[d], (uint32_t)__popc(peers));
        });
        __syncthreads();
        if (threadIdx.x == 0) {
            uint32_t cum = 0, sel = 0;
            for (int d = 255; d >= 0; --d) {
                if (cum + s_hist[d] >= want) { sel = (uint32_t)d; break; }
                cum += s_hist[d];
            }
            s_sel[0] = sel;
            s_sel[1] = want - cum;
        }
        __syncthreads();
        prefix |= (uint64_t)s_sel[0] << shift;
        mask |= (uint64_t)255u << shift;
        want = s_sel[1];
        __syncthreads();
    }
    return prefix;
}

__global__ void __launch_bounds__(kClipThreads) clip_select_kernel(
    int T, int E, int k, int C, int smem_keys, const int32_t *__restrict__ topk_idx,
    const float *__restrict__ topk_w, const int32_t *__restrict__ counts,
    int32_t *__restrict__ kept_counts, uint64_t *__restrict__ thr) {
    extern __shared__ __align__(16) unsigned char s_raw[];
    __shared__ uint32_t s_hist[256];
    __shared__ uint32_t s_sel[2];
    __shared__ uint32_t s_n;
    const int e = blockIdx.x;
    const int n = counts[e];
    if (C < 0 || n <= C) {
        if (threadIdx.x == 0) { kept_counts[e] = n; thr[e] = 0; }
        return;
    }
    if (C == 0) {
        if (threadIdx.x == 0) { kept_counts[e] = 0; thr[e] = ~0ull; }
        return;
    }
    const size_t total = (size_t)T * k;
    uint64_t key;
    if (n <= smem_keys) {
        uint64_t *s_keys = reinterpret_cast<uint64_t *>(s_raw);
        if (threadIdx.x == 0) s_n = 0;
        __syncthreads();
        for (size_t a = threadIdx.x; a < total; a += blockDim.x) {
            if (__ldg(topk_idx + a) == e) {
                const uint32_t slot = atomicAdd(&s_n, 1u);
                if (slot < (uint32_t)smem_keys) s_keys[slot] = clip_key(__ldg(topk_w + a), (int)(a / k));
            }
        }
        __syncthreads();
        const uint32_t m = min(s_n, (uint32_t)smem_keys);
        key = radix_select_desc(
            [&](auto f) {
                for (uint32_t i = threadIdx.x; i < m; i += blockDim.x) f(s_keys[i]);
            },
            (uint32_t)C, s_hist, s_sel);
    } else {
        key = radix_select_desc(
            [&](auto f) {
                for (size_t a = threadIdx.x; a < total; a += blockDim.x)
                    if (__ldg(topk_idx + a) == e) f(clip_key(__ldg(topk_w + a), (int)(a / k)));
            },
            (uint32_t)C, s_hist, s_sel);
    }
    if (threadIdx.x == 0) { kept_counts[e] = C; thr[e] = key; }
}

__global__ void clip_mark_kernel(int T, int E, int k, const int32_t *__restrict__ topk_idx,
                                 const float *__restrict__ topk_w,
                                 const uint64_t *__restrict__ thr, uint8_t *__restrict__ keep,
                                 uint32_t *__restrict__ status) {
    const size_t total = (size_t)T * k;
    bool bad = false;
    for (size_t a = (size_t)blockIdx.x * blockDim.x + threadIdx.x; a < total;
         a += (size_t)gridDim.x * blockDim.x) {
        const int e = topk_idx[a];
        uint8_t kv = 0;
        if (e < 0 || e >= E) bad = true;
        else kv = clip_key(topk_w[a], (int)(a / k)) >= thr[e] ? 1 : 0;
        keep[a] = kv;
    }
    if (bad) raise_status(status, MOE_DEV_BAD_INDEX);
}

cudaError_t launch_capacity_clip(const moe_config &c, const int32_t *topk_idx,
                                 const float *topk_w, const int32_t *counts, uint8_t *keep,
                                 int32_t *kept_counts, uint64_t *thr, uint32_t *status,
                                 cudaStream_t s, int num_sms) {
    int smem_keys = c.T < kClipMaxSmemKeys ? c.T : kClipMaxSmemKeys;
    if (smem_keys < 1) smem_keys = 1;
    const size_t smem = sizeof(uint64_t) * (size_t)smem_keys;
    cudaError_t err;
    static size_t configured = 48 * 1024;
    if (smem > configured) {
        err = cudaFuncSetAttribute(clip_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)smem);
        if (err != cudaSuccess) return err;
        configured = smem;
    }
    clip_select_kernel<<<c.E, kClipThreads, smem, s>>>(c.T, c.E, c.k, c.capacity, smem_keys,
                                                       topk_idx, topk_w, counts, kept_counts, thr);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    const size_t total = (size_t)c.T * c.k;
    if (total == 0) return cudaSuccess;
    int blocks = (int)((total + 255) / 256);
    if (blocks > num_sms * 16) blocks = num_sms * 16;
    clip_mark_kernel<<<blocks, 256, 0, s>>>(c.T, c.E, c.k, topk_idx, topk_w, thr, keep, status);
    return cudaGetLastError();
}

}  // namespace moe
