// Step 2: per-expert token capacity (axolotl ExpertParallelArgs,
// expert_parallel_token_capacity): an expert holding more than C assignments
// keeps the C with the largest weight; the lowest-weight excess is dropped,
// and among equal weights the higher token index goes first.
//
// Every assignment (t, j) of expert e gets the 64-bit key
//     (bits(w[t, j]) << 32) | (2^32 - 1 - t),
// which orders by weight descending then token ascending (weights are >= 0,
// so their bit patterns order like their values; keys of one expert are
// distinct because a token picks an expert at most once).
//
//   clip_prep    one CTA: which experts are over capacity, their key segment
//                offsets (prefix sum of their counts); thresholds of the rest
//   clip_gather  one pass over all assignments: the keys of over-capacity
//                experts go to their segments (per-CTA ranges reserved with one
//                atomic per CTA and expert; slots inside a range by shared atomics)
//   clip_select  one CTA per over-capacity expert: the C-th largest key of its
//                segment by an MSB-first radix select (up to 8 passes of 8-bit
//                digits, ending early once one key is left under the prefix)
//   clip_mark    keep[t, j] = key >= threshold of its expert, which keeps exactly C
#include "moe_common.cuh"

namespace moe {

constexpr int kClipThreads = 1024;
constexpr int kClipMaxSmemKeys = 24576;  // 192 KiB of keys; larger segments stream from global

__device__ __forceinline__ uint64_t clip_key(float w, int t) {
    return ((uint64_t)__float_as_uint(w) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)t);
}

// Radix select of the rank-`want` (1-based, descending) key among the keys that
// `visit` produces.  visit(f) calls f(key) for every key of the segment; it is
// called once per pass by every thread of the CTA (whole warps enter f
// together, the last iteration of a strided loop possibly with fewer lanes).
// The digit holding the
// target rank is found by warp 0 with a suffix-sum over the 256 bins.  Once the
// chosen bin holds a single key, that key is the answer: one more visit picks
// it up instead of the remaining digit passes (distinct fp32 weights are
// usually told apart by the first two or three digits).
template <typename Visit>
__device__ uint64_t radix_select_desc(Visit visit, uint32_t want, uint32_t *s_hist,
                                      uint32_t *s_sel, uint64_t *s_found) {
    uint64_t prefix = 0, mask = 0;
    const int lane = threadIdx.x & 31;
    for (int pass = 0; pass < 8; ++pass) {
        const int shift = 56 - 8 * pass;
        for (int i = threadIdx.x; i < 256; i += blockDim.x) s_hist[i] = 0;
        __syncthreads();
        visit([&](uint64_t key) {
            // keys of one expert share their leading digits: when a whole warp
            // holds one digit (the common case in the first passes) one lane adds
            // the warp's count, otherwise each key adds itself (the bins are then
            // mostly distinct)
            const unsigned active = __activemask();
            const int d = ((key & mask) == prefix) ? (int)((key >> shift) & 255u) : -1;
            const int first = __ffs(active) - 1;
            const int d0 = __shfl_sync(active, d, first);
            if (__all_sync(active, d == d0)) {
                if (d0 >= 0 && (int)(threadIdx.x & 31) == first)
                    atomicAdd(&s_hist[d0], (uint32_t)__popc(active));
            } else if (d >= 0) {
                atomicAdd(&s_hist[d], 1u);
            }
        });
        __syncthreads();
        if (threadIdx.x < 32) {
            // lane l owns bins 255-8l .. 248-8l (high digits first)
            uint32_t c[8], tot = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) { c[i] = s_hist[255 - 8 * lane - i]; tot += c[i]; }
            uint32_t incl = tot;   // inclusive prefix over lanes = counts of digits >= this lane's
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const uint32_t o = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += o;
            }
            const uint32_t before = incl - tot;
            const bool mine = before < want && want <= incl;
            if (mine) {
                uint32_t cum = before;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    if (cum + c[i] >= want) {
                        s_sel[0] = 255 - 8 * lane - i; s_sel[1] = want - cum; s_sel[2] = c[i];
                        break;
                    }
                    cum += c[i];
                }
            }
        }
        __syncthreads();
        prefix |= (uint64_t)s_sel[0] << shift;
        mask |= (uint64_t)255u << shift;
        want = s_sel[1];
        const uint32_t left = s_sel[2];
        __syncthreads();
        if (left == 1 && pass < 7) {
            // the only key under this prefix (keys are distinct)
            visit([&](uint64_t key) {
                if ((key & mask) == prefix) *s_found = key;
            });
            __syncthreads();
            return *s_found;
        }
    }
    return prefix;
}

constexpr int kGatherThreads = 256;
constexpr int kGatherPerThread = 8;

__global__ void __launch_bounds__(1024) clip_prep_kernel(int E, int C, const int32_t *__restrict__ counts,
                                                         int32_t *__restrict__ seg,  // [2][E+1]: offsets, cursors
                                                         int32_t *__restrict__ kept_counts,
                                                         uint64_t *__restrict__ thr) {
    grid_dependency_wait();
    grid_dependents_launch();
    __shared__ int32_t s_v[1025];
    __shared__ int32_t s_w[33];
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const int n = counts[e];
        const bool over = C >= 0 && n > C;
        s_v[e] = over ? n : 0;
        if (!over) { kept_counts[e] = n; thr[e] = 0; }
        else { kept_counts[e] = C; if (C == 0) thr[e] = ~0ull; }
    }
    __syncthreads();
    // exclusive scan of s_v (E <= 1024) by one warp, 32 entries per lane
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        int sum = 0;
        for (int i = 0; i < 32; ++i) { const int e = lane * 32 + i; if (e < E) sum += s_v[e]; }
        int incl = sum;
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += o;
        }
        int run = incl - sum;
        for (int i = 0; i < 32; ++i) {
            const int e = lane * 32 + i;
            if (e < E) { const int v = s_v[e]; s_v[e] = run; run += v; }
        }
        if (lane == 31) s_w[0] = incl;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) { seg[e] = s_v[e]; seg[E + 1 + e] = 0; }
    if (threadIdx.x == 0) seg[E] = s_w[0];
}

__global__ void __launch_bounds__(kGatherThreads) clip_gather_kernel(
    int T, int E, int k, int C, const int32_t *__restrict__ topk_idx,
    const float *__restrict__ topk_w, const int32_t *__restrict__ counts,
    int32_t *__restrict__ seg, uint64_t *__restrict__ keys) {
    grid_dependency_wait();
    grid_dependents_launch();
    extern __shared__ int32_t s_cnt[];   // [E] this CTA's keys per expert, then its base
    const size_t total = (size_t)T * k;
    const size_t a0 = (size_t)blockIdx.x * kGatherThreads * kGatherPerThread;
    for (int e = threadIdx.x; e < E; e += blockDim.x) s_cnt[e] = 0;
    __syncthreads();
    int ex[kGatherPerThread], slot[kGatherPerThread];
    // all of the thread's expert ids, then all their counts, are loaded before the
    // first warp-collective step, so the loads overlap instead of queueing
#pragma unroll
    for (int i = 0; i < kGatherPerThread; ++i) {
        const size_t a = a0 + (size_t)i * kGatherThreads + threadIdx.x;
        ex[i] = a < total ? __ldg(topk_idx + a) : -1;
    }
    int cnt[kGatherPerThread];
#pragma unroll
    for (int i = 0; i < kGatherPerThread; ++i)
        cnt[i] = (ex[i] >= 0 && ex[i] < E) ? __ldg(counts + ex[i]) : 0;
#pragma unroll
    for (int i = 0; i < kGatherPerThread; ++i) {
        const int ev = ex[i];
        const int e = (ev >= 0 && ev < E && C > 0 && cnt[i] > C) ? ev : -1;
        ex[i] = e;
        slot[i] = -1;
        // a slot in this CTA's range of expert e (the order inside a segment does
        // not matter: the select finds a threshold): one reservation when the whole
        // warp holds one expert, otherwise one shared atomic per key
        const unsigned active = __activemask();
        const int lane = threadIdx.x & 31;
        const int first = __ffs(active) - 1;
        const int e0 = __shfl_sync(active, e, first);
        if (__all_sync(active, e == e0)) {
            if (e0 >= 0) {
                int base = 0;
                if (lane == first) base = atomicAdd(&s_cnt[e0], __popc(active));
                base = __shfl_sync(active, base, first);
                slot[i] = base + __popc(active & ((1u << lane) - 1u));
            }
        } else if (e >= 0) {
            slot[i] = atomicAdd(&s_cnt[e], 1);
        }
    }
    __syncthreads();
    // reserve this CTA's range in each touched expert's segment
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const int n = s_cnt[e];
        s_cnt[e] = n > 0 ? seg[e] + atomicAdd(&seg[E + 1 + e], n) : 0;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kGatherPerThread; ++i) {
        if (ex[i] < 0) continue;
        const size_t a = a0 + (size_t)i * kGatherThreads + threadIdx.x;
        const size_t dst = (size_t)s_cnt[ex[i]] + slot[i];
        if (dst < total)   // counts inconsistent with topk_idx cannot write out of range
            keys[dst] = clip_key(__ldg(topk_w + a), (int)(a / (size_t)k));
    }
}

__global__ void __launch_bounds__(kClipThreads) clip_select_kernel(
    int E, int C, int smem_keys, long long total_keys, const int32_t *__restrict__ counts,
    const int32_t *__restrict__ seg, const uint64_t *__restrict__ keys, uint64_t *__restrict__ thr) {
    grid_dependency_wait();
    grid_dependents_launch();
    extern __shared__ __align__(16) unsigned char s_raw[];
    __shared__ uint32_t s_hist[256];
    __shared__ uint32_t s_sel[3];
    __shared__ uint64_t s_found;
    const int e = blockIdx.x;
    int n = counts[e];
    if (C <= 0 || n <= C) return;    // thresholds of these experts come from clip_prep
    const uint64_t *mine = keys + seg[e];
    if ((long long)seg[e] + n > total_keys) n = (int)(total_keys - seg[e]);   // inconsistent counts
    uint64_t key;
    if (n <= smem_keys) {
        uint64_t *s_keys = reinterpret_cast<uint64_t *>(s_raw);
        // eight loads in flight per thread before the stores to shared memory
        for (int i0 = threadIdx.x; i0 < n; i0 += 8 * blockDim.x) {
            uint64_t v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = i0 + u * (int)blockDim.x;
                v[u] = i < n ? __ldcg(mine + i) : 0ull;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = i0 + u * (int)blockDim.x;
                if (i < n) s_keys[i] = v[u];
            }
        }
        __syncthreads();
        key = radix_select_desc(
            [&](auto f) {
                for (int i = threadIdx.x; i < n; i += blockDim.x) f(s_keys[i]);
            },
            (uint32_t)C, s_hist, s_sel, &s_found);
    } else {
        key = radix_select_desc(
            [&](auto f) {
                for (int i = threadIdx.x; i < n; i += blockDim.x) f(__ldcg(mine + i));
            },
            (uint32_t)C, s_hist, s_sel, &s_found);
    }
    if (threadIdx.x == 0) thr[e] = key;
}

__global__ void clip_mark_kernel(int T, int E, int k, const int32_t *__restrict__ topk_idx,
                                 const float *__restrict__ topk_w,
                                 const uint64_t *__restrict__ thr, uint8_t *__restrict__ keep,
                                 uint32_t *__restrict__ status) {
    grid_dependency_wait();
    grid_dependents_launch();
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

// No capacity (C < 0): every valid assignment is kept and the kept counts are
// the routed counts; one pass, the same index check as the marking pass.
__global__ void clip_all_kernel(int T, int E, int k, const int32_t *__restrict__ topk_idx,
                                const int32_t *__restrict__ counts, uint8_t *__restrict__ keep,
                                int32_t *__restrict__ kept_counts, uint32_t *__restrict__ status) {
    grid_dependency_wait();
    grid_dependents_launch();
    if (blockIdx.x == 0)
        for (int e = threadIdx.x; e < E; e += blockDim.x) kept_counts[e] = counts[e];
    const size_t total = (size_t)T * k;
    bool bad = false;
    for (size_t a = (size_t)blockIdx.x * blockDim.x + threadIdx.x; a < total;
         a += (size_t)gridDim.x * blockDim.x) {
        const int e = topk_idx[a];
        const bool ok = e >= 0 && e < E;
        bad |= !ok;
        keep[a] = ok ? 1 : 0;
    }
    if (bad) raise_status(status, MOE_DEV_BAD_INDEX);
}

cudaError_t launch_capacity_clip(const moe_config &c, const int32_t *topk_idx,
                                 const float *topk_w, const int32_t *counts, uint8_t *keep,
                                 int32_t *kept_counts, uint64_t *thr, int32_t *seg, uint64_t *keys,
                                 uint32_t *status, cudaStream_t s, int num_sms) {
    if (c.capacity < 0) {
        const size_t total = (size_t)c.T * c.k;
        int blocks = (int)((total + 255) / 256);
        if (blocks > num_sms * 16) blocks = num_sms * 16;
        if (blocks < 1) blocks = 1;
        return launch_dependent(clip_all_kernel, blocks, 256, 0, s, c.T, c.E, c.k, topk_idx, counts, keep,
                                kept_counts, status);
    }
    cudaError_t err = launch_dependent(clip_prep_kernel, 1, 1024, 0, s, c.E, c.capacity, counts, seg, kept_counts, thr);
    if (err != cudaSuccess) return err;
    const size_t total = (size_t)c.T * c.k;
    if (total == 0) return cudaSuccess;
    if (c.capacity > 0) {
        const int per_block = kGatherThreads * kGatherPerThread;
        const int gblocks = (int)((total + per_block - 1) / per_block);
        err = launch_dependent(clip_gather_kernel, gblocks, kGatherThreads, sizeof(int32_t) * c.E, s,
                               c.T, c.E, c.k, c.capacity, topk_idx, topk_w, counts, seg, keys);
        if (err != cudaSuccess) return err;
        int smem_keys = c.T < kClipMaxSmemKeys ? c.T : kClipMaxSmemKeys;
        if (smem_keys < 1) smem_keys = 1;
        const size_t smem = sizeof(uint64_t) * (size_t)smem_keys;
        static SmemOptIn opt_in;
        if ((err = opt_in.ensure(clip_select_kernel, smem)) != cudaSuccess) return err;
        err = launch_dependent(clip_select_kernel, c.E, kClipThreads, smem, s, c.E, c.capacity, smem_keys,
                               (long long)total, counts, seg, keys, thr);
        if (err != cudaSuccess) return err;
    }
    int blocks = (int)((total + 255) / 256);
    if (blocks > num_sms * 16) blocks = num_sms * 16;
    return launch_dependent(clip_mark_kernel, blocks, 256, 0, s, c.T, c.E, c.k, topk_idx, topk_w, thr, keep, status);
}

}  // namespace moe
