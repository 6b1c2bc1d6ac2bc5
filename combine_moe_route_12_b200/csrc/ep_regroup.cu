// Expert-parallel exchange, the receive side's regroup (axolotl ExpertParallelArgs,
// expert_parallel_backend = torch: all_to_all_single over the EP group, which
// hands each rank the rows of every source rank, source after source).
//
// A source rank sends a destination the rows of the destination's experts in its
// own (expert, token) order, so after the variable all-to-all the destination holds
// them source-major: cell (s, e) - the rows source s sent for local expert e - at
// src_off[s] + (rows of s for experts before e).  The grouped FFN wants them expert
// by expert; with sources owning contiguous token blocks, (expert, source, token)
// is the (expert, token) order of the whole EP group, so cell (s, e) goes to
// exp_off[e] + (rows of e from sources before s).  The inverse brings the expert
// outputs back to source-major order for the reverse all-to-all.
//
// One kernel: every CTA builds both cell tables in shared memory (two block scans
// over n_src * n_exp counts), then each warp copies whole rows with 16-byte loads
// and stores.  A count table whose total differs from the rows given raises
// MOE_DEV_BAD_INDEX (when a status word is given) and rows outside either range are
// skipped: nothing is read or written past `rows`.
#include "moe_common.cuh"

namespace moe {

constexpr int kRegroupThreads = 256;
constexpr int kRegroupMaxCells = 1024;   // n_src * n_exp: the experts of the whole group

// Exclusive scan of n values taken from cnt[order(i)] into out[order(i)], in place
// order; returns the total.  n <= kRegroupMaxCells, 256 threads, 4 values each.
template <class Order>
__device__ int regroup_scan(int n, const int32_t *cnt, int32_t *out, Order order, int32_t *s_warp) {
    constexpr int kPer = kRegroupMaxCells / kRegroupThreads;
    const int lo = threadIdx.x * kPer;
    int v[kPer];
    int sum = 0;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
        v[j] = lo + j < n ? cnt[order(lo + j)] : 0;
        sum += v[j];
    }
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) s_warp[wid] = incl;
    __syncthreads();
    if (threadIdx.x == 0) {
        int run = 0;
        for (int w = 0; w < kRegroupThreads / 32; ++w) {
            const int t = s_warp[w];
            s_warp[w] = run;
            run += t;
        }
        s_warp[kRegroupThreads / 32] = run;
    }
    __syncthreads();
    int run = s_warp[wid] + incl - sum;
#pragma unroll
    for (int j = 0; j < kPer; ++j)
        if (lo + j < n) { out[order(lo + j)] = run; run += v[j]; }
    const int total = s_warp[kRegroupThreads / 32];
    __syncthreads();
    return total;
}

__global__ void __launch_bounds__(kRegroupThreads) ep_regroup_kernel(
    int n_src, int n_exp, const int32_t *__restrict__ counts, const uint4 *__restrict__ in,
    uint4 *__restrict__ out, int64_t rows, int row_vecs, int inverse, int32_t *__restrict__ expert_offsets,
    uint32_t *__restrict__ status) {
    __shared__ int32_t s_cnt[kRegroupMaxCells];
    __shared__ int32_t s_src[kRegroupMaxCells + 1];   // cell (s, e) = s * n_exp + e: source-major start
    __shared__ int32_t s_exp[kRegroupMaxCells];       // the same cell's expert-major start
    __shared__ int32_t s_warp[kRegroupThreads / 32 + 1];
    const int cells = n_src * n_exp;
    for (int c = threadIdx.x; c < cells; c += blockDim.x) s_cnt[c] = max(0, counts[c]);
    __syncthreads();
    // source-major: cells in index order; expert-major: cell order (e, s)
    const int total = regroup_scan(cells, s_cnt, s_src, [](int i) { return i; }, s_warp);
    regroup_scan(cells, s_cnt, s_exp, [n_src, n_exp](int i) { return (i % n_src) * n_exp + i / n_src; },
                 s_warp);
    if (threadIdx.x == 0) s_src[cells] = total;
    __syncthreads();
    if (blockIdx.x == 0) {
        if (total != rows && status && threadIdx.x == 0) raise_status(status, MOE_DEV_BAD_INDEX);
        // the expert-major buffer's expert offsets: expert e starts with its rows from source 0
        if (expert_offsets)
            for (int e = threadIdx.x; e <= n_exp; e += blockDim.x) expert_offsets[e] = e < n_exp ? s_exp[e] : total;
    }

    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t p = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); p < rows && p < total;
         p += warps) {
        int lo = 0, hi = cells - 1;   // the last cell with s_src[c] <= p (empty cells skipped)
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_src[mid] <= p) lo = mid; else hi = mid - 1;
        }
        const int64_t q = (int64_t)s_exp[lo] + (p - s_src[lo]);
        if (q >= rows) continue;   // only with a count table that does not add up to rows
        const uint4 *from = in + (inverse ? q : p) * row_vecs;
        uint4 *to = out + (inverse ? p : q) * row_vecs;
        for (int v = lane; v < row_vecs; v += 32) to[v] = from[v];
    }
}

cudaError_t launch_ep_regroup(int n_src, int n_exp, const int32_t *counts, const void *in, void *out,
                              int64_t rows, int row_bytes, int inverse, int32_t *expert_offsets, uint32_t *status,
                              cudaStream_t s, int num_sms) {
    if (rows <= 0) return cudaSuccess;
    const int64_t warps_wanted = rows;
    int64_t blocks = (warps_wanted + kRegroupThreads / 32 - 1) / (kRegroupThreads / 32);
    if (blocks > (int64_t)num_sms * 8) blocks = (int64_t)num_sms * 8;
    ep_regroup_kernel<<<(int)blocks, kRegroupThreads, 0, s>>>(
        n_src, n_exp, counts, static_cast<const uint4 *>(in), static_cast<uint4 *>(out), rows, row_bytes / 16,
        inverse, expert_offsets, status);
    return cudaGetLastError();
}

}  // namespace moe
