// Step 3: dispatch layout (axolotl ExpertParallelArgs, expert_parallel_backend
// = torch: all_to_all_single over the EP group; LightLLM PR 1687: the expert
// prefix-sum "psum" layout that the grouped GEMM consumes).
//
// Receive rows are the kept (token, expert) assignments of a token chunk in
// stable order by (expert, token).  With experts owned by contiguous rank
// blocks this is also the (destination rank, expert, token) order, i.e. the
// all_to_all_single arrival order regrouped by expert.  The order is built by
// a stable counting sort:
//
//   layout_hist     per-expert kept counts of the chunk (shared-memory
//                   histogram, one global atomic per CTA and expert);
//   layout_scatter  one CTA per 256-token tile, tiles taken in launch order
//                   from an atomic ticket.  Each tile ranks its assignments
//                   per expert in token order (warps walk their tokens with
//                   __match_any_sync), publishes its per-expert counts, and
//                   finds its prefix over earlier tiles by a decoupled
//                   look-back (Merrill & Garland 2016), one expert per thread.
//                   The row of (t, j) is expert_offsets[e] + (rows of e in
//                   earlier tiles) + (rank of t among this tile's rows of e).
//   layout_splits   one CTA per destination rank counts its rows by source
//                   rank, giving the EP x EP all_to_all_single split matrix.
//
// The look-back waits are bounded: on a timeout the tile raises
// MOE_DEV_WAIT_TIMEOUT, publishes what it has so that later tiles finish,
// and skips every write that would leave the receive buffers.
#include "moe_common.cuh"

namespace moe {

constexpr int kLayoutThreads = 256;
constexpr int kLayoutWarps = kLayoutThreads / 32;
constexpr int kTokensPerWarp = kLayoutTileTokens / kLayoutWarps;
constexpr uint32_t kFlagAggregate = 1u << 30;
constexpr uint32_t kFlagInclusive = 2u << 30;
constexpr uint32_t kValueMask = (1u << 30) - 1;

__global__ void __launch_bounds__(kLayoutThreads) layout_hist_kernel(
    int tb, int tc, int k, int E, const int32_t *__restrict__ topk_idx,
    const uint8_t *__restrict__ keep, int32_t *__restrict__ chunk_counts) {
    extern __shared__ int32_t s_hist[];
    for (int e = threadIdx.x; e < E; e += blockDim.x) s_hist[e] = 0;
    __syncthreads();
    const size_t a0 = (size_t)tb * k, a1 = (size_t)(tb + tc) * k;
    for (size_t a = a0 + (size_t)blockIdx.x * blockDim.x + threadIdx.x; a < a1;
         a += (size_t)gridDim.x * blockDim.x) {
        const int e = keep[a] ? topk_idx[a] : -1;
        if (e >= 0 && e < E) atomicAdd(&s_hist[e], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        if (s_hist[e]) atomicAdd(&chunk_counts[e], s_hist[e]);
}

// Exclusive scan of s[0..n) in place (n <= 4 * blockDim.x); returns the total.
__device__ int block_exclusive_scan(int32_t *s, int n, int32_t *s_warp_tot) {
    const int per = (n + blockDim.x - 1) / blockDim.x;  // <= 4
    const int lo = threadIdx.x * per;
    int v[4];
    int sum = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[i] = (i < per && lo + i < n) ? s[lo + i] : 0;
        sum += v[i];
    }
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) s_warp_tot[wid] = incl;
    __syncthreads();
    if (threadIdx.x == 0) {
        int run = 0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
            const int t = s_warp_tot[w];
            s_warp_tot[w] = run;
            run += t;
        }
        s_warp_tot[32] = run;
    }
    __syncthreads();
    int run = s_warp_tot[wid] + incl - sum;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (i < per && lo + i < n) { s[lo + i] = run; run += v[i]; }
    }
    const int total = s_warp_tot[32];
    __syncthreads();
    return total;
}

__global__ void __launch_bounds__(kLayoutThreads) layout_scatter_kernel(
    int tb, int tc, int k, int E, int ep, int64_t n_rows_max,
    const int32_t *__restrict__ topk_idx, const uint8_t *__restrict__ keep,
    const int32_t *__restrict__ chunk_counts, uint32_t *__restrict__ ticket,
    uint32_t *__restrict__ tile_state, int32_t *__restrict__ expert_offsets,
    int32_t *__restrict__ rank_offsets, int32_t *__restrict__ recv_token,
    int32_t *__restrict__ recv_slot, int32_t *__restrict__ pos, uint32_t *__restrict__ status) {
    extern __shared__ int32_t s_dyn[];
    int32_t *s_eoff = s_dyn;                                 // [E + 1]
    int32_t *s_base = s_eoff + (E + 1);                      // [E]
    int32_t *s_cnt = s_base + E;                             // [kLayoutWarps][E]
    int32_t *s_rank = s_cnt + kLayoutWarps * E;              // [kLayoutTileTokens * k]
    __shared__ int32_t s_warp_tot[33];
    __shared__ uint32_t s_tile;

    if (threadIdx.x == 0) s_tile = atomicAdd(ticket, 1u);
    for (int e = threadIdx.x; e < E; e += blockDim.x) s_eoff[e] = chunk_counts[e];
    for (int i = threadIdx.x; i < kLayoutWarps * E; i += blockDim.x) s_cnt[i] = 0;
    __syncthreads();
    const int tile = (int)s_tile;
    const int total = block_exclusive_scan(s_eoff, E, s_warp_tot);
    if (threadIdx.x == 0) s_eoff[E] = total;
    __syncthreads();

    if (tile == 0) {
        const int epr = E / ep;
        for (int e = threadIdx.x; e <= E; e += blockDim.x) expert_offsets[e] = s_eoff[e];
        for (int d = threadIdx.x; d <= ep; d += blockDim.x) rank_offsets[d] = s_eoff[d * epr];
    }

    // 1) rank every kept assignment of this tile among the warp's rows of its expert
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int t_tile0 = tb + tile * kLayoutTileTokens;
    const int G = 32 / k;                      // tokens per warp step
    const unsigned lt_mask = (1u << lane) - 1u;
    bool bad = false;
    for (int b = 0; b < kTokensPerWarp; b += G) {
        const int ti = wid * kTokensPerWarp + b + lane / k;  // token within the tile
        const int j = lane % k;
        const int t = t_tile0 + ti;
        int e = -1 - lane;                     // unique sentinel: matches nobody
        if (lane < G * k && b + lane / k < kTokensPerWarp && t < tb + tc) {
            const size_t a = (size_t)t * k + j;
            if (keep[a]) {
                const int ev = topk_idx[a];
                if (ev >= 0 && ev < E) e = ev;
                else bad = true;
            }
        }
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        if (e >= 0) s_rank[ti * k + j] = s_cnt[wid * E + e] + __popc(peers & lt_mask);
        __syncwarp();
        if (e >= 0 && (31 - __clz(peers)) == lane) s_cnt[wid * E + e] += __popc(peers);
        __syncwarp();
    }
    __syncthreads();

    // 2) per-expert warp offsets and tile aggregate; publish, look back, publish inclusive
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = 0;
        for (int w = 0; w < kLayoutWarps; ++w) {
            const int c = s_cnt[w * E + e];
            s_cnt[w * E + e] = run;
            run += c;
        }
        const uint32_t agg = (uint32_t)run;
        uint32_t *my = tile_state + (size_t)tile * E + e;
        uint32_t excl = 0;
        if (tile == 0) {
            st_release_u32(my, kFlagInclusive | agg);
        } else {
            st_release_u32(my, kFlagAggregate | agg);
            for (int p = tile - 1; p >= 0; --p) {
                const uint32_t *q = tile_state + (size_t)p * E + e;
                uint32_t v = ld_acquire_u32(q);
                if ((v >> 30) == 0) {
                    const uint64_t t0 = global_timer_ns();
                    while (((v = ld_acquire_u32(q)) >> 30) == 0)
                        if (global_timer_ns() - t0 > kWaitLimitNs) break;
                }
                if ((v >> 30) == 0) {                 // gave up: predecessor never published
                    raise_status(status, MOE_DEV_WAIT_TIMEOUT);
                    excl = 0x3FFFFFFFu;               // forces every write of this expert out of range
                    break;
                }
                excl += v & kValueMask;
                if ((v & ~kValueMask) == kFlagInclusive) break;
            }
            st_release_u32(my, kFlagInclusive | ((excl + agg) & kValueMask));
        }
        s_base[e] = s_eoff[e] + (int)excl;
    }
    __syncthreads();

    // 3) scatter rows: recv_token / recv_slot / pos
    const int nt = min(kLayoutTileTokens, tb + tc - t_tile0);
    for (int i = threadIdx.x; i < nt * k; i += blockDim.x) {
        const int ti = i / k, j = i % k;
        const int t = t_tile0 + ti;
        const size_t a = (size_t)t * k + j;
        int p = -1;
        if (keep[a]) {
            const int e = topk_idx[a];
            if (e >= 0 && e < E) {
                const int w = ti / kTokensPerWarp;
                const long long row = (long long)s_base[e] + s_cnt[w * E + e] + s_rank[ti * k + j];
                if (row >= 0 && row < n_rows_max) {
                    p = (int)row;
                    recv_token[p] = t;
                    recv_slot[p] = j;
                } else {
                    bad = true;
                }
            }
        }
        pos[(size_t)(t - tb) * k + j] = p;
    }
    if (bad) raise_status(status, MOE_DEV_BAD_INDEX);
}

__global__ void __launch_bounds__(kLayoutThreads) layout_splits_kernel(
    int tb, int tc, int ep, const int32_t *__restrict__ rank_offsets,
    const int32_t *__restrict__ recv_token, int32_t *__restrict__ send_splits) {
    extern __shared__ int32_t s_src[];  // [ep]
    const int d = blockIdx.x;
    for (int s = threadIdx.x; s < ep; s += blockDim.x) s_src[s] = 0;
    __syncthreads();
    const int tpr = tc / ep;
    const int p0 = rank_offsets[d], p1 = rank_offsets[d + 1];
    for (int p = p0 + threadIdx.x; p < p1; p += blockDim.x) {
        const int s = (recv_token[p] - tb) / tpr;
        const unsigned active = __activemask();
        const unsigned peers = __match_any_sync(active, s);
        if ((int)(threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&s_src[s], __popc(peers));
    }
    __syncthreads();
    for (int s = threadIdx.x; s < ep; s += blockDim.x) send_splits[(size_t)s * ep + d] = s_src[s];
}

size_t layout_scatter_smem(const moe_config &c) {
    return sizeof(int32_t) * ((size_t)(c.E + 1) + c.E + (size_t)kLayoutWarps * c.E +
                              (size_t)kLayoutTileTokens * c.k);
}

cudaError_t launch_dispatch_layout(const moe_config &c, int tb, int tc,
                                   const int32_t *topk_idx, const uint8_t *keep,
                                   int32_t *expert_offsets, int32_t *rank_offsets,
                                   int32_t *recv_token, int32_t *recv_slot, int32_t *pos,
                                   int32_t *send_splits, int32_t *splits_host, void *ws,
                                   int64_t n_rows_max, cudaStream_t s, int num_sms) {
    const ScratchLayout L = scratch_layout(c);
    uint32_t *status = ws_at<uint32_t>(ws, L.status);
    uint32_t *ticket = ws_at<uint32_t>(ws, L.ticket);
    int32_t *chunk_counts = ws_at<int32_t>(ws, L.chunk_counts);
    uint32_t *tile_state = ws_at<uint32_t>(ws, L.tile_state);
    const int n_tiles = (tc + kLayoutTileTokens - 1) / kLayoutTileTokens;
    // ticket, chunk counts and the tiles' look-back descriptors start at zero
    const size_t clear_bytes = L.tile_state - L.ticket + sizeof(uint32_t) * (size_t)n_tiles * c.E;
    cudaError_t err = cudaMemsetAsync(ws_at<char>(ws, L.ticket), 0, clear_bytes, s);
    if (err != cudaSuccess) return err;
    if (tc == 0) {
        err = cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (size_t)(c.E + 1), s);
        if (err == cudaSuccess) err = cudaMemsetAsync(rank_offsets, 0, sizeof(int32_t) * (size_t)(c.ep + 1), s);
        if (err == cudaSuccess) err = cudaMemsetAsync(send_splits, 0, sizeof(int32_t) * (size_t)c.ep * c.ep, s);
    } else {
        int hb = (int)(((size_t)tc * c.k + kLayoutThreads - 1) / kLayoutThreads);
        if (hb > num_sms * 4) hb = num_sms * 4;
        layout_hist_kernel<<<hb, kLayoutThreads, sizeof(int32_t) * c.E, s>>>(
            tb, tc, c.k, c.E, topk_idx, keep, chunk_counts);
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
        const size_t smem = layout_scatter_smem(c);
        err = cudaFuncSetAttribute(layout_scatter_kernel,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
        layout_scatter_kernel<<<n_tiles, kLayoutThreads, smem, s>>>(
            tb, tc, c.k, c.E, c.ep, n_rows_max, topk_idx, keep, chunk_counts, ticket, tile_state,
            expert_offsets, rank_offsets, recv_token, recv_slot, pos, status);
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
        layout_splits_kernel<<<c.ep, kLayoutThreads, sizeof(int32_t) * c.ep, s>>>(
            tb, tc, c.ep, rank_offsets, recv_token, send_splits);
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
    }
    if (err != cudaSuccess) return err;
    if (splits_host) {
        err = cudaMemcpyAsync(splits_host, expert_offsets, sizeof(int32_t) * (size_t)(c.E + 1),
                              cudaMemcpyDeviceToHost, s);
        if (err == cudaSuccess)
            err = cudaMemcpyAsync(splits_host + c.E + 1, send_splits,
                                  sizeof(int32_t) * (size_t)c.ep * c.ep, cudaMemcpyDeviceToHost, s);
    }
    return err;
}

}  // namespace moe
