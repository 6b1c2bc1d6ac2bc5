// Step 3: dispatch layout (axolotl ExpertParallelArgs, expert_parallel_backend
// = torch: all_to_all_single over the EP group; LightLLM PR 1687: the expert
// prefix-sum "psum" layout that the grouped GEMM consumes).
//
// Receive rows are the kept (token, expert) assignments of a token chunk in
// stable order by (expert, token).  With experts owned by contiguous rank
// blocks this is also the (destination rank, expert, token) order, i.e. the
// all_to_all_single arrival order regrouped by expert.  The order is built by
// a stable counting sort over tiles of 64, 128 or 256 tokens (the smallest
// that keeps the launch within max(64, tokens / 256) tiles):
//
//   layout_hist     one CTA per tile: the tile's kept assignments per expert
//                   (shared-memory histogram), written column by column to
//                   tile_counts[expert][tile], zeros included;
//   layout_scatter  one CTA per tile.  Each warp sums one expert's column of
//                   tile_counts at a time (lanes over tiles, two warp
//                   reductions): the expert's rows in the tiles before this one
//                   and in the whole chunk; a block scan of the totals gives the
//                   expert offsets.  The tile ranks its assignments per expert in
//                   token order (warps walk their tokens with __match_any_sync);
//                   the row of (t, j) is expert_offsets[e] + (rows of e in earlier
//                   tiles) + (rank of t among this tile's rows of e).  While
//                   scattering, each tile also counts its rows by (source rank,
//                   destination rank): the EP x EP all_to_all_single split matrix.
//
// No CTA waits for another: the first kernel's histograms are complete when the
// second starts, and every scatter CTA reads them all (n_tiles x E counts, from
// L2).  Rows outside the receive buffer, and expert ids outside [0, E) of kept
// assignments, raise MOE_DEV_BAD_INDEX and are not written.
#include <mutex>

#include "moe_common.cuh"

namespace moe {

constexpr int kLayoutThreads = 256;
constexpr int kLayoutWarps = kLayoutThreads / 32;
constexpr int kLoadBatch = 8;              // warp steps whose loads are issued together

__global__ void __launch_bounds__(kLayoutThreads) layout_hist_kernel(
    int tb, int tc, int k, int E, int ep, int tile_tokens, int n_tiles, const int32_t *__restrict__ topk_idx,
    const uint8_t *__restrict__ keep, int32_t *__restrict__ tile_counts, int32_t *__restrict__ send_splits) {
    grid_dependency_wait();
    grid_dependents_launch();
    extern __shared__ int32_t s_hist[];
    for (int e = threadIdx.x; e < E; e += blockDim.x) s_hist[e] = 0;
    if (blockIdx.x == 0)   // the scatter kernel accumulates the split matrix into zeros
        for (int i = threadIdx.x; i < ep * ep; i += blockDim.x) send_splits[i] = 0;
    __syncthreads();
    const int t0 = tb + blockIdx.x * tile_tokens;
    const int t1 = min(tb + tc, t0 + tile_tokens);
    for (size_t a = (size_t)t0 * k + threadIdx.x; a < (size_t)t1 * k; a += blockDim.x) {
        const int e = keep[a] ? topk_idx[a] : -1;
        if (e >= 0 && e < E) atomicAdd(&s_hist[e], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) tile_counts[(size_t)e * n_tiles + blockIdx.x] = s_hist[e];
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

// The split matrix is accumulated in shared memory when it fits.
constexpr int kSplitSmemMax = 4096;
constexpr int kColBatch = 8;   // expert columns a warp sums together (loads in flight)

__global__ void __launch_bounds__(kLayoutThreads) layout_scatter_kernel(
    int tb, int tc, int k, int E, int ep, int tile_tokens, int n_tiles, int64_t n_rows_max,
    const int32_t *__restrict__ topk_idx, const uint8_t *__restrict__ keep,
    const int32_t *__restrict__ tile_counts, int32_t *__restrict__ expert_offsets,
    int32_t *__restrict__ rank_offsets, int32_t *__restrict__ recv_token,
    int32_t *__restrict__ recv_slot, int32_t *__restrict__ pos, int32_t *__restrict__ send_splits,
    uint32_t *__restrict__ status) {
    grid_dependency_wait();
    grid_dependents_launch();
    extern __shared__ int32_t s_dyn[];
    int32_t *s_eoff = s_dyn;                                 // [E + 1]
    int32_t *s_base = s_eoff + (E + 1);                      // [E]
    int32_t *s_cnt = s_base + E;                             // [kLayoutWarps][E]
    int32_t *s_rank = s_cnt + kLayoutWarps * E;              // [tile_tokens * k]
    int32_t *s_exp = s_rank + tile_tokens * k;               // [tile_tokens * k] expert or -1
    int32_t *s_split = s_exp + tile_tokens * k;              // [ep * ep] when it fits
    __shared__ int32_t s_warp_tot[33];
    const bool split_in_smem = ep * ep <= kSplitSmemMax;
    const int tile = blockIdx.x;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;

    for (int i = threadIdx.x; i < kLayoutWarps * E; i += blockDim.x) s_cnt[i] = 0;
    if (split_in_smem)
        for (int i = threadIdx.x; i < ep * ep; i += blockDim.x) s_split[i] = 0;
    // 0) each expert's rows in the tiles before this one (s_base) and in the chunk
    // (s_eoff): warp w sums the columns of experts w, w + 8, ..., kColBatch at a
    // time, lane j the tiles j, j + 32, ...
    for (int e0 = wid; e0 < E; e0 += kLayoutWarps * kColBatch) {
        int pre[kColBatch], tot[kColBatch];
#pragma unroll
        for (int u = 0; u < kColBatch; ++u) pre[u] = tot[u] = 0;
        for (int j = lane; j < n_tiles; j += 32) {
            int v[kColBatch];
#pragma unroll
            for (int u = 0; u < kColBatch; ++u) {
                const int e = e0 + u * kLayoutWarps;
                v[u] = e < E ? __ldg(tile_counts + (size_t)e * n_tiles + j) : 0;
            }
#pragma unroll
            for (int u = 0; u < kColBatch; ++u) {
                tot[u] += v[u];
                if (j < tile) pre[u] += v[u];
            }
        }
#pragma unroll
        for (int u = 0; u < kColBatch; ++u) {
            const int e = e0 + u * kLayoutWarps;
            const int p = __reduce_add_sync(0xffffffffu, pre[u]);
            const int q = __reduce_add_sync(0xffffffffu, tot[u]);
            if (lane == 0 && e < E) { s_base[e] = p; s_eoff[e] = q; }
        }
    }
    __syncthreads();
    const int total = block_exclusive_scan(s_eoff, E, s_warp_tot);
    if (threadIdx.x == 0) s_eoff[E] = total;
    __syncthreads();

    if (tile == 0) {
        const int epr = E / ep;
        for (int e = threadIdx.x; e <= E; e += blockDim.x) expert_offsets[e] = s_eoff[e];
        for (int d = threadIdx.x; d <= ep; d += blockDim.x) rank_offsets[d] = s_eoff[d * epr];
    }

    // 1) rank every kept assignment of this tile among the warp's rows of its expert.
    // Warp w walks its tokens_per_warp tokens G = 32 / k at a time (lane -> token
    // b + lane / k, slot lane % k).  The experts of up to kLoadBatch steps are
    // loaded before the first is ranked, so a walk costs a memory round trip per
    // batch instead of per step; step 3 reads them back from shared memory.
    const int t_tile0 = tb + tile * tile_tokens;
    const int tokens_per_warp = tile_tokens / kLayoutWarps;   // 8, 16 or 32
    const int G = 32 / k;                      // tokens per warp step
    const int n_steps = (tokens_per_warp + G - 1) / G;
    const unsigned lt_mask = (1u << lane) - 1u;
    const int jl = lane % k;
    bool bad = false;
    for (int s0 = 0; s0 < n_steps; s0 += kLoadBatch) {
        uint8_t kv[kLoadBatch];
        int ix[kLoadBatch];
#pragma unroll
        for (int i = 0; i < kLoadBatch; ++i) {
            kv[i] = 0;
            ix[i] = -1;
            const int b = (s0 + i) * G;
            const int t = t_tile0 + wid * tokens_per_warp + b + lane / k;
            if (s0 + i < n_steps && lane < G * k && b + lane / k < tokens_per_warp && t < tb + tc) {
                const size_t a = (size_t)t * k + jl;
                kv[i] = __ldg(keep + a);
                ix[i] = __ldg(topk_idx + a);
            }
        }
#pragma unroll
        for (int i = 0; i < kLoadBatch; ++i) {
            if (s0 + i >= n_steps) break;
            const int b = (s0 + i) * G;
            const int ti = wid * tokens_per_warp + b + lane / k;   // token within the tile
            const bool mine = lane < G * k && b + lane / k < tokens_per_warp;
            int e = -1;
            if (kv[i]) {
                if (ix[i] >= 0 && ix[i] < E) e = ix[i];
                else bad = true;
            }
            if (mine) s_exp[ti * k + jl] = e;
            const int me = e >= 0 ? e : -1 - lane;                 // unique sentinel: matches nobody
            const unsigned peers = __match_any_sync(0xffffffffu, me);
            if (e >= 0) s_rank[ti * k + jl] = s_cnt[wid * E + e] + __popc(peers & lt_mask);
            __syncwarp();
            if (e >= 0 && (31 - __clz(peers)) == lane) s_cnt[wid * E + e] += __popc(peers);
            __syncwarp();
        }
    }
    __syncthreads();

    // 2) per-expert warp offsets inside the tile; the tile's first row of each expert
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = 0;
        for (int w = 0; w < kLayoutWarps; ++w) {
            const int c = s_cnt[w * E + e];
            s_cnt[w * E + e] = run;
            run += c;
        }
        s_base[e] += s_eoff[e];
    }
    __syncthreads();

    // 3) scatter rows (recv_token / recv_slot / pos) and count the split matrix,
    // with the same lane -> assignment map as step 1
    const int tpr = tc / ep, epr = E / ep;
    for (int st = 0; st < n_steps; ++st) {
        const int b = st * G;
        const int ti = wid * tokens_per_warp + b + lane / k;
        const int t = t_tile0 + ti;
        const bool mine = lane < G * k && b + lane / k < tokens_per_warp && t < tb + tc;
        int p = -1;
        int key = -1;
        const int e = mine ? s_exp[ti * k + jl] : -1;
        if (mine && e >= 0) {
            const long long row = (long long)s_base[e] + s_cnt[wid * E + e] + s_rank[ti * k + jl];
            if (row >= 0 && row < n_rows_max) {
                p = (int)row;
                recv_token[p] = t;
                recv_slot[p] = jl;
                key = ((t - tb) / tpr) * ep + e / epr;
            } else {
                bad = true;
            }
        }
        if (mine) pos[(size_t)(t - tb) * k + jl] = p;
        const unsigned peers = __match_any_sync(0xffffffffu, key);
        if (key >= 0 && lane == __ffs(peers) - 1) {
            if (split_in_smem) atomicAdd(&s_split[key], __popc(peers));
            else atomicAdd(&send_splits[key], __popc(peers));
        }
    }
    if (split_in_smem) {
        __syncthreads();
        for (int i = threadIdx.x; i < ep * ep; i += blockDim.x)
            if (s_split[i]) atomicAdd(&send_splits[i], s_split[i]);
    }
    if (bad) raise_status(status, MOE_DEV_BAD_INDEX);
}

size_t layout_scatter_smem(const moe_config &c, int tile_tokens) {
    const size_t split = (size_t)c.ep * c.ep <= (size_t)kSplitSmemMax ? (size_t)c.ep * c.ep : 0;
    return sizeof(int32_t) * ((size_t)(c.E + 1) + c.E + (size_t)kLayoutWarps * c.E +
                              2 * (size_t)tile_tokens * c.k + split);
}

// The scatter's dynamic shared memory opt-in, shared by the workspace and the
// allocation-free entry points.
SmemOptIn g_scatter_opt_in;

// Both layout kernels over tc > 0 tokens; tile_counts holds n_tiles * E int32.
cudaError_t launch_layout_kernels(const moe_config &c, int tb, int tc, const int32_t *topk_idx,
                                  const uint8_t *keep, int32_t *tile_counts, int32_t *expert_offsets,
                                  int32_t *rank_offsets, int32_t *recv_token, int32_t *recv_slot, int32_t *pos,
                                  int32_t *send_splits, uint32_t *status, int64_t n_rows_max, cudaStream_t s) {
    const int tile_tokens = layout_tile_tokens(tc);
    const int n_tiles = (tc + tile_tokens - 1) / tile_tokens;
    cudaError_t err = launch_dependent(layout_hist_kernel, n_tiles, kLayoutThreads, sizeof(int32_t) * c.E, s,
                                       tb, tc, c.k, c.E, c.ep, tile_tokens, n_tiles, topk_idx, keep, tile_counts,
                                       send_splits);
    if (err != cudaSuccess) return err;
    const size_t smem = layout_scatter_smem(c, tile_tokens);
    if ((err = g_scatter_opt_in.ensure(layout_scatter_kernel, smem)) != cudaSuccess) return err;
    return launch_dependent(layout_scatter_kernel, n_tiles, kLayoutThreads, smem, s, tb, tc, c.k, c.E, c.ep,
                            tile_tokens, n_tiles, n_rows_max, topk_idx, keep, tile_counts, expert_offsets,
                            rank_offsets, recv_token, recv_slot, pos, send_splits, status);
}

cudaError_t launch_dispatch_layout(const moe_config &c, int tb, int tc,
                                   const int32_t *topk_idx, const uint8_t *keep,
                                   int32_t *expert_offsets, int32_t *rank_offsets,
                                   int32_t *recv_token, int32_t *recv_slot, int32_t *pos,
                                   int32_t *send_splits, int32_t *splits_host, void *ws,
                                   int64_t n_rows_max, cudaStream_t s, int num_sms) {
    const ScratchLayout L = scratch_layout(c);
    uint32_t *status = ws_at<uint32_t>(ws, L.status);
    int32_t *tile_counts = ws_at<int32_t>(ws, L.tile_counts);
    cudaError_t err = cudaSuccess;
    if (tc == 0) {
        err = cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (size_t)(c.E + 1), s);
        if (err == cudaSuccess) err = cudaMemsetAsync(rank_offsets, 0, sizeof(int32_t) * (size_t)(c.ep + 1), s);
        if (err == cudaSuccess) err = cudaMemsetAsync(send_splits, 0, sizeof(int32_t) * (size_t)c.ep * c.ep, s);
    } else {
        err = launch_layout_kernels(c, tb, tc, topk_idx, keep, tile_counts, expert_offsets, rank_offsets,
                                    recv_token, recv_slot, pos, send_splits, status, n_rows_max, s);
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

// ---------------------------------------------------------------------------
// Allocation-free variant of moe_dispatch_layout.
//
// Some callers cannot call cudaMalloc or hand the library a workspace: code
// that runs while another framework is capturing the stream into a CUDA graph
// (an allocation there would break or be left out of the capture), code whose
// device memory all belongs to an allocator it does not control (a
// pre-reserved pool it may not grow), and latency-critical loops that must not
// hit the implicit device synchronisation of cudaMalloc / cudaFree.  For them
// this entry point keeps the dispatch layout's scratch (a status word and the
// tiles' per-expert counts) in one fixed device array inside the library
// instead of a caller workspace.
//
// Limits: at most kNoAllocMaxTiles * 256 tokens per call and E <= 1024.  The
// array (about 256 KiB) exists on every device that loads the library, until
// the process exits.  Every call shares it: calls that may overlap on the GPU
// (different streams without ordering, or several host threads) race and
// corrupt each other's layouts; order them.  The first call on a device looks
// up the array's device address (cudaGetSymbolAddress) with that device
// current; make that first call before any stream capture.  The address is
// looked up again when the device's context has changed since (after a
// cudaDeviceReset, which reloads the module and may move the array).
namespace {

constexpr int kNoAllocMaxTiles = 64;   // 16384 tokens per call
constexpr size_t kNoAllocStatus = 0;
constexpr size_t kNoAllocTiles = 256;
constexpr size_t kNoAllocBytes = kNoAllocTiles + sizeof(int32_t) * (size_t)kNoAllocMaxTiles * moe::kMaxExperts;

static __device__ __align__(256) unsigned char g_noalloc_layout_scratch[kNoAllocBytes];

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mutex;
void *g_noalloc_base[kNoAllocMaxDevices] = {};
unsigned long long g_noalloc_ctx[kNoAllocMaxDevices] = {};

// Device address of the array for the current device: looked up once per
// device and context (the context id is 0 before the first lookup has created
// the context, or when the driver cannot report it: then it is looked up on
// every call).
cudaError_t noalloc_scratch(void **out) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= kNoAllocMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    const unsigned long long ctx = moe::current_context_id();
    if (!g_noalloc_base[dev] || ctx == 0 || ctx != g_noalloc_ctx[dev]) {
        void *p = nullptr;
        err = cudaGetSymbolAddress(&p, g_noalloc_layout_scratch);
        if (err != cudaSuccess) return err;
        g_noalloc_base[dev] = p;
        g_noalloc_ctx[dev] = moe::current_context_id();
    }
    *out = g_noalloc_base[dev];
    return cudaSuccess;
}

}  // namespace

namespace moe {
moe_status report_error(moe_status st, const char *msg);
int64_t max_recv_rows_of(const moe_config &c, int32_t tok_count);
}

extern "C" moe_status moe_dispatch_layout_noalloc(
    const moe_config *cfg, int32_t tok_begin, int32_t tok_count, const int32_t *topk_idx,
    const uint8_t *keep, int32_t *expert_offsets, int32_t *rank_offsets, int32_t *recv_token,
    int32_t *recv_slot, int32_t *pos, int32_t *send_splits, int32_t *splits_host,
    uint32_t *status, cudaStream_t stream) {
    using namespace moe;
    moe_status st = moe_config_check(cfg);
    if (st != MOE_OK) return st;
    const moe_config &c = *cfg;
    if (tok_begin < 0 || tok_count < 0 || (int64_t)tok_begin + tok_count > c.T || tok_count % c.ep != 0)
        return report_error(MOE_ERR_INVALID_ARG, "token range outside [0, T) or not divisible by ep");
    const int tile_tokens = layout_tile_tokens(tok_count);
    const int n_tiles = (tok_count + tile_tokens - 1) / tile_tokens;
    if (n_tiles > kNoAllocMaxTiles)
        return report_error(MOE_ERR_UNSUPPORTED,
                            "moe_dispatch_layout_noalloc handles at most 16384 tokens per call");
    if (!expert_offsets || !rank_offsets || !send_splits ||
        (tok_count > 0 && (!topk_idx || !keep || !recv_token || !recv_slot || !pos)))
        return report_error(MOE_ERR_INVALID_ARG, "NULL pointer argument");
    void *base = nullptr;
    cudaError_t err = noalloc_scratch(&base);
    if (err != cudaSuccess) return report_error(MOE_ERR_CUDA, cudaGetErrorString(err));
    unsigned char *b = static_cast<unsigned char *>(base);
    uint32_t *st_word = status ? status : reinterpret_cast<uint32_t *>(b + kNoAllocStatus);
    int32_t *tile_counts = reinterpret_cast<int32_t *>(b + kNoAllocTiles);
    if (tok_count == 0) {
        err = cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (size_t)(c.E + 1), stream);
        if (err == cudaSuccess) err = cudaMemsetAsync(rank_offsets, 0, sizeof(int32_t) * (size_t)(c.ep + 1), stream);
        if (err == cudaSuccess) err = cudaMemsetAsync(send_splits, 0, sizeof(int32_t) * (size_t)c.ep * c.ep, stream);
    } else {
        err = launch_layout_kernels(c, tok_begin, tok_count, topk_idx, keep, tile_counts, expert_offsets,
                                    rank_offsets, recv_token, recv_slot, pos, send_splits, st_word,
                                    max_recv_rows_of(c, tok_count), stream);
    }
    if (err == cudaSuccess && splits_host) {
        err = cudaMemcpyAsync(splits_host, expert_offsets, sizeof(int32_t) * (size_t)(c.E + 1),
                              cudaMemcpyDeviceToHost, stream);
        if (err == cudaSuccess)
            err = cudaMemcpyAsync(splits_host + c.E + 1, send_splits,
                                  sizeof(int32_t) * (size_t)c.ep * c.ep, cudaMemcpyDeviceToHost, stream);
    }
    if (err != cudaSuccess) return report_error(MOE_ERR_CUDA, cudaGetErrorString(err));
    return MOE_OK;
}
