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
//   layout_scatter  one CTA per tile of 64, 128 or 256 tokens (the smallest that
//                   keeps the launch within max(64, tokens / 256) tiles), taken in launch order
//                   from an atomic ticket.  Each tile ranks its assignments
//                   per expert in token order (warps walk their tokens with
//                   __match_any_sync), publishes its per-expert counts, and
//                   finds its prefix over earlier tiles by a decoupled
//                   look-back (Merrill & Garland 2016), one expert per thread.
//                   The row of (t, j) is expert_offsets[e] + (rows of e in
//                   earlier tiles) + (rank of t among this tile's rows of e).
//                   While scattering, each tile also counts its rows by
//                   (source rank, destination rank): the EP x EP
//                   all_to_all_single split matrix.
//
// The look-back waits are bounded: on a timeout the tile raises
// MOE_DEV_WAIT_TIMEOUT, publishes what it has so that later tiles finish,
// and skips every write that would leave the receive buffers.
#include <mutex>

#include "moe_common.cuh"

namespace moe {

constexpr int kLayoutThreads = 256;
constexpr int kLayoutWarps = kLayoutThreads / 32;
constexpr int kLoadBatch = 8;              // warp steps whose loads are issued together
constexpr uint32_t kFlagAggregate = 1u << 30;
constexpr uint32_t kFlagInclusive = 2u << 30;
constexpr uint32_t kValueMask = (1u << 30) - 1;

__global__ void __launch_bounds__(kLayoutThreads) layout_hist_kernel(
    int tb, int tc, int k, int E, int ep, const int32_t *__restrict__ topk_idx,
    const uint8_t *__restrict__ keep, int32_t *__restrict__ chunk_counts,
    int32_t *__restrict__ send_splits) {
    extern __shared__ int32_t s_hist[];
    for (int e = threadIdx.x; e < E; e += blockDim.x) s_hist[e] = 0;
    if (blockIdx.x == 0)   // the scatter kernel accumulates the split matrix into zeros
        for (int i = threadIdx.x; i < ep * ep; i += blockDim.x) send_splits[i] = 0;
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

// The split matrix is accumulated in shared memory when it fits.
constexpr int kSplitSmemMax = 4096;
constexpr int kLookbackWindow = 8;

__device__ __forceinline__ uint32_t ld_relaxed_u32(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Exclusive prefix of expert e over the tiles before `tile`, by decoupled
// look-back: descriptors pack a 2-bit flag (aggregate / inclusive prefix) and a
// 30-bit count in one word, so relaxed loads of the word are enough.  Loads run
// kLookbackWindow predecessors at a time.  Returns false if a predecessor never
// published within the wait limit.
__device__ __forceinline__ bool lookback_prefix(const uint32_t *tile_state, int tile, int E, int e,
                                                uint32_t &excl) {
    excl = 0;
    int p = tile - 1;
    while (p >= 0) {
        const int n = min(kLookbackWindow, p + 1);
        uint32_t v[kLookbackWindow];
#pragma unroll
        for (int i = 0; i < kLookbackWindow; ++i)
            if (i < n) v[i] = ld_relaxed_u32(tile_state + (size_t)(p - i) * E + e);
#pragma unroll
        for (int i = 0; i < kLookbackWindow; ++i) {
            if (i >= n) break;
            uint32_t w = v[i];
            if ((w >> 30) == 0 &&
                !wait_flag_word_bounded(tile_state + (size_t)(p - i) * E + e, w))
                return false;
            excl += w & kValueMask;
            if ((w & ~kValueMask) == kFlagInclusive) return true;
        }
        p -= n;
    }
    return true;
}

__global__ void __launch_bounds__(kLayoutThreads) layout_scatter_kernel(
    int tb, int tc, int k, int E, int ep, int tile_tokens, int64_t n_rows_max,
    const int32_t *__restrict__ topk_idx, const uint8_t *__restrict__ keep,
    const int32_t *__restrict__ chunk_counts, uint32_t *__restrict__ ticket,
    uint32_t *__restrict__ tile_state, int32_t *__restrict__ expert_offsets,
    int32_t *__restrict__ rank_offsets, int32_t *__restrict__ recv_token,
    int32_t *__restrict__ recv_slot, int32_t *__restrict__ pos, int32_t *__restrict__ send_splits,
    uint32_t *__restrict__ status) {
    extern __shared__ int32_t s_dyn[];
    int32_t *s_eoff = s_dyn;                                 // [E + 1]
    int32_t *s_base = s_eoff + (E + 1);                      // [E]
    int32_t *s_cnt = s_base + E;                             // [kLayoutWarps][E]
    int32_t *s_rank = s_cnt + kLayoutWarps * E;              // [tile_tokens * k]
    int32_t *s_exp = s_rank + tile_tokens * k;               // [tile_tokens * k] expert or -1
    int32_t *s_split = s_exp + tile_tokens * k;              // [ep * ep] when it fits
    __shared__ int32_t s_warp_tot[33];
    __shared__ uint32_t s_tile;
    const bool split_in_smem = ep * ep <= kSplitSmemMax;

    if (threadIdx.x == 0) s_tile = atomicAdd(ticket, 1u);
    for (int e = threadIdx.x; e < E; e += blockDim.x) s_eoff[e] = chunk_counts[e];
    for (int i = threadIdx.x; i < kLayoutWarps * E; i += blockDim.x) s_cnt[i] = 0;
    if (split_in_smem)
        for (int i = threadIdx.x; i < ep * ep; i += blockDim.x) s_split[i] = 0;
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

    // 1) rank every kept assignment of this tile among the warp's rows of its expert.
    // Warp w walks its tokens_per_warp tokens G = 32 / k at a time (lane -> token
    // b + lane / k, slot lane % k).  The experts of up to kLoadBatch steps are
    // loaded before the first is ranked, so a walk costs a memory round trip per
    // batch instead of per step; step 3 reads them back from shared memory.
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
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
            if (!lookback_prefix(tile_state, tile, E, e, excl)) {
                raise_status(status, MOE_DEV_WAIT_TIMEOUT);
                excl = 0x3FFFFFFFu;  // forces every write of this expert out of range
            }
            st_release_u32(my, kFlagInclusive | ((excl + agg) & kValueMask));
        }
        s_base[e] = s_eoff[e] + (int)excl;
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
    const int tile_tokens = layout_tile_tokens(tc);
    const int n_tiles = (tc + tile_tokens - 1) / tile_tokens;
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
        if (hb > num_sms * 2) hb = num_sms * 2;
        layout_hist_kernel<<<hb, kLayoutThreads, sizeof(int32_t) * c.E, s>>>(
            tb, tc, c.k, c.E, c.ep, topk_idx, keep, chunk_counts, send_splits);
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
        const size_t smem = layout_scatter_smem(c, tile_tokens);
        if ((err = g_scatter_opt_in.ensure(layout_scatter_kernel, smem)) != cudaSuccess) return err;
        layout_scatter_kernel<<<n_tiles, kLayoutThreads, smem, s>>>(
            tb, tc, c.k, c.E, c.ep, tile_tokens, n_rows_max, topk_idx, keep, chunk_counts, ticket, tile_state,
            expert_offsets, rank_offsets, recv_token, recv_slot, pos, send_splits, status);
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

// ---------------------------------------------------------------------------
// Allocation-free variant of moe_dispatch_layout.
//
// Some callers cannot call cudaMalloc or hand the library a workspace: code
// that runs while another framework is capturing the stream into a CUDA graph
// (an allocation there would break or be left out of the capture), code whose
// device memory all belongs to an allocator it does not control (a
// pre-reserved pool it may not grow), and latency-critical loops that must not
// hit the implicit device synchronisation of cudaMalloc / cudaFree.  For them
// this entry point keeps the dispatch layout's scratch (the tile ticket, the
// chunk's per-expert counts and the look-back descriptors) in one fixed
// device array inside the library instead of a caller workspace.
//
// Limits: at most kNoAllocMaxTiles * 256 tokens per call and E <= 1024.  The
// array (about 261 KiB) exists on every device that loads the library, until
// the process exits.  Every call shares it: calls that may overlap on the GPU
// (different streams without ordering, or several host threads) race and
// corrupt each other's layouts; order them.  The first call on a device looks
// up the array's device address (cudaGetSymbolAddress) with that device
// current; make that first call before any stream capture.  The address is
// looked up again when the device's context has changed since (after a
// cudaDeviceReset, which reloads the module and may move the array).
namespace {

constexpr int kNoAllocMaxTiles = 64;   // 16384 tokens per call
constexpr size_t kNoAllocTicket = 0;
constexpr size_t kNoAllocStatus = 256;
constexpr size_t kNoAllocCounts = 512;
constexpr size_t kNoAllocTiles = kNoAllocCounts + sizeof(int32_t) * moe::kMaxExperts;
constexpr size_t kNoAllocBytes = kNoAllocTiles + sizeof(uint32_t) * (size_t)kNoAllocMaxTiles * moe::kMaxExperts;

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
    uint32_t *ticket = reinterpret_cast<uint32_t *>(b + kNoAllocTicket);
    uint32_t *st_word = status ? status : reinterpret_cast<uint32_t *>(b + kNoAllocStatus);
    int32_t *chunk_counts = reinterpret_cast<int32_t *>(b + kNoAllocCounts);
    uint32_t *tile_state = reinterpret_cast<uint32_t *>(b + kNoAllocTiles);
    const int num_sms = [] { int d = 0, n = 148; cudaGetDevice(&d); cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d); return n; }();
    // the previous call's ticket, counts and look-back descriptors start again at zero
    err = cudaMemsetAsync(b, 0, kNoAllocTiles + sizeof(uint32_t) * (size_t)n_tiles * c.E, stream);
    if (err == cudaSuccess && tok_count == 0) {
        err = cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (size_t)(c.E + 1), stream);
        if (err == cudaSuccess) err = cudaMemsetAsync(rank_offsets, 0, sizeof(int32_t) * (size_t)(c.ep + 1), stream);
        if (err == cudaSuccess) err = cudaMemsetAsync(send_splits, 0, sizeof(int32_t) * (size_t)c.ep * c.ep, stream);
    } else if (err == cudaSuccess) {
        int hb = (int)(((size_t)tok_count * c.k + kLayoutThreads - 1) / kLayoutThreads);
        if (hb > num_sms * 2) hb = num_sms * 2;
        layout_hist_kernel<<<hb, kLayoutThreads, sizeof(int32_t) * c.E, stream>>>(
            tok_begin, tok_count, c.k, c.E, c.ep, topk_idx, keep, chunk_counts, send_splits);
        err = cudaGetLastError();
        const size_t smem = layout_scatter_smem(c, tile_tokens);
        if (err == cudaSuccess) err = g_scatter_opt_in.ensure(layout_scatter_kernel, smem);
        if (err == cudaSuccess) {
            layout_scatter_kernel<<<n_tiles, kLayoutThreads, smem, stream>>>(
                tok_begin, tok_count, c.k, c.E, c.ep, tile_tokens, max_recv_rows_of(c, tok_count), topk_idx, keep,
                chunk_counts, ticket, tile_state, expert_offsets, rank_offsets, recv_token, recv_slot,
                pos, send_splits, st_word);
            err = cudaGetLastError();
        }
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
