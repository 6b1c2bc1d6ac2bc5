// Shared device helpers of the sm_100a MoE kernels: workspace layout, the
// device status word, bounded waits, and thin inline-PTX wrappers for
// mbarriers, TMA and tcgen05 (5th-generation tensor cores with TMEM).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <mutex>

#include "../../include/moe_b200.h"

namespace moe {

// ---------------------------------------------------------------- constants
constexpr int kMaxTopK = 32;
constexpr int kMaxExperts = 1024;
constexpr int kMaxGroups = 32;              // grouped top-k: groups per token
constexpr int kLayoutTileTokens = 256;      // largest dispatch-layout tile (tokens)
constexpr int kLayoutMinTiles = 64;         // tiles shrink while there are at most this many

// A dispatch-layout launch over tc tokens uses tiles of 64, 128 or 256 tokens:
// the smallest that keeps the tile count within max(64, ceil(tc / 256)), so a
// chunk of a few thousand tokens still spreads over dozens of CTAs.
inline int layout_tile_tokens(int64_t tc) {
    const int64_t cap = (tc + kLayoutTileTokens - 1) / kLayoutTileTokens;
    const int64_t max_tiles = cap > kLayoutMinTiles ? cap : kLayoutMinTiles;
    for (int t = kLayoutTileTokens / 4; t < kLayoutTileTokens; t *= 2)
        if ((tc + t - 1) / t <= max_tiles) return t;
    return kLayoutTileTokens;
}
inline int64_t layout_max_tiles(int64_t tc) {
    const int64_t cap = (tc + kLayoutTileTokens - 1) / kLayoutTileTokens;
    return cap > kLayoutMinTiles ? cap : kLayoutMinTiles;
}
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // a bounded wait gives up after 2 s

// Unique id of the CUDA context current on the calling thread (cuCtxGetId), 0
// when no context is current yet or the driver does not offer the call.  A
// device reset (cudaDeviceReset) replaces the context, and with it every
// module-level state: kernel attributes and the addresses of __device__
// variables.  Per-device caches of such state compare this id to notice it.
inline unsigned long long current_context_id() {
    using GetCurrent = CUresult (*)(CUcontext *);
    using GetId = CUresult (*)(CUcontext, unsigned long long *);
    struct Fns {
        GetCurrent cur = nullptr;
        GetId id = nullptr;
        Fns() {
            void *p = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
                q == cudaDriverEntryPointSuccess)
                cur = reinterpret_cast<GetCurrent>(p);
            p = nullptr;
            if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
                q == cudaDriverEntryPointSuccess)
                id = reinterpret_cast<GetId>(p);
        }
    };
    static const Fns fns;   // looked up once per process
    if (!fns.cur || !fns.id) return 0;
    CUcontext ctx = nullptr;
    if (fns.cur(&ctx) != CUDA_SUCCESS || !ctx) return 0;
    unsigned long long v = 0;
    return fns.id(ctx, &v) == CUDA_SUCCESS ? v : 0;
}

// Opens a kernel's dynamic shared memory beyond the default 48 KiB.  The
// attribute belongs to the device's current context, so the largest size
// already set is remembered per device together with the context it was set
// in; a new context (after a device reset) starts again from the default.
class SmemOptIn {
  public:
    template <typename Kernel>
    cudaError_t ensure(Kernel *kernel, size_t bytes) {
        if (bytes <= kDefault) return cudaSuccess;
        int dev = 0;
        cudaError_t err = cudaGetDevice(&dev);
        if (err != cudaSuccess) return err;
        const unsigned long long ctx = current_context_id();
        if (dev < 0 || dev >= kDevices || ctx == 0)
            return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
        std::lock_guard<std::mutex> lock(m_);
        if (ctx_[dev] != ctx) { ctx_[dev] = ctx; set_[dev] = 0; }
        if (bytes <= set_[dev]) return cudaSuccess;
        err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
        if (err == cudaSuccess) set_[dev] = bytes;
        return err;
    }

  private:
    static constexpr size_t kDefault = 48 * 1024;
    static constexpr int kDevices = 64;
    std::mutex m_;
    size_t set_[kDevices] = {};
    unsigned long long ctx_[kDevices] = {};
};

// ---------------------------------------------------------------- workspace
// Scratch layout (all offsets 256-byte aligned):
//   [0, 256)        status word (uint32 at offset 0)
//   tile_counts     int32[E * max_tiles] (dispatch layout: rows per expert and tile)
//   clip threshold  uint64[E]
//   ffn counters    uint32[2] (dynamic work distribution of the FFN GEMMs)
//   shared expert   uint32[2] counters, int32[2] expert offsets
//   clip segments   int32[2 * (E + 1)] offsets / cursors, keys uint64[T * k]
struct ScratchLayout {
    size_t status, tile_counts, clip_thr, ffn_ctr;
    size_t shared_ctr, shared_off;
    size_t clip_seg, clip_keys, total;
    int max_tiles;
};

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

inline ScratchLayout scratch_layout(const moe_config &c) {
    ScratchLayout L{};
    size_t off = 0;
    L.status = off;               off += 256;
    L.max_tiles = (int)layout_max_tiles(c.T);
    L.tile_counts = off;          off = align_up(off + sizeof(int32_t) * (size_t)L.max_tiles * c.E, 256);
    L.clip_thr = off;             off = align_up(off + sizeof(uint64_t) * (size_t)c.E, 256);
    L.ffn_ctr = off;              off += 256;   // work counters of the two FFN launches
    L.shared_ctr = off;           off += 256;   // the shared expert's own two counters
    L.shared_off = off;           off += 256;   // its expert offsets {0, rows}
    L.clip_seg = off;             off = align_up(off + sizeof(int32_t) * 2 * ((size_t)c.E + 1), 256);
    L.clip_keys = off;            off = align_up(off + sizeof(uint64_t) * (size_t)c.T * c.k, 256);
    L.total = off;
    return L;
}

template <typename T>
inline T *ws_at(void *ws, size_t off) { return reinterpret_cast<T *>(static_cast<char *>(ws) + off); }

// ---------------------------------------------------------------- device status
__device__ __forceinline__ void raise_status(uint32_t *status, uint32_t bits) {
    atomicOr(status, bits);
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------- shared memory
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarriers
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}"
                 ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}
// Waits for the phase with the given parity to complete.  Gives up after
// kWaitLimitNs or as soon as another role of the CTA set *abort_flag;
// returns false then.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity,
                                                  volatile int *abort_flag,
                                                  uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 0u) {
            if (*abort_flag) return false;
            if (global_timer_ns() - t0 > limit_ns) return false;
        }
    }
}

// ---------------------------------------------------------------- dependent launch
// The index-path, permute and combine kernels are launched with programmatic
// stream serialisation: the GPU may start one while the kernel before it in the
// stream is still finishing, which hides the launch gap between two dependent
// kernels.  Each such kernel calls grid_dependency_wait() before its first
// global-memory access, in every thread: the wait returns once the earlier
// kernels of the stream have completed and their writes are visible (at once
// when the kernel was launched without the attribute).  grid_dependents_launch()
// lets the next kernel be scheduled early; it still waits for this one to
// complete before it touches memory.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dependents_launch() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_dependent(void (*kernel)(KArgs...), unsigned grid, unsigned block, size_t smem,
                                    cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const void *tmap) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Waits for this thread's TMEM loads and ties r to the wait, so that no use of
// r can be scheduled before the data has arrived.
__device__ __forceinline__ void tc_wait_ld_regs(uint32_t (&r)[32]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                   "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                   "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]),
                   "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                   "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                   "+r"(r[30]), "+r"(r[31])
                 :: "memory");
}
// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp gets lane (base lane + i).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 "
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
                 "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
                   "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]),
                   "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
                   "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
                   "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr) : "memory");
}

// ---------------------------------------------------------------- CTA pairs (clusters of 2)
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// shared::cluster address of the same shared-memory object in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t mapa_shared(uint32_t smem_addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
    return r;
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// Arrive on a (possibly remote) mbarrier with cluster-scope release: orders this
// thread's earlier shared::cluster stores before the arrival.
__device__ __forceinline__ void mbar_arrive_cluster_release(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ void st_cluster_u32(uint32_t cluster_addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}
// try_wait with cluster-scope acquire (pairs with mbar_arrive_cluster_release)
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_cluster_bounded(uint64_t *bar, uint32_t parity,
                                                          volatile int *abort_flag,
                                                          uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait_cluster(bar, parity)) return true;
        if ((i & 255u) == 0u) {
            if (*abort_flag) return false;
            if (global_timer_ns() - t0 > limit_ns) return false;
        }
    }
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// TMA loads into this CTA's shared memory whose completion is counted on an
// mbarrier that may live in the peer CTA of the pair (no multicast).
__device__ __forceinline__ void tma_load_3d_pair(void *smem_dst, const void *tmap, uint32_t mbar_cluster_addr,
                                                 int32_t x, int32_t y, int32_t z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];"
        ::"r"(smem_u32(smem_dst)), "l"(tmap), "r"(mbar_cluster_addr), "r"(x), "r"(y), "r"(z)
        : "memory");
}
__device__ __forceinline__ void tma_load_4d_pair(void *smem_dst, const void *tmap, uint32_t mbar_cluster_addr,
                                                 int32_t x, int32_t y, int32_t z, int32_t w) {
    asm volatile(
        "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];"
        ::"r"(smem_u32(smem_dst)), "l"(tmap), "r"(mbar_cluster_addr), "r"(x), "r"(y), "r"(z), "r"(w)
        : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t *smem_dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(smem_dst)), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// D (+)= A * B^T across the CTA pair: A rows split over the two CTAs (M/2 each),
// B rows split over the two CTAs (N/2 each); issued by the pair's leader only.
__device__ __forceinline__ void tc_mma_f16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                                uint32_t idesc, uint32_t accumulate) {
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                 ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}
// The same with E4M3 operands (kind::f8f6f4), fp32 accumulator.
__device__ __forceinline__ void tc_mma_f8_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
                 ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}
// Arrives once on the mbarrier at the same offset in every CTA of cta_mask when
// all tcgen05 ops issued so far by this thread complete.
__device__ __forceinline__ void tc_commit_pair_mc(uint64_t *bar, uint16_t cta_mask) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
                 ::"r"(smem_u32(bar)), "h"(cta_mask) : "memory");
}

// Shared-memory matrix descriptor for a K-major operand tile stored with the
// 128-byte swizzle that TMA writes: rows of 64 bf16 (128 B), 8-row core groups
// 1024 B apart.  Fields: start address >> 4 in bits [0,14), leading byte
// offset (unused for this swizzle, set to 1) in [16,30), stride byte offset
// 1024 >> 4 in [32,46), descriptor version 1 in [46,48), swizzle mode 2
// (128 B) in [61,64).
__device__ __forceinline__ uint64_t make_sw128_desc(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}

// Instruction descriptor of kind::f16 with bf16 A and B, fp32 accumulator,
// both operands K-major: c_format (F32 = 1) bits [4,6), a_format (BF16 = 1)
// [7,10), b_format (BF16 = 1) [10,13), N >> 3 in [17,23), M >> 4 in [24,29).
__host__ __device__ constexpr uint32_t make_idesc_bf16_f32(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

// Instruction descriptor of kind::f8f6f4 with E4M3 A and B (format code 0 in
// both [7,10) and [10,13)), fp32 accumulator, both operands K-major.
__host__ __device__ constexpr uint32_t make_idesc_e4m3_f32(int M, int N) {
    return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// kind::f16 with bf16 A and B and an fp32 accumulator, with the major-ness of
// each operand: bit 15 set = A is MN-major, bit 16 set = B is MN-major.
__host__ __device__ constexpr uint32_t make_idesc_bf16_f32_major(int M, int N, bool a_mn, bool b_mn) {
    return make_idesc_bf16_f32(M, N) | (a_mn ? 1u << 15 : 0u) | (b_mn ? 1u << 16 : 0u);
}

// Shared-memory descriptor of an MN-major operand stored with the 128-byte
// swizzle: each 128-byte row holds 64 consecutive M (or N) elements of one k,
// 8 consecutive k rows form a 1024-byte swizzle atom (stride byte offset 1024),
// and the next 64 M elements start `mn_block_bytes` further on (leading byte
// offset).  An MMA k-step of 16 k rows starts 2048 bytes after the previous one.
__device__ __forceinline__ uint64_t make_sw128_desc_mn(uint32_t smem_addr, uint32_t mn_block_bytes) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
    d |= (uint64_t)((mn_block_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}

// ---------------------------------------------------------------- single-CTA tcgen05
// TMA load into this CTA's shared memory, completion counted on this CTA's mbarrier.
__device__ __forceinline__ void tma_load_3d(void *smem_dst, const void *tmap, uint64_t *mbar,
                                            int32_t x, int32_t y, int32_t z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];"
        ::"r"(smem_u32(smem_dst)), "l"(tmap), "r"(smem_u32(mbar)), "r"(x), "r"(y), "r"(z)
        : "memory");
}
__device__ __forceinline__ void tma_load_4d(void *smem_dst, const void *tmap, uint64_t *mbar,
                                            int32_t x, int32_t y, int32_t z, int32_t w) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];"
        ::"r"(smem_u32(smem_dst)), "l"(tmap), "r"(smem_u32(mbar)), "r"(x), "r"(y), "r"(z), "r"(w)
        : "memory");
}
__device__ __forceinline__ void tmem_alloc_1(uint32_t *smem_dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(smem_dst)), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish_1() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_1(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// D (+)= A * B^T on this CTA alone (M = 64 or 128).
__device__ __forceinline__ void tc_mma_f16_1(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                 ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}
// Arrives once on this CTA's mbarrier when all tcgen05 ops issued so far by
// this thread complete.
__device__ __forceinline__ void tc_commit_1(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_u32(bar)) : "memory");
}
// ---------------------------------------------------------------- block-scaled FP8 (MX) tcgen05
// Shared-memory descriptor of a 512-byte scale-factor atom for tcgen05.cp: 32
// rows of 16 bytes, no swizzle (K-major, 8-row core groups 128 bytes apart).
__device__ __forceinline__ uint64_t make_sf_atom_desc(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;                 // leading byte offset 16 (one 16-byte column)
    d |= (uint64_t)(128u >> 4) << 32;        // stride byte offset 128
    d |= (uint64_t)1u << 46;                 // version 1; layout 0 = no swizzle
    return d;
}
// 32 TMEM lanes x 128 bits from the atom, the same into each of the four lane
// quadrants (tmem_col .. tmem_col + 3).
__device__ __forceinline__ void tc_cp_sf_atom(uint32_t tmem_col, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(tmem_col), "l"(sdesc) : "memory");
}
// Instruction descriptor of kind::mxf8f6f4 with E4M3 A and B, UE8M0 scale
// factors (scale format bit 23), K-major operands, the scale byte sf_id of the
// TMEM scale words for both A (bits 29-30) and B (bits 4-5).
__host__ __device__ constexpr uint32_t make_idesc_mx_e4m3(int M, int N, uint32_t sf_id) {
    return ((sf_id & 3u) << 4) | ((uint32_t)(N >> 3) << 17) | (1u << 23) | ((uint32_t)(M >> 4) << 24) |
           ((sf_id & 3u) << 29);
}
// D (+)= (A * 2^sfa) * (B * 2^sfb)^T with one UE8M0 scale per row (column) and
// 32 K values, the scales read from TMEM at tsfa / tsfb (top two address bits:
// the scale byte).  Single CTA, M = 128.
__device__ __forceinline__ void tc_mma_mx_1(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t tsfa, uint32_t tsfb,
                                            uint32_t accumulate) {
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
                 ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb)
                 : "memory");
}

// The same across a CTA pair (issued by the leader): each CTA's atom, at the
// same shared-memory offset, into its own TMEM at tmem_col.
__device__ __forceinline__ void tc_cp_sf_atom_pair(uint32_t tmem_col, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(tmem_col), "l"(sdesc) : "memory");
}
// Block-scaled MMA across the CTA pair (M = 256, issued by the leader): each
// CTA's TMEM holds the scales of its own 128 A rows at tsfa and the scales of
// all N B rows at tsfb.
__device__ __forceinline__ void tc_mma_mx_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                               uint32_t idesc, uint32_t tsfa, uint32_t tsfb,
                                               uint32_t accumulate) {
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
                 ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb)
                 : "memory");
}

// Orders this thread's generic-proxy shared-memory writes before later
// async-proxy reads of them (the tensor core's operand fetch, TMA).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 4-byte asynchronous copy global -> shared; src_bytes = 0 writes zeros and reads
// nothing (src must still be a 4-byte aligned address).
__device__ __forceinline__ void cp_async_4(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
                 : "memory");
}

// One arrival on `bar` once every cp.async this thread issued before it has
// landed; the arrival is counted in the barrier's initial count (.noinc).
__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Waits until every cp.async this thread issued has landed.
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

}  // namespace moe
