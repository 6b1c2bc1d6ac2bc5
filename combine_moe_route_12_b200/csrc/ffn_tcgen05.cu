// Step 5 (bf16): grouped SwiGLU expert FFN on the expert-contiguous receive
// rows (LightLLM PR 1687: contiguous "psum" grouped GEMM, silu_and_mul, second
// grouped GEMM; decode reduces w*y straight into a dense output).
//
// Two launches of one persistent, warp-specialised tcgen05 kernel that runs on
// CTA pairs (clusters of 2, cta_group::2 MMA with M = 256):
//   GEMM1  gate|up = W13[e] . xr^T, epilogue h = silu(gate) * up (bf16)
//   GEMM2  y = W2[e] . h^T (bf16), or in decode form
//          out_reduce[t] += w * y in fp32.
//
// Operands are swapped relative to the row-major product: the weights are the
// M operand and the expert's tokens are the N operand, so a pair tile is
// (expert, 256 weight rows, up to 288 tokens) and the token count is only
// rounded up to the MMA's N granularity of 16: a ragged expert segment wastes
// < 16 rows instead of up to 127, and each weight tile meets all of its tile's
// tokens while it sits in shared memory.  The pair's MMA keeps
// 128 weight rows and half the tokens in each CTA's shared memory, which
// halves the operand bytes each SM's shared memory must deliver per MMA;
// with one CTA per MMA the shared memory (tile fills plus operand reads), not
// the tensor pipe, bounds the main loop.
//
// In GEMM1 a CTA's 128 weight rows are the gate rows of 64 features followed
// by the up rows of the same 64 features, so TMEM lanes i and 64+i hold gate_i
// and up_i; the two epilogue warps that own them swap half their columns
// through shared memory and each finishes h for half the tokens.
//
// CTA = 10 warps.  Warp 8 (one lane) of each CTA streams its weight and token
// tiles with TMA into a ring of three 68 KiB stages of 128B-swizzled buffers,
// counting the bytes on the leader CTA's mbarrier.  A stage holds two 64-column
// k-chunks and takes two TMA boxes: the weights (GEMM1: one 4-D box of 64 gate
// rows and the 64 matching up rows) and 144 token rows.  Each TMA issue costs
// the producer on the order of a hundred cycles whatever its size, so few large
// boxes keep it ahead of the tensor pipe (token rows of a box past the tile's N
// are loaded but never read by the MMA).  Warp 9 (one lane) of the leader
// issues the pair's tcgen05.mma (bf16 -> fp32) into one of two TMEM accumulators
// and commits to both CTAs' barriers, so the epilogue of tile i overlaps the main
// loop of tile i+1.  Tiles cover an expert's rows 256 at a time, and its last tile
// takes up to 288.  Each accumulator owns 224 TMEM columns, and the 64 between them
// are two halves of a shared part: a main MMA of more than 224 tokens extends into
// its accumulator's adjacent half, and a tile of more than 256 tokens issues a
// second MMA per k-step (N = 32, the same weights) into the other half, so an
// expert of up to 288 rows streams its weights once.  Each half has its own
// barrier: the epilogue drains the chunks that hold a half first and releases it,
// and the next tile that writes it waits for that.  An expert of more rows takes
// several tiles; the tiles of one weight slice are dealt back to back, so the
// later ones read the slice from L2.  The leader's producer takes tiles from a global counter, one ticket ahead, and publishes
// them to both CTAs through a small mbarrier queue; warps 0-7 of each CTA
// drain its TMEM (warps q and q+4 own lanes 32q..32q+31 and take alternate
// 32-column chunks, each two runs of 16 consecutive receive rows) and write
// h / y one token row at a time.  Tiles run expert
// by expert, weight block by weight block, token block innermost.
//
// Every mbarrier wait is bounded (2 s); a timeout raises MOE_DEV_WAIT_TIMEOUT,
// stops the other roles, lets in-flight copies and MMAs land, frees TMEM and
// returns.  No TMA load uses cluster multicast.
#include <cudaTypedefs.h>

#include "ffn_pair.cuh"

namespace moe {

constexpr int kBK = 64;                              // bf16 columns of one 128-byte swizzled k-chunk
constexpr int kBK8 = 128;                            // E4M3 columns of one 128-byte k-chunk
constexpr int kKS = 2;                               // k-chunks per ring stage (one TMA box each)
constexpr int kRowsPerCta = 128;                     // weight rows (MMA M / 2) per CTA
constexpr int kSlotCols = 224;                       // TMEM columns each accumulator owns outright
constexpr int kXHalf = 32;                           // TMEM columns of each half of the shared part
constexpr int kTileTok = kSlotCols + kXHalf;         // 256: tokens of a tile's main MMA (N <= 256)
constexpr int kTileMax = kTileTok + kXHalf;          // an expert's last tile takes up to 288 tokens
constexpr int kBoxRows = kTileTok / 2 + kXHalf / 2;  // 144 token rows per CTA: main half, then extra half
constexpr int kEpiWarps = 8;                         // two per TMEM lane quadrant
constexpr int kProdWarp = kEpiWarps, kMmaWarp = kEpiWarps + 1;
constexpr int kFfnThreads = 32 * (kEpiWarps + 2);
constexpr uint32_t kWBytes = kRowsPerCta * kBK * 2;         // 16 KiB: a CTA's weight rows of one k-chunk
constexpr uint32_t kTokBytes = kBoxRows * kBK * 2;           // 18 KiB: a CTA's 144 token rows of one k-chunk
constexpr uint32_t kStageBytes = kKS * (kWBytes + kTokBytes);  // 68 KiB
constexpr int kSmallBoxRows = 32;                            // token box of tiles with N <= 64
constexpr int kStages = 3;
constexpr uint32_t kRingBytes = kStages * kStageBytes;       // 204 KiB
// TMEM: accumulator 0 owns [0, 224), half a of the shared part is [224, 256), half b
// [256, 288), accumulator 1 owns [288, 512).  A main MMA of more than 224 tokens
// takes its accumulator's adjacent half (0: [0, 256), 1: [256, 512)); a tile of
// more than 256 tokens puts its extra 32 columns in the other half.
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kXCol = kSlotCols;                // half a; half b follows
constexpr uint32_t kXchgBytes = 16 * 1024;           // GEMM1 gate/up exchange (4 warp pairs x 2 ways x 2 KiB)

// Epilogues: the forward's SwiGLU (h), store (y) and decode reduce; the
// backward's store of the recomputed gate and up values (g | u side by side)
// and its SwiGLU backward (dh in TMEM, g and u read back: h, dg, du).
enum EpiMode : int { kEpiSwiGLU = 0, kEpiStore = 1, kEpiReduce = 2, kEpiStoreGU = 3, kEpiSwiGLUBwd = 4 };

struct FfnGemmParams {
    const int32_t *expert_offsets;
    int E;
    int K;                 // reduction length (H for GEMM1, I for GEMM2)
    int n_fblocks;         // pair feature blocks per expert: I/128 (GEMM1) or H/256 (GEMM2), rounded up
    int feat_per_cta;      // output features per CTA of a pair tile: 64 (GEMM1) or 128 (GEMM2)
    int w_rows_per_expert; // 2I for GEMM1, H for GEMM2
    int out_cols;          // row length of the output (I for h, H for y / out_reduce)
    void *out;             // h or y
    float *out_reduce;
    const int32_t *recv_token;
    const int32_t *recv_slot;
    const float *topk_w;
    int k;
    uint32_t *status;
    // FP8 operands: UE8M0 scale bytes of the weight rows (index e *
    // w_rows_per_expert + row within the expert) and of the token rows
    // (t_scale[recv_token[p]] when t_scale_by_token, else t_scale[p])
    const uint8_t *w_scale;
    const uint8_t *t_scale;
    int t_scale_by_token;
    // row stride of `out` in elements (out_cols for the forward's outputs; 2I for
    // the backward's g | u rows, whose up half starts half_cols further on)
    int out_ld;
    int half_cols;
    // SwiGLU backward: g | u rows [n, 2I] (read) and dg | du rows [n, 2I] (written)
    const __nv_bfloat16 *gu;
    __nv_bfloat16 *out2;
};

struct FfnSmem {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t tmem_full[2];
    uint64_t tmem_empty[2];
    uint64_t x_empty[2];       // a half of the shared part drained (leader CTA): a, b
    uint64_t mma_done;
    uint64_t q_full[kQueue];   // slice queue: published (count 1), per CTA
    uint64_t q_empty[kQueue];  // slice queue: read by every consumer (leader CTA only)
    int q_slice[kQueue];
    uint32_t tmem_base;
    int pair_slice[4];     // GEMM1: slice the gate warp of a warp pair read for its partner
    int go_flag[4];        // GEMM1: per warp pair, did the gate warp's accumulator wait succeed
    int abort_flag;
    int total_slices;      // tiles (the name is kept for the queue's work units)
};

// Token blocks of an expert with m rows: 256-token tiles, the last one taking up to
// 288, so an expert of up to 288 rows streams its weights once.
__device__ __forceinline__ int expert_tiles(int m) {
    return m <= 0 ? 0 : m <= kTileMax ? 1 : (m - kXHalf + kTileTok - 1) / kTileTok;
}

// A tile: n_valid <= 288 tokens from receive row p0.  n_main: the main MMA's N (the
// token count rounded to 16, or 256 past 224 tokens); n_x: the extra MMA's N, 32 for
// a tile of more than 256 tokens, else 0.  The pair's token rows: CTA 0 holds main
// columns [0, n_main / 2) then extra columns [0, n_x / 2), CTA 1 the rest of both,
// each in one box of consecutive receive rows: main column j is receive row p0 + j
// (+ n_x / 2 past CTA 0's half), extra column j is p0 + n_main / 2 + j (+ n_main / 2
// past CTA 0's half).
struct TileInfo {
    int e, f_blk, p0, n_valid, n_main, n_x;
};

__device__ __forceinline__ TileInfo tile_info(int e, int f_blk, int t_blk, const FfnGemmParams &P) {
    TileInfo t;
    t.e = e;
    t.f_blk = f_blk;
    const int off = P.expert_offsets[e];
    const int m_e = P.expert_offsets[e + 1] - off;
    t.p0 = off + t_blk * kTileTok;
    t.n_valid = t_blk == expert_tiles(m_e) - 1 ? m_e - t_blk * kTileTok : kTileTok;
    t.n_main = t.n_valid > kSlotCols ? kTileTok : (t.n_valid + 15) & ~15;
    t.n_x = t.n_valid > kTileTok ? kXHalf : 0;
    return t;
}

// TMEM columns of a tile in accumulator acc: its main MMA's first column and its
// extra MMA's; the half a main MMA of more than 224 columns takes is the
// accumulator's own (a for 0, b for 1), the extra MMA's the other one.
__device__ __forceinline__ uint32_t main_col(const TileInfo &ti, int acc) {
    return acc == 0 ? 0u : ti.n_main > kSlotCols ? (uint32_t)kSlotCols + kXHalf : (uint32_t)kSlotCols + 2 * kXHalf;
}
__device__ __forceinline__ uint32_t extra_col(int acc) { return acc == 0 ? kXCol + kXHalf : kXCol; }

// Epilogue chunk ch of a tile (32 TMEM columns): its first TMEM column, the receive
// rows (from p0) of its two 16-column halves, each a run of consecutive rows, and
// the half of the shared part it holds (-1: none).  Chunks that hold a half of the
// shared part come first (the extra MMA's, then the main MMA's own half), so that
// the epilogue can release them before the rest.
struct ChunkMap {
    uint32_t tcol;
    int rel_lo, rel_hi, xh;
};
__device__ __forceinline__ int chunk_count(const TileInfo &ti) { return ti.n_x / 32 + (ti.n_main + 31) / 32; }
__device__ __forceinline__ ChunkMap chunk_map(const TileInfo &ti, int ch, int acc) {
    ChunkMap m;
    const int nxc = ti.n_x / 32;
    if (ch < nxc) {   // the extra MMA: columns [0, 16) from CTA 0, [16, 32) from CTA 1
        m.tcol = extra_col(acc);
        m.rel_lo = ti.n_main / 2;
        m.rel_hi = ti.n_main + 16;
        m.xh = acc ^ 1;
        return m;
    }
    int c = ch - nxc;   // main MMA chunk; accumulator 0's own half is its last chunk (7)
    const bool own = ti.n_main > kSlotCols;
    if (own && acc == 0) c = c == 0 ? kSlotCols / 32 : c - 1;
    const int j = 32 * c;
    m.tcol = main_col(ti, acc) + (uint32_t)j;
    m.rel_lo = j < ti.n_main / 2 ? j : j + ti.n_x / 2;
    m.rel_hi = j + 16 < ti.n_main / 2 ? j + 16 : j + 16 + ti.n_x / 2;
    m.xh = own && ch == nxc ? acc : -1;
    return m;
}
__device__ __forceinline__ int chunk_rel(const ChunkMap &m, int j) { return j < 16 ? m.rel_lo + j : m.rel_hi + j - 16; }

// Tile number -> (expert, feature block, token block); s_tpre[e] is the first
// tile of expert e, which owns tb(e) * n_fblocks tiles.
__device__ __forceinline__ void decode_tile_pre(int tile, const int32_t *s_tpre, int E, int n_fblocks,
                                                int &e, int &f_blk, int &t_blk) {
    int lo = 0, hi = E - 1;  // last e with s_tpre[e] <= tile (it owns >= 1 tile)
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_tpre[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    e = lo;
    const int local = tile - s_tpre[lo];
    const int tb = (s_tpre[lo + 1] - s_tpre[lo]) / n_fblocks;
    f_blk = local / tb;
    t_blk = local - f_blk * tb;
}

// A UE8M0 scale byte as a float: 2^(b - 127) (b = 0 gives the subnormal 2^-127).
__device__ __forceinline__ float ue8m0_value(uint32_t b) {
    return b == 0 ? __uint_as_float(0x00400000u) : __uint_as_float(b << 23);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);   // lo in the low half
    return *reinterpret_cast<const uint32_t *>(&p);
}

// The epilogue holds one feature per lane and T tokens per lane; global rows
// want tokens.  Three butterfly rounds (lane bit 0, 1, 2) swap halves so that,
// for each group g of 8 tokens, lane L ends up with token 8g + (L & 7) and the
// 8 consecutive features 8 (L >> 3) .. +7, rounded to bf16 and packed: one
// 16-byte store per lane and group instead of one 2-byte store per token.
template <int T>
__device__ __forceinline__ void warp_tokens_to_rows(const float (&v)[T], uint4 (&out)[T / 8], int lane) {
    const bool b0 = lane & 1, b1 = (lane >> 1) & 1, b2 = (lane >> 2) & 1;
    uint32_t p1[T / 2];     // features {L & ~1, L | 1} of token a + (L & 1)
#pragma unroll
    for (int a = 0; a < T; a += 2) {
        const float recv = __shfl_xor_sync(0xffffffffu, b0 ? v[a] : v[a + 1], 1);
        p1[a / 2] = b0 ? pack_bf16x2(recv, v[a + 1]) : pack_bf16x2(v[a], recv);
    }
    uint32_t q[T / 4][2];   // features 4 (L >> 2) .. +3 of token 4k + (L & 3)
#pragma unroll
    for (int k = 0; k < T / 4; ++k) {
        const uint32_t recv = __shfl_xor_sync(0xffffffffu, b1 ? p1[2 * k] : p1[2 * k + 1], 2);
        q[k][0] = b1 ? recv : p1[2 * k];
        q[k][1] = b1 ? p1[2 * k + 1] : recv;
    }
#pragma unroll
    for (int g = 0; g < T / 8; ++g) {
        const uint32_t r0 = __shfl_xor_sync(0xffffffffu, b2 ? q[2 * g][0] : q[2 * g + 1][0], 4);
        const uint32_t r1 = __shfl_xor_sync(0xffffffffu, b2 ? q[2 * g][1] : q[2 * g + 1][1], 4);
        out[g].x = b2 ? r0 : q[2 * g][0];
        out[g].y = b2 ? r1 : q[2 * g][1];
        out[g].z = b2 ? q[2 * g + 1][0] : r0;
        out[g].w = b2 ? q[2 * g + 1][1] : r1;
    }
}

// F8: E4M3 operands (tcgen05 kind::f8f6f4, 128 columns per k-chunk) with the
// row scales applied to the fp32 accumulators in the epilogue; else bf16.
// A_MN: the weight operand is read transposed, MN-major (the backward's
// W2^T and W13^T): a ring stage holds its 128 k rows of the CTA's 128 output
// features as two 64-feature blocks of 128-byte rows, one 3-D TMA box.
template <int MODE, bool F8, bool A_MN>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kFfnThreads, 1) ffn_gemm_tcgen05_kernel(
    const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
    const __grid_constant__ CUtensorMap tmap_xs,
    const FfnGemmParams P, uint32_t *__restrict__ work_counter) {
    constexpr bool kSwiGLU = MODE == kEpiSwiGLU;
    // gate and up rows of W13 side by side in a CTA's 128 weight rows
    constexpr bool kGateUp = MODE == kEpiSwiGLU || MODE == kEpiStoreGU;
    static_assert(!(A_MN && (F8 || kGateUp)), "the transposed weight operand is bf16 with plain rows");
    // queue consumers per entry: the MMA thread, the follower's producer, and
    // every epilogue warp of both CTAs (GEMM1: the gate warp of each pair only)
    constexpr uint32_t kQueueConsumers = 2 + 2 * (kSwiGLU ? kEpiWarps / 2 : kEpiWarps);
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // 1024-byte alignment for the swizzled tiles (same offsets in both CTAs of the pair)
    unsigned char *base = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char *tiles = base;                              // [kStages][weights | tokens]
    float *xchg = reinterpret_cast<float *>(base + kRingBytes);   // GEMM1 only
    FfnSmem *S = reinterpret_cast<FfnSmem *>(base + kRingBytes + (kSwiGLU ? kXchgBytes : 0));
    int32_t *s_tpre = reinterpret_cast<int32_t *>(S + 1);   // [E + 1] tile prefix

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();                  // 0: leader (issues the MMA)

    // --- slice table (every CTA builds the same one from the expert offsets)
    if (warp == 0) {
        int run = 0;
        for (int e0 = 0; e0 < P.E; e0 += 32) {
            const int e = e0 + lane;
            int tb = 0;
            if (e < P.E) tb = expert_tiles(P.expert_offsets[e + 1] - P.expert_offsets[e]);
            const int t = tb * P.n_fblocks;
            int incl = t;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int o = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += o;
            }
            if (e < P.E) s_tpre[e] = run + incl - t;
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) { s_tpre[P.E] = run; S->total_slices = run; }
    }
    if (threadIdx.x == 32) {
        for (int s = 0; s < kStages; ++s) { mbar_init(&S->full[s], 1); mbar_init(&S->empty[s], 1); }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&S->tmem_full[a], 1);
            mbar_init(&S->tmem_empty[a], 2 * kEpiWarps);   // every epilogue warp of both CTAs
        }
        mbar_init(&S->x_empty[0], 2 * kEpiWarps);
        mbar_init(&S->x_empty[1], 2 * kEpiWarps);
        for (int i = 0; i < kQueue; ++i) { mbar_init(&S->q_full[i], 1); mbar_init(&S->q_empty[i], kQueueConsumers); }
        mbar_init(&S->mma_done, 1);
        S->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kProdWarp && lane == 0) {
        tma_prefetch_desc(&tmap_w);
        tma_prefetch_desc(&tmap_x);
        tma_prefetch_desc(&tmap_xs);
    }
    if (warp == kMmaWarp) { tmem_alloc_pair(&S->tmem_base, kTmemCols); tmem_relinquish_pair(); }
    tc_fence_before();
    cluster_sync_all();      // barriers of both CTAs initialised, TMEM allocated
    tc_fence_after();

    const int total = S->total_slices;
    const uint32_t tmem_base = S->tmem_base;
    constexpr int kChunkCols = F8 ? kBK8 : kBK;             // columns of a 128-byte k-chunk
    const int num_k = (P.K + kChunkCols * kKS - 1) / (kChunkCols * kKS);   // ring stages per tile
    volatile int *abort_flag = &S->abort_flag;

    if (warp == kProdWarp) {
        // ------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            bool ok = true;
            // leader: takes slices from the global counter and publishes them to
            // every consumer of both CTAs; follower: reads them like a consumer
            int qi = 0;
            uint32_t qph = 0;
            SliceReader reader;
            // the leader holds one ticket ahead: the counter's round trip for the
            // next tile overlaps the loads of the current one
            int ticket = rank == 0 ? (int)atomicAdd(work_counter, 1u) : 0;
            auto next_slice = [&](int &slice) -> bool {
                if (rank != 0) return reader.next(S, abort_flag, true, slice);
                if (!mbar_wait_bounded(&S->q_empty[qi], qph ^ 1u, abort_flag)) return false;
                slice = ticket < total ? ticket : -1;
                S->q_slice[qi] = slice;
                st_cluster_u32(mapa_shared(smem_u32(&S->q_slice[qi]), 1), (uint32_t)slice);
                mbar_arrive(&S->q_full[qi]);
                mbar_arrive_cluster_release(mapa_shared(smem_u32(&S->q_full[qi]), 1));
                if (++qi == kQueue) { qi = 0; qph ^= 1u; }
                if (slice >= 0) ticket = (int)atomicAdd(work_counter, 1u);
                return true;
            };
            int slice;
            while (ok) {
                if (!next_slice(slice)) { ok = false; break; }
                if (slice < 0) break;
                int se, sf, t_blk;
                decode_tile_pre(slice, s_tpre, P.E, P.n_fblocks, se, sf, t_blk);
                // this CTA's weight rows: GEMM1 64 gate rows + the matching 64 up rows
                // (one 4-D box), GEMM2 128 rows; its token rows: half of the tile's N
                const int f_row = (sf * 2 + (int)rank) * P.feat_per_cta;
                const int w_row = se * P.w_rows_per_expert + f_row;
                const TileInfo ti = tile_info(se, sf, t_blk, P);
                const int tok_row = ti.p0 + (int)rank * (ti.n_main / 2 + ti.n_x / 2);
                // a tile of an expert's short last token block takes a 32-row token box:
                // fewer bytes through L2 for the same stage slot
                const bool small_box = ti.n_x == 0 && ti.n_main / 2 <= kSmallBoxRows;
                const uint32_t stage_bytes = small_box ? kKS * (kWBytes + kSmallBoxRows * kBK * 2) : kStageBytes;
                for (int kb = 0; kb < num_k; ++kb) {
                    if (!mbar_wait_bounded(&S->empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
                    unsigned char *st = tiles + stage * kStageBytes;
                    const uint32_t full_leader = mapa_shared(smem_u32(&S->full[stage]), 0);
                    const int ch = kb * kKS;   // first k-chunk of the stage
                    // full boxes land in both CTAs (rows or chunks past the tensor are zero-filled)
                    if (rank == 0) mbar_arrive_expect_tx(&S->full[stage], 2 * stage_bytes);
                    if (kGateUp)
                        tma_load_4d_pair(st, &tmap_w, full_leader, 0, f_row, 2 * se, ch);
                    else if (A_MN)   // k rows of the expert, the CTA's two 64-feature blocks
                        tma_load_3d_pair(st, &tmap_w, full_leader, 0, se * P.K + ch * kBK, f_row / kBK);
                    else
                        tma_load_3d_pair(st, &tmap_w, full_leader, 0, w_row, ch);
                    tma_load_3d_pair(st + kKS * kWBytes, small_box ? &tmap_xs : &tmap_x, full_leader, 0, tok_row, ch);
                    ++issued;
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                }
            }
            if (!ok) {
                raise_status(P.status, MOE_DEV_WAIT_TIMEOUT);
                *abort_flag = 1;
            }
            // the leader's full barriers count both CTAs' bytes: let the last copies land
            if (rank == 0) {
                volatile int never = 0;
                const long long last = issued < kStages ? issued : kStages;
                int st = stage;
                uint32_t ph = phase;
                for (long long i = 0; i < last; ++i) {
                    if (--st < 0) { st = kStages - 1; ph ^= 1u; }
                    mbar_wait_bounded(&S->full[st], ph, &never);
                }
            }
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------ MMA issuer (leader CTA)
        if (lane == 0) {
            if (rank == 0) {
                int stage = 0;
                uint32_t phase = 0;
                int acc = 0;
                uint32_t acc_phase = 0;
                uint32_t x_phase = 0;   // bit h: the phase of half h's barrier
                bool ok = true;
                SliceReader reader;
                int slice;
                while (ok) {
                  if (!reader.next(S, abort_flag, true, slice)) { ok = false; break; }
                  if (slice < 0) break;
                  int se, sf, t_blk;
                  decode_tile_pre(slice, s_tpre, P.E, P.n_fblocks, se, sf, t_blk);
                  {
                    const TileInfo ti = tile_info(se, sf, t_blk, P);
                    const uint32_t idesc = F8 ? make_idesc_e4m3_f32(2 * kRowsPerCta, ti.n_main)
                                              : make_idesc_bf16_f32_major(2 * kRowsPerCta, ti.n_main, A_MN, false);
                    const bool merged = ti.n_x > 0;
                    const uint32_t idesc_x = !merged ? 0u
                                             : F8 ? make_idesc_e4m3_f32(2 * kRowsPerCta, ti.n_x)
                                                  : make_idesc_bf16_f32_major(2 * kRowsPerCta, ti.n_x, A_MN, false);
                    if (!mbar_wait_bounded(&S->tmem_empty[acc], acc_phase ^ 1u, abort_flag)) { ok = false; break; }
                    // the halves of the shared part this tile writes (its own past 224 main
                    // columns, the other one for the extra MMA): drained by the epilogue of
                    // the last tile that wrote them
                    {
                        bool x_ok = true;
                        for (int hx = 0; hx < 2 && x_ok; ++hx) {
                            const bool uses = hx == acc ? ti.n_main > kSlotCols : merged;
                            if (!uses) continue;
                            x_ok = mbar_wait_bounded(&S->x_empty[hx], ((x_phase >> hx) & 1u) ^ 1u, abort_flag);
                            x_phase ^= 1u << hx;
                        }
                        if (!x_ok) { ok = false; break; }
                    }
                    tc_fence_after();
                    const uint32_t d = tmem_base + main_col(ti, acc);
                    const uint32_t dx = tmem_base + extra_col(acc);
                    // k-chunk stride inside the stage's token box (32 or 144 rows); the
                    // extra part's rows follow the main half's in both CTAs
                    const bool small_box = ti.n_x == 0 && ti.n_main / 2 <= kSmallBoxRows;
                    const uint32_t tchunk = small_box ? kSmallBoxRows * kBK * 2 : kTokBytes;
                    const uint32_t x_row_off = (uint32_t)(ti.n_main / 2) * 128;   // 128 rows of 128 bytes
                    for (int kb = 0; kb < num_k; ++kb) {
                        if (!mbar_wait_bounded(&S->full[stage], phase, abort_flag)) { ok = false; break; }
                        tc_fence_after();
                        const uint32_t st = smem_u32(tiles + stage * kStageBytes);
                        // the stage's main MMAs, then its extra-part MMAs: consecutive MMAs
                        // into the same accumulator
#pragma unroll
                        for (int part = 0; part < 2; ++part) {
                            if (part == 1 && !merged) break;
#pragma unroll
                            for (int c = 0; c < kKS; ++c) {
#pragma unroll
                                for (int kk = 0; kk < 4; ++kk) {   // 32-byte k-steps: 16 bf16 or 32 E4M3
                                    // MN-major: k-chunk c is rows 64c.. of each 64-feature block
                                    // (blocks 16 KiB apart), a k-step 16 rows of 128 bytes
                                    const uint64_t wdesc = A_MN
                                        ? make_sw128_desc_mn(st + c * (kWBytes / 2) + kk * 2048, kWBytes)
                                        : make_sw128_desc(st + c * kWBytes + kk * 32);
                                    const uint32_t taddr = st + kKS * kWBytes + c * tchunk + kk * 32 +
                                                           (part ? x_row_off : 0u);
                                    const uint64_t tdesc = make_sw128_desc(taddr);
                                    const uint32_t accum = (kb > 0 || c > 0 || kk > 0) ? 1u : 0u;
                                    if (F8) tc_mma_f8_pair(part ? dx : d, wdesc, tdesc, part ? idesc_x : idesc, accum);
                                    else tc_mma_f16_pair(part ? dx : d, wdesc, tdesc, part ? idesc_x : idesc, accum);
                                }
                            }
                        }
                        tc_commit_pair_mc(&S->empty[stage], 0x3);   // frees the stage in both CTAs
                        if (++stage == kStages) { stage = 0; phase ^= 1u; }
                    }
                    if (!ok) break;
                    tc_commit_pair_mc(&S->tmem_full[acc], 0x3);    // accumulator ready in both CTAs
                    if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
                  }
                }
                if (!ok) {
                    raise_status(P.status, MOE_DEV_WAIT_TIMEOUT);
                    *abort_flag = 1;
                }
                tc_commit_pair_mc(&S->mma_done, 0x3);
            }
            // every MMA issued so far must finish before TMEM is released
            volatile int never = 0;
            mbar_wait_bounded(&S->mma_done, 0, &never);
        }
    } else {
        // ------------------------------------------------ epilogue (warps 0-7 of both CTAs)
        // warp w drains TMEM lanes 32q .. 32q+31 (q = w % 4) for the 32-token
        // chunks of parity w / 4, so two warps share each lane quadrant
        const int q = warp & 3, half = warp >> 2;
        // GEMM1: quadrants 0-1 hold gate, quadrants 2-3 the up rows of the same features;
        // GEMM2: quadrant q holds output features 32q .. 32q+31 of this CTA's 128
        const int feat_lane = kGateUp ? (q & 1) * 32 + lane : q * 32 + lane;
        const bool is_gate = q < 2;
        const int xpair = half * 2 + (q & 1);                 // gate/up warp pair (GEMM1)
        const uint32_t empty_leader[2] = {mapa_shared(smem_u32(&S->tmem_empty[0]), 0),
                                          mapa_shared(smem_u32(&S->tmem_empty[1]), 0)};
        // the leader's barrier of half h of the shared part (the two are adjacent)
        const uint32_t x_empty_leader0 = mapa_shared(smem_u32(&S->x_empty[0]), 0);
        auto x_empty_leader = [&](int h) { return x_empty_leader0 + 8u * (uint32_t)h; };
        int acc = 0;
        uint32_t acc_phase = 0;
        SliceReader reader;
        bool run_on = true;
        while (run_on) {
          int slice = -1;
          if (kSwiGLU) {
              // the gate warp reads the queue and hands the slice to its up partner;
              // both then pass the same exchange barriers or both leave
              if (is_gate) {
                  if (!reader.next(S, abort_flag, lane == 0, slice)) slice = -2;
                  if (lane == 0) S->pair_slice[xpair] = slice;
              }
              named_barrier_sync(1 + xpair, 64);
              if (!is_gate) slice = *reinterpret_cast<volatile int *>(&S->pair_slice[xpair]);
          } else {
              if (!reader.next(S, abort_flag, lane == 0, slice)) slice = -2;
          }
          if (slice == -2) {
              if (lane == 0) { raise_status(P.status, MOE_DEV_WAIT_TIMEOUT); *abort_flag = 1; }
              break;
          }
          if (slice < 0) break;
          int se, sf, t_blk;
          decode_tile_pre(slice, s_tpre, P.E, P.n_fblocks, se, sf, t_blk);
          {
           const TileInfo ti = tile_info(se, sf, t_blk, P);
           const int f = (ti.f_blk * 2 + (int)rank) * P.feat_per_cta + feat_lane;  // output feature
           const bool f_ok = f < P.out_cols;
           // FP8: this lane's weight-row scale, and the token scale of column `lane`
           // of each of the warp's chunks (chunks half, half + 2, ...), loaded before
           // the accumulator wait so that their latency hides behind it
           const int nch = chunk_count(ti);
           float wsc = 1.0f;
           float tsc[5] = {1.0f, 1.0f, 1.0f, 1.0f, 1.0f};
           if (F8) {
               if (f_ok)
                   wsc = ue8m0_value(P.w_scale[(size_t)ti.e * P.w_rows_per_expert +
                                               (kGateUp && !is_gate ? P.out_cols : 0) + f]);
#pragma unroll
               for (int i = 0; i < 5; ++i) {
                   const int ch = half + 2 * i;
                   if (ch < nch) {
                       const int rel = chunk_rel(chunk_map(ti, ch, acc), lane);
                       if (rel < ti.n_valid) {
                           const int p = ti.p0 + rel;
                           tsc[i] = ue8m0_value(P.t_scale[P.t_scale_by_token ? P.recv_token[p] : p]);
                       }
                   }
               }
           }
           do {   // one pass; `break` leaves it on a failed wait
            bool go;
            if (kSwiGLU) {
                // same hand-over for the accumulator wait
                if (is_gate) {
                    go = mbar_wait_bounded(&S->tmem_full[acc], acc_phase, abort_flag);
                    if (lane == 0) S->go_flag[xpair] = go ? 1 : 0;
                }
                named_barrier_sync(1 + xpair, 64);
                if (!is_gate) go = S->go_flag[xpair] != 0;
            } else {
                go = mbar_wait_bounded(&S->tmem_full[acc], acc_phase, abort_flag);
            }
            if (!go) {
                if (lane == 0) { raise_status(P.status, MOE_DEV_WAIT_TIMEOUT); *abort_flag = 1; }
                run_on = false;
                break;
            }
            tc_fence_after();
            const uint32_t tlane = tmem_base + ((uint32_t)(q * 32) << 16);
            // a half of the shared part held by a chunk of the other warp parity is
            // released at once (such chunks are the first one or two of the tile)
            for (int ch = 0; ch < 2 && ch < nch; ++ch) {
                const int xh = chunk_map(ti, ch, acc).xh;
                if (xh >= 0 && (ch & 1) != half) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(x_empty_leader(xh));
                }
            }

            int ci = 0;
            for (int ch = half; ch < nch; ch += 2, ++ci) {
                const ChunkMap cm = chunk_map(ti, ch, acc);
                uint32_t r[32];
                tmem_ld_32x32b_x32(tlane + cm.tcol, r);
                tc_wait_ld_regs(r);
                if (cm.xh >= 0) {   // a half of the shared part is in registers: release it
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(x_empty_leader(cm.xh));
                }
                // FP8: the scale of the token in column `lane`
                const float ts_lane = ci == 0 ? tsc[0] : ci == 1 ? tsc[1] : ci == 2 ? tsc[2] : ci == 3 ? tsc[3] : tsc[4];
                // rows of the two 16-column halves, and how many of each are tokens
                const int nc_lo = min(16, ti.n_valid - cm.rel_lo), nc_hi = min(16, ti.n_valid - cm.rel_hi);
                if (kSwiGLU) {
                    // exchange: gate warps hand over columns 16..31, up warps columns 0..15
                    float *mine = xchg + (xpair * 2 + (is_gate ? 0 : 1)) * 512;
                    float *theirs = xchg + (xpair * 2 + (is_gate ? 1 : 0)) * 512;
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        mine[j * 32 + lane] = __uint_as_float(r[is_gate ? 16 + j : j]) * (F8 ? wsc : 1.0f);
                    named_barrier_sync(1 + xpair, 64);
                    const int cbase = is_gate ? cm.rel_lo : cm.rel_hi;
                    const int nc = is_gate ? nc_lo : nc_hi;
                    // all 16 partner values into registers before the first store:
                    // h and the exchange buffer are both generic pointers, so a load
                    // after a store could not be moved ahead of it and every token
                    // would wait for the previous one's whole chain
                    float other[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) other[j] = theirs[j * 32 + lane];
                    named_barrier_sync(1 + xpair, 64);   // both read before the next chunk's writes
                    // h of this warp's 16 tokens (every lane, for the shuffles; tokens
                    // past nc are never stored)
                    float hv[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float own = __uint_as_float(r[is_gate ? j : 16 + j]) * (F8 ? wsc : 1.0f);
                        float g = is_gate ? own : other[j], u = is_gate ? other[j] : own;
                        if (F8) {
                            const float tj = __shfl_sync(0xffffffffu, ts_lane, (is_gate ? 0 : 16) + j);
                            g *= tj;
                            u *= tj;
                        }
                        hv[j] = silu_f(g) * u;
                    }
                    uint4 o[2];
                    warp_tokens_to_rows<16>(hv, o, lane);
                    const int col = f - feat_lane + (q & 1) * 32 + 8 * (lane >> 3);   // this lane's 8 features
                    if (col + 8 <= P.out_cols) {
                        __nv_bfloat16 *h = static_cast<__nv_bfloat16 *>(P.out) + (size_t)(ti.p0 + cbase) * P.out_cols + col;
#pragma unroll
                        for (int g8 = 0; g8 < 2; ++g8) {
                            const int tok = 8 * g8 + (lane & 7);
                            if (tok < nc) *reinterpret_cast<uint4 *>(h + (size_t)tok * P.out_cols) = o[g8];
                        }
                    }
                } else if (MODE == kEpiStoreGU) {
                    // the gate value of feature f to column f, the up value to column I + f
                    __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(P.out) + (size_t)ti.p0 * P.out_ld +
                                       f + (is_gate ? 0 : P.half_cols);
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (f_ok && (j < 16 ? j < nc_lo : j - 16 < nc_hi))
                            o[(size_t)chunk_rel(cm, j) * P.out_ld] = __float2bfloat16_rn(__uint_as_float(r[j]));
                } else if (MODE == kEpiSwiGLUBwd) {
                    // r = dh of feature f for 32 tokens; with s = sigmoid(g):
                    //   h = g s u,  dg = dh u s (1 + g (1 - s)),  du = dh g s
                    float g[32], u[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        g[j] = 0.0f;
                        u[j] = 0.0f;
                        if (f_ok && (j < 16 ? j < nc_lo : j - 16 < nc_hi)) {
                            const __nv_bfloat16 *gr = P.gu + (size_t)(ti.p0 + chunk_rel(cm, j)) * P.out_ld + f;
                            g[j] = __bfloat162float(gr[0]);
                            u[j] = __bfloat162float(gr[P.half_cols]);
                        }
                    }
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float dh = __uint_as_float(r[j]);
                        const float sg = __fdividef(1.0f, 1.0f + __expf(-g[j]));
                        const float sl = g[j] * sg;
                        if (f_ok && (j < 16 ? j < nc_lo : j - 16 < nc_hi)) {
                            const size_t row = (size_t)(ti.p0 + chunk_rel(cm, j));
                            static_cast<__nv_bfloat16 *>(P.out)[row * P.out_cols + f] = __float2bfloat16_rn(sl * u[j]);
                            __nv_bfloat16 *dgo = P.out2 + row * P.out_ld + f;
                            dgo[0] = __float2bfloat16_rn(dh * u[j] * sg * (1.0f + g[j] * (1.0f - sg)));
                            dgo[P.half_cols] = __float2bfloat16_rn(dh * sl);
                        }
                    }
                } else if (MODE == kEpiStore) {
                    // one 64-byte warp store per token row (the shuffle rearrangement
                    // of the SwiGLU epilogue measured slower here), down a running row
                    // pointer that restarts at the second half's first row
                    __nv_bfloat16 *const out = static_cast<__nv_bfloat16 *>(P.out);
                    if (F8) {
                        // each token's scale from the lane that loaded it, times this
                        // lane's weight-row scale, all taken before the stores
                        float v[32];
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            v[j] = __uint_as_float(r[j]) * (__shfl_sync(0xffffffffu, ts_lane, j) * wsc);
                        const int lo = f_ok ? nc_lo : 0, hi = f_ok ? nc_hi : 0;
                        __nv_bfloat16 *y = out + (size_t)(ti.p0 + cm.rel_lo) * P.out_ld + f;
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            if (j == 16) y = out + (size_t)(ti.p0 + cm.rel_hi) * P.out_ld + f;
                            if (j < 16 ? j < lo : j - 16 < hi) *y = __float2bfloat16_rn(v[j]);
                            y += P.out_ld;
                        }
                    } else {
                        __nv_bfloat16 *y = out + (size_t)(ti.p0 + cm.rel_lo) * P.out_ld + f;
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            if (j == 16) y = out + (size_t)(ti.p0 + cm.rel_hi) * P.out_ld + f;
                            if (f_ok && (j < 16 ? j < nc_lo : j - 16 < nc_hi))
                                *y = __float2bfloat16_rn(__uint_as_float(r[j]));
                            y += P.out_ld;
                        }
                    }
                } else {  // kEpiReduce: out_reduce[t] += w * y, one token column at a time
                    int my_t = 0;
                    float my_w = 0.0f;
                    const bool tok_ok = lane < 16 ? lane < nc_lo : lane - 16 < nc_hi;
                    if (tok_ok) {
                        const int p = ti.p0 + chunk_rel(cm, lane);
                        my_t = P.recv_token[p];
                        my_w = P.topk_w[(size_t)my_t * P.k + P.recv_slot[p]];
                        if (F8) my_w *= ts_lane;
                    }
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int t = __shfl_sync(0xffffffffu, my_t, j);
                        const float w = __shfl_sync(0xffffffffu, my_w, j);
                        if ((j < 16 ? j < nc_lo : j - 16 < nc_hi) && f_ok)
                            atomicAdd(P.out_reduce + (size_t)t * P.out_cols + f,
                                      w * (__uint_as_float(r[j]) * (F8 ? wsc : 1.0f)));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(empty_leader[acc]);   // release the pair's accumulator
            if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
           } while (0);
          }
        }
    }

    tc_fence_before();
    cluster_sync_all();      // both CTAs done: no MMA, copy or remote arrive in flight
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, kTmemCols);
    }
}

// ------------------------------------------------------------------ host side

static PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// A tensor map with 128-byte swizzled boxes whose innermost extent is one
// 128-byte k-chunk (64 bf16 or 128 E4M3 columns); the k-chunk index is the
// outermost dimension, so one box brings kKS consecutive k-chunks of its rows.
static bool make_tmap_kchunks(CUtensorMap *m, const void *ptr, bool f8, int rank,
                              const cuuint64_t *dims, const cuuint64_t *strides,
                              const cuuint32_t *box) {
    auto enc = get_encode_fn();
    if (!enc) return false;
    cuuint32_t estr[5] = {1u, 1u, 1u, 1u, 1u};
    CUresult r = enc(m, f8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank,
                     const_cast<void *>(ptr), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Rows [rows][K] (row stride K elements) as (cc, rows, K / cc), cc the columns
// of a 128-byte k-chunk.
static bool make_tmap_rows(CUtensorMap *m, const void *ptr, uint64_t rows, uint64_t K,
                           uint32_t box_rows, bool f8 = false) {
    const uint64_t cc = f8 ? kBK8 : kBK, es = f8 ? 1 : 2;
    const cuuint64_t dims[3] = {(cuuint64_t)cc, rows, K / cc};
    const cuuint64_t strides[2] = {K * es, (cuuint64_t)cc * es};
    const cuuint32_t box[3] = {(cuuint32_t)cc, box_rows, (cuuint32_t)kKS};
    return make_tmap_kchunks(m, ptr, f8, 3, dims, strides, box);
}

// W13 [E][2][I][H] as (cc, I, 2E, H / cc): one box holds 64 gate rows of a
// feature block followed by the 64 matching up rows, kKS k-chunks deep.
static bool make_tmap_w13(CUtensorMap *m, const void *ptr, uint64_t E, uint64_t I, uint64_t H,
                          bool f8 = false) {
    const uint64_t cc = f8 ? kBK8 : kBK, es = f8 ? 1 : 2;
    const cuuint64_t dims[4] = {(cuuint64_t)cc, I, 2 * E, H / cc};
    const cuuint64_t strides[3] = {H * es, I * H * es, (cuuint64_t)cc * es};
    const cuuint32_t box[4] = {(cuuint32_t)cc, (cuuint32_t)kRowsPerCta / 2, 2u, (cuuint32_t)kKS};
    return make_tmap_kchunks(m, ptr, f8, 4, dims, strides, box);
}

size_t ffn_tcgen05_smem(int E, bool swiglu) {
    return 1024 + (size_t)kRingBytes + (swiglu ? kXchgBytes : 0) + sizeof(FfnSmem) +
           sizeof(int32_t) * ((size_t)E + 1) + 64;
}

template <int MODE, bool F8, bool A_MN = false>
static cudaError_t launch_gemm(const CUtensorMap &tw, const CUtensorMap &tx, const CUtensorMap &txs,
                               const FfnGemmParams &P, int grid, uint32_t *counter, cudaStream_t s) {
    const size_t smem = ffn_tcgen05_smem(P.E, MODE == kEpiSwiGLU);
    static SmemOptIn opt_in;   // one per kernel instantiation
    cudaError_t err = opt_in.ensure(ffn_gemm_tcgen05_kernel<MODE, F8, A_MN>, smem);
    if (err != cudaSuccess) return err;
    ffn_gemm_tcgen05_kernel<MODE, F8, A_MN><<<grid, kFfnThreads, smem, s>>>(tw, tx, txs, P, counter);
    return cudaGetLastError();
}

// The two launches' parameters (GEMM1 then GEMM2) of one grouped FFN.
static void ffn_params(const moe_config &c, const int32_t *expert_offsets, void *h, void *y,
                       const int32_t *recv_token, const int32_t *recv_slot, const float *topk_w,
                       float *out_reduce, uint32_t *status, FfnGemmParams &P1, FfnGemmParams &P2) {
    P1 = FfnGemmParams{};
    P1.expert_offsets = expert_offsets;
    P1.E = c.E;
    P1.K = c.H;
    P1.feat_per_cta = kRowsPerCta / 2;
    P1.n_fblocks = (c.I + 2 * P1.feat_per_cta - 1) / (2 * P1.feat_per_cta);
    P1.w_rows_per_expert = 2 * c.I;
    P1.out_cols = c.I;
    P1.out_ld = c.I;
    P1.out = h;
    P1.k = c.k;
    P1.status = status;
    P1.recv_token = recv_token;
    P2 = P1;
    P2.K = c.I;
    P2.feat_per_cta = kRowsPerCta;
    P2.n_fblocks = (c.H + 2 * P2.feat_per_cta - 1) / (2 * P2.feat_per_cta);
    P2.w_rows_per_expert = c.H;
    P2.out_cols = c.H;
    P2.out_ld = c.H;
    P2.out = y;
    P2.out_reduce = out_reduce;
    P2.recv_slot = recv_slot;
    P2.topk_w = topk_w;
}

// CTA pairs: an upper bound on the pair tiles is (n_rows / 224 + E) * n_fblocks
static int ffn_grid(const moe_config &c, int64_t n_rows, const FfnGemmParams &P, int num_sms) {
    const long long max_pairs = num_sms / 2;
    const long long g = (n_rows / kTileTok + c.E) * (long long)P.n_fblocks;
    return 2 * (int)(g < max_pairs ? g : max_pairs);
}

// Returns cudaErrorNotSupported when the tensor-map encoder is unavailable.
cudaError_t launch_ffn_tcgen05(const moe_config &c, int64_t n_rows, const void *xr,
                               const int32_t *expert_offsets, const void *w13, const void *w2,
                               void *h, void *y, const int32_t *recv_token,
                               const int32_t *recv_slot, const float *topk_w, float *out_reduce,
                               uint32_t *status, uint32_t *counters, cudaStream_t s, int num_sms) {
    if (n_rows <= 0) return cudaSuccess;
    // the two launches' work counters start at zero
    cudaError_t cerr = cudaMemsetAsync(counters, 0, 2 * sizeof(uint32_t), s);
    if (cerr != cudaSuccess) return cerr;
    CUtensorMap tw1, tx1, tw2, tx2, tx1s, tx2s;
    if (!make_tmap_rows(&tx1s, xr, (uint64_t)n_rows, (uint64_t)c.H, kSmallBoxRows) ||
        !make_tmap_rows(&tx2s, h, (uint64_t)n_rows, (uint64_t)c.I, kSmallBoxRows))
        return cudaErrorNotSupported;
    if (!make_tmap_w13(&tw1, w13, (uint64_t)c.E, (uint64_t)c.I, (uint64_t)c.H) ||
        !make_tmap_rows(&tx1, xr, (uint64_t)n_rows, (uint64_t)c.H, kBoxRows) ||
        !make_tmap_rows(&tw2, w2, (uint64_t)c.E * c.H, (uint64_t)c.I, kRowsPerCta) ||
        !make_tmap_rows(&tx2, h, (uint64_t)n_rows, (uint64_t)c.I, kBoxRows))
        return cudaErrorNotSupported;

    FfnGemmParams P1, P2;
    ffn_params(c, expert_offsets, h, y, recv_token, recv_slot, topk_w, out_reduce, status, P1, P2);
    cudaError_t err = launch_gemm<kEpiSwiGLU, false>(tw1, tx1, tx1s, P1, ffn_grid(c, n_rows, P1, num_sms),
                                                     counters, s);
    if (err != cudaSuccess) return err;
    const int grid2 = ffn_grid(c, n_rows, P2, num_sms);
    if (c.reduce_dense) return launch_gemm<kEpiReduce, false>(tw2, tx2, tx2s, P2, grid2, counters + 1, s);
    return launch_gemm<kEpiStore, false>(tw2, tx2, tx2s, P2, grid2, counters + 1, s);
}

// A row-major bf16 [rows, cols] matrix read MN-major: (64, rows, cols / 64),
// boxes of 128 rows of two 64-element blocks (the smem image: block b's row r at
// b * 16 KiB + r * 128 bytes, 128-byte swizzle).  Serves the transposed
// weights of the backward's data-gradient GEMMs (W2^T: rows E*H, cols I; W13^T:
// rows E*2I, cols H) and the token-row operands of its weight gradients.
static bool make_tmap_mn(CUtensorMap *m, const void *ptr, uint64_t rows, uint64_t cols) {
    const cuuint64_t dims[3] = {(cuuint64_t)kBK, rows, cols / kBK};
    const cuuint64_t strides[2] = {cols * 2, (cuuint64_t)kBK * 2};
    const cuuint32_t box[3] = {(cuuint32_t)kBK, 128u, 2u};
    return make_tmap_kchunks(m, ptr, false, 3, dims, strides, box);
}

cudaError_t launch_wgrad_tcgen05(const CUtensorMap &tmap_a, const CUtensorMap &tmap_b,
                                 const int32_t *expert_offsets, int n_seg, long long seg_rows, int E,
                                 int M, int N, float *out, int accumulate, uint32_t *status,
                                 cudaStream_t s, int num_sms);

// Data gradients of the bf16 grouped SwiGLU FFN over one receive buffer (rows
// of expert e: [expert_offsets[e], expert_offsets[e+1])), for incoming dy:
//   1. g | u = W13[e] . xr^T                   (the forward's GEMM1, stored [n, 2I])
//   2. dh = W2[e]^T . dy^T; h = silu(g) u, dg = dh u s (1 + g (1 - s)),
//      du = dh silu(g) with s = sigmoid(g)     (h [n, I], dg | du [n, 2I])
//   3. dxr = W13[e]^T . [dg | du]^T            ([n, H])
// counters: three work counters.
cudaError_t launch_ffn_tcgen05_dgrad(const moe_config &c, int64_t n_rows, const void *xr, const void *dy,
                                     const int32_t *expert_offsets, const void *w13, const void *w2,
                                     void *gu, void *h, void *dgu, void *dxr, uint32_t *status,
                                     uint32_t *counters, cudaStream_t s, int num_sms) {
    if (n_rows <= 0) return cudaSuccess;
    cudaError_t cerr = cudaMemsetAsync(counters, 0, 3 * sizeof(uint32_t), s);
    if (cerr != cudaSuccess) return cerr;
    const uint64_t H = c.H, I = c.I, E = c.E, n = (uint64_t)n_rows;
    CUtensorMap tw13, tx, txs, tw2t, tdy, tdys, tw13t, tdgu, tdgus;
    if (!make_tmap_w13(&tw13, w13, E, I, H) || !make_tmap_rows(&tx, xr, n, H, kBoxRows) ||
        !make_tmap_rows(&txs, xr, n, H, kSmallBoxRows) || !make_tmap_mn(&tw2t, w2, E * H, I) ||
        !make_tmap_rows(&tdy, dy, n, H, kBoxRows) || !make_tmap_rows(&tdys, dy, n, H, kSmallBoxRows) ||
        !make_tmap_mn(&tw13t, w13, E * 2 * I, H) || !make_tmap_rows(&tdgu, dgu, n, 2 * I, kBoxRows) ||
        !make_tmap_rows(&tdgus, dgu, n, 2 * I, kSmallBoxRows))
        return cudaErrorNotSupported;

    FfnGemmParams P1, P2;
    ffn_params(c, expert_offsets, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, status, P1, P2);
    // 1. the forward's GEMM1, g and u stored side by side
    FfnGemmParams Pa = P1;
    Pa.out = gu;
    Pa.out_ld = 2 * c.I;
    Pa.half_cols = c.I;
    cudaError_t err = launch_gemm<kEpiStoreGU, false>(tw13, tx, txs, Pa, ffn_grid(c, n_rows, Pa, num_sms),
                                                      counters, s);
    if (err != cudaSuccess) return err;
    // 2. dh over K = H with W2 read transposed; 128 features of I per CTA
    FfnGemmParams Pb = P2;
    Pb.K = c.H;
    Pb.feat_per_cta = kRowsPerCta;
    Pb.n_fblocks = (c.I + 2 * kRowsPerCta - 1) / (2 * kRowsPerCta);
    Pb.w_rows_per_expert = c.H;
    Pb.out_cols = c.I;
    Pb.out = h;
    Pb.out_ld = 2 * c.I;
    Pb.half_cols = c.I;
    Pb.gu = static_cast<const __nv_bfloat16 *>(gu);
    Pb.out2 = static_cast<__nv_bfloat16 *>(dgu);
    err = launch_gemm<kEpiSwiGLUBwd, false, true>(tw2t, tdy, tdys, Pb, ffn_grid(c, n_rows, Pb, num_sms),
                                                  counters + 1, s);
    if (err != cudaSuccess) return err;
    // 3. dxr over K = 2I with W13 read transposed; 128 features of H per CTA
    FfnGemmParams Pc = P2;
    Pc.K = 2 * c.I;
    Pc.feat_per_cta = kRowsPerCta;
    Pc.n_fblocks = (c.H + 2 * kRowsPerCta - 1) / (2 * kRowsPerCta);
    Pc.w_rows_per_expert = 2 * c.I;
    Pc.out_cols = c.H;
    Pc.out_ld = c.H;
    Pc.out = dxr;
    return launch_gemm<kEpiStore, false, true>(tw13t, tdgu, tdgus, Pc, ffn_grid(c, n_rows, Pc, num_sms),
                                               counters + 2, s);
}

// Weight gradients over n_seg receive buffers laid one after another, seg_rows
// rows apart (segment s: expert offsets expert_offsets + s * (E + 1)), in one
// pass: dW2[e] (+)= dy^T h and dW13[e] (+)= [dg | du]^T xr over the expert's
// rows of every segment (fp32).  xr, dy [n_seg * seg_rows, H], h [.., I],
// dgu [.., 2I].
cudaError_t launch_ffn_tcgen05_wgrad(const moe_config &c, int n_seg, int64_t seg_rows,
                                     const int32_t *expert_offsets, const void *xr, const void *dy,
                                     const void *h, const void *dgu, float *dw13, float *dw2,
                                     int accumulate, uint32_t *status, cudaStream_t s, int num_sms) {
    const uint64_t rows = (uint64_t)n_seg * (uint64_t)seg_rows;
    if (rows == 0) return cudaErrorInvalidValue;
    CUtensorMap a_dy, b_h, a_dgu, b_xr;
    if (!make_tmap_mn(&a_dy, dy, rows, c.H) || !make_tmap_mn(&b_h, h, rows, c.I) ||
        !make_tmap_mn(&a_dgu, dgu, rows, 2 * (uint64_t)c.I) || !make_tmap_mn(&b_xr, xr, rows, c.H))
        return cudaErrorNotSupported;
    cudaError_t err = launch_wgrad_tcgen05(a_dy, b_h, expert_offsets, n_seg, seg_rows, c.E, c.H, c.I, dw2,
                                           accumulate, status, s, num_sms);
    if (err != cudaSuccess) return err;
    return launch_wgrad_tcgen05(a_dgu, b_xr, expert_offsets, n_seg, seg_rows, c.E, 2 * c.I, c.H, dw13,
                                accumulate, status, s, num_sms);
}

// The whole backward of one receive buffer: data gradients, then weight gradients.
cudaError_t launch_ffn_tcgen05_bwd(const moe_config &c, int64_t n_rows, const void *xr, const void *dy,
                                   const int32_t *expert_offsets, const void *w13, const void *w2,
                                   void *gu, void *h, void *dgu, void *dxr, float *dw13, float *dw2,
                                   int accumulate, uint32_t *status, uint32_t *counters,
                                   cudaStream_t s, int num_sms) {
    if (n_rows <= 0) return cudaSuccess;
    cudaError_t err = launch_ffn_tcgen05_dgrad(c, n_rows, xr, dy, expert_offsets, w13, w2, gu, h, dgu, dxr,
                                               status, counters, s, num_sms);
    if (err != cudaSuccess) return err;
    return launch_ffn_tcgen05_wgrad(c, 1, n_rows, expert_offsets, xr, dy, h, dgu, dw13, dw2, accumulate,
                                    status, s, num_sms);
}

cudaError_t launch_quant_rows(int64_t rows, int cols, bool bf16, const void *in, uint8_t *codes,
                              uint8_t *scales, const int32_t *n_dev, cudaStream_t s, int num_sms);

// The FP8 form: GEMM1 on E4M3 codes of xr and W13, h stored in bf16, h
// quantised by rows (its first expert_offsets[E] rows), GEMM2 on the codes of
// h and W2.  Returns cudaErrorNotSupported when the tensor-map encoder is
// unavailable.
cudaError_t launch_ffn_tcgen05_fp8(const moe_config &c, int64_t n_rows, const uint8_t *xr_q,
                                   const uint8_t *x_scale, const int32_t *expert_offsets,
                                   const uint8_t *w13_q, const uint8_t *w13_scale,
                                   const uint8_t *w2_q, const uint8_t *w2_scale, void *h,
                                   uint8_t *h_q, uint8_t *h_scale, void *y,
                                   const int32_t *recv_token, const int32_t *recv_slot,
                                   const float *topk_w, float *out_reduce, uint32_t *status,
                                   uint32_t *counters, cudaStream_t s, int num_sms) {
    if (n_rows <= 0) return cudaSuccess;
    cudaError_t cerr = cudaMemsetAsync(counters, 0, 2 * sizeof(uint32_t), s);
    if (cerr != cudaSuccess) return cerr;
    CUtensorMap tw1, tx1, tw2, tx2, tx1s, tx2s;
    if (!make_tmap_rows(&tx1s, xr_q, (uint64_t)n_rows, (uint64_t)c.H, kSmallBoxRows, true) ||
        !make_tmap_rows(&tx2s, h_q, (uint64_t)n_rows, (uint64_t)c.I, kSmallBoxRows, true) ||
        !make_tmap_w13(&tw1, w13_q, (uint64_t)c.E, (uint64_t)c.I, (uint64_t)c.H, true) ||
        !make_tmap_rows(&tx1, xr_q, (uint64_t)n_rows, (uint64_t)c.H, kBoxRows, true) ||
        !make_tmap_rows(&tw2, w2_q, (uint64_t)c.E * c.H, (uint64_t)c.I, kRowsPerCta, true) ||
        !make_tmap_rows(&tx2, h_q, (uint64_t)n_rows, (uint64_t)c.I, kBoxRows, true))
        return cudaErrorNotSupported;
    FfnGemmParams P1, P2;
    ffn_params(c, expert_offsets, h, y, recv_token, recv_slot, topk_w, out_reduce, status, P1, P2);
    P1.w_scale = w13_scale;
    P1.t_scale = x_scale;
    P1.t_scale_by_token = 1;
    P2.w_scale = w2_scale;
    P2.t_scale = h_scale;
    P2.t_scale_by_token = 0;
    cudaError_t err = launch_gemm<kEpiSwiGLU, true>(tw1, tx1, tx1s, P1, ffn_grid(c, n_rows, P1, num_sms),
                                                    counters, s);
    if (err != cudaSuccess) return err;
    err = launch_quant_rows(n_rows, c.I, true, h, h_q, h_scale, expert_offsets + c.E, s, num_sms);
    if (err != cudaSuccess) return err;
    const int grid2 = ffn_grid(c, n_rows, P2, num_sms);
    if (c.reduce_dense) return launch_gemm<kEpiReduce, true>(tw2, tx2, tx2s, P2, grid2, counters + 1, s);
    return launch_gemm<kEpiStore, true>(tw2, tx2, tx2s, P2, grid2, counters + 1, s);
}

}  // namespace moe
