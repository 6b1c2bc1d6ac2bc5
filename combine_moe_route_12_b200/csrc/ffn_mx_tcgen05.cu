// Step 5 in FP8 with K-blocked UE8M0 scales (LightLLM PR 1687: the FP8 grouped
// GEMM over the psum layout with UE8M0 scales packed four to an int32, and
// silu_and_mul followed by the quantisation of h).  Every operand row carries
// one UE8M0 scale per 32 K values: x's receive rows, h's rows, and each weight
// row of W13 and W2; four consecutive block scales of a row read as an int32
// (block 4i in the low byte) are one 128-value k-chunk's scales.
//
// Two launches of one persistent, warp-specialised kernel on CTA pairs
// (clusters of 2) with the block-scaled tensor-core MMA across the pair
// (tcgen05.mma cta_group::2 kind::mxf8f6f4.block_scale, M = 256 weight rows,
// N <= 224 tokens, K = 32 per instruction, fp32 in TMEM):
//   GEMM1  gate|up = W13[e] . xr^T; epilogue h = silu(gate) * up rounded to
//          bf16, then quantised by 32-feature blocks: E4M3 codes h_q [n, I]
//          and scales h_sf [n, I/32] (no bf16 h is stored);
//   GEMM2  y = W2[e] . h_q^T (bf16), or in decode form out_reduce += w * y.
//
// Why pairs: with one CTA per 128 x 128 tile every SM streams 256 operand bytes
// per 128-value k-step for 128 x 128 products, and FP8's doubled MMA rate made
// that stream (through L2, where each token block is re-read for every weight
// block and each weight block for every token block) the bound.  A pair tile
// (256 weight rows, up to 224 tokens) keeps 128 weight rows and half the
// tokens in each CTA, so each SM streams half the bytes per product.
//
// A pair tile is (expert, 256 weight rows, <= 224 tokens); 224, not 256,
// because TMEM holds two accumulators (epilogue of tile i beside the main loop
// of tile i+1) and the scales: accumulators at columns 0 and 256, the scales
// of alternate ring stages at columns 224 and 480 (weight-row scales of the
// stage's two k-chunks in 8 columns, then token scales in 16).  In GEMM1 a
// CTA's 128 weight rows are the gate rows of 64 features and their 64 up rows
// (TMEM lanes i and 64 + i); in GEMM2 128 output features.
//
// Roles (11 warps per CTA).  Warp 8 (one lane) of each CTA streams its ring
// stages (two k-chunks: 32 KiB of weight rows and up to 28 KiB of token rows by
// TMA - a 112-row token box, or 64 or 32 rows for tiles of at most 128 or 64
// tokens - counted on the leader's barrier).  Warp 10 gathers, with all its lanes, the
// scale words of the same stages into a separate, deeper ring of 3 KiB slots:
// 4-byte cp.async copies into 512-byte scale atoms (row r's word at byte
// 16 (r % 32) + 4 (r / 32), the layout tcgen05.cp spreads over the four TMEM
// lane quadrants) - its CTA's own 128 weight rows, and all the tile's tokens,
// which both CTAs hold in TMEM.  A scale slot is free again as soon as its atoms
// are in TMEM, so the gather runs several stages ahead of the operands and its
// latency (scattered words, and the hop below) stays off the stage's refill
// chain.  The leader's gather lanes signal the leader's scale barrier; the
// follower's signal a local one that the follower's warp 9 (otherwise idle)
// forwards to the leader's.  The leader's warp 10 also deals the tiles (a global
// counter, one ticket ahead) and publishes them to every role of both CTAs
// through the pair's slice queue.  The leader's warp 9 (one lane) copies both
// CTAs' atoms to TMEM (tcgen05.cp cta_group::2), frees the scale slot, issues
// the stage's eight block-scaled MMAs and commits to both CTAs' barriers.
// Warps 0-7 of each CTA drain TMEM (warps q and q + 4 share lane quadrant q and
// take alternate 32-token chunks); in GEMM1 the gate and up warps swap half
// their tokens through shared memory, and each warp then quantises its 32
// features (one 32-value block of h) for 16 tokens with a warp max per token.
//
// Every wait is bounded (2 s); a timeout raises MOE_DEV_WAIT_TIMEOUT, stops the
// other roles, lets in-flight copies and MMAs land, frees TMEM and returns.  No
// TMA load uses cluster multicast.
#include <cudaTypedefs.h>
#include <cuda_fp8.h>

#include "ffn_pair.cuh"

namespace moe {

constexpr int kMxRows = 128;                                  // weight rows per CTA (MMA M / 2)
constexpr int kMxTileTok = 224;                               // tokens per tile (MMA N <= 224)
constexpr int kMxBoxTok = kMxTileTok / 2;                     // token rows per CTA box
constexpr int kMxSmallBox = 32;                               // token box of tiles with N <= 64
constexpr int kMxMidBox = 64;                                 // token box of tiles with N <= 128
constexpr int kMxKS = 2;                                      // 128-value k-chunks per ring stage
constexpr uint32_t kMxWChunk = kMxRows * 128;                 // 16 KiB of weight rows per k-chunk
constexpr uint32_t kMxTChunk = kMxBoxTok * 128;               // 14 KiB of token rows per k-chunk
constexpr uint32_t kMxAtom = 512;                             // 128 rows x 4 block scales
// operand stage: [W c0 | W c1 | T c0 | T c1]
constexpr uint32_t kMxTOff = kMxKS * kMxWChunk;
constexpr uint32_t kMxStageBytes = kMxTOff + kMxKS * kMxTChunk;   // 60 KiB
constexpr int kMxStages = 3;
constexpr uint32_t kMxRingBytes = kMxStages * kMxStageBytes;
static_assert(kMxStageBytes % 1024 == 0 && kMxTOff % 1024 == 0 && kMxTChunk % 1024 == 0,
              "swizzled tiles need 1024-byte alignment");
// scale slot of one stage: [SFA c0 | SFA c1 | SFB c0 a0 | c0 a1 | c1 a0 | c1 a1]
constexpr int kMxSfAtoms = 3 * kMxKS;                         // per stage: one weight atom and two token atoms per k-chunk
constexpr uint32_t kMxSfSlotBytes = kMxSfAtoms * kMxAtom;
constexpr uint32_t kMxSfCols = 4 * kMxSfAtoms;                 // TMEM columns of one scale slot
constexpr int kMxSfStages = 6;
constexpr uint32_t kMxSfRingBytes = kMxSfStages * kMxSfSlotBytes;
constexpr int kMxEpiWarps = 8;
constexpr int kMxProdWarp = kMxEpiWarps, kMxMmaWarp = kMxEpiWarps + 1, kMxSfWarp = kMxEpiWarps + 2;
constexpr int kMxThreads = 32 * (kMxEpiWarps + 3);
constexpr uint32_t kMxTmemCols = 512;
constexpr uint32_t kMxAccStride = 256;                        // accumulator a at column 256 a
constexpr uint32_t kMxSfCol = kMxTileTok;                    // scale slot a at kMxSfCol + 256 a
static_assert(kMxAccStride + kMxTileTok + kMxSfCols <= kMxTmemCols, "scale columns exceed TMEM");
constexpr uint32_t kMxXchgBytes = 16 * 1024;                  // GEMM1 gate / up exchange
constexpr int kMxMaxExperts = 512;

enum MxMode : int { kMxSwiGLUQuant = 0, kMxStore = 1, kMxReduce = 2 };

struct MxParams {
    const int32_t *expert_offsets;
    int E;
    int K;                  // H (GEMM1) or I (GEMM2)
    int n_fblocks;          // pair feature blocks per expert: I/128 (GEMM1) or ceil(H/256) (GEMM2)
    int feat_per_cta;       // output features per CTA of a pair tile: 64 (GEMM1) or 128 (GEMM2)
    int w_rows_per_expert;  // 2I or H
    int out_cols;           // I (h) or H (y)
    const uint32_t *w_sf;   // [E * w_rows_per_expert, K/128] scale words
    const uint32_t *t_sf;   // [n_rows, K/128] scale words of the token rows
    uint8_t *h_q;           // GEMM1: [n_rows, I] codes
    uint8_t *h_sf;          // GEMM1: [n_rows, I/32] scale bytes
    __nv_bfloat16 *y;       // GEMM2: [n_rows, H]
    float *out_reduce;      // GEMM2 decode form: [T, H]
    const int32_t *recv_token;
    const int32_t *recv_slot;
    const float *topk_w;
    int k;
    uint32_t *status;
};

struct MxSmem {
    uint64_t full[kMxStages];        // leader: the TMA bytes of both CTAs
    uint64_t empty[kMxStages];       // the stage's MMAs are done (both CTAs)
    uint64_t sf_full[kMxSfStages];   // leader: its 32 gather lanes and the follower's forward;
                                     // follower: its 32 gather lanes
    uint64_t sf_empty[kMxSfStages];  // the slot's atoms are in TMEM (both CTAs)
    uint64_t tmem_full[2];
    uint64_t tmem_empty[2];
    uint64_t mma_done;
    uint64_t q_full[kQueue];
    uint64_t q_empty[kQueue];
    int q_slice[kQueue];
    uint32_t tmem_base;
    int pair_slice[4];
    int go_flag[4];
    int abort_flag;
    int total_slices;
};

struct MxTile {
    int e, f_blk, p0, n_valid, n_mma;   // n_valid <= 224 tokens; n_mma: the MMA's N (rounded to 16)
};

// Rows of the token box a CTA loads for a tile of n_mma tokens (it reads n_mma / 2).
__device__ __forceinline__ int mx_token_box(int n_mma) {
    return n_mma / 2 <= kMxSmallBox ? kMxSmallBox : n_mma / 2 <= kMxMidBox ? kMxMidBox : kMxBoxTok;
}

__device__ __forceinline__ MxTile mx_tile_info(int e, int f_blk, int t_blk, const MxParams &P) {
    MxTile t;
    t.e = e;
    t.f_blk = f_blk;
    const int off = P.expert_offsets[e];
    t.p0 = off + t_blk * kMxTileTok;
    t.n_valid = min(kMxTileTok, P.expert_offsets[e + 1] - t.p0);
    t.n_mma = (t.n_valid + 15) & ~15;
    return t;
}

// The block exponent of a 32-value block whose largest magnitude has the float
// bits b (b >= 0 as a float): the smallest e in [-126, 127] with
// amax <= 448 * 2^e; 0 for a zero (or NaN) block, 127 for an infinite one.
// With amax = 1.m * 2^(x - 127) (x the biased exponent) and 448 = 1.75 * 2^8:
// e = x - 135 when 1.m <= 1.75 (m <= 0x600000), else x - 134.
__device__ __forceinline__ int mx_exponent_bits(uint32_t b) {
    if (b == 0u || b > 0x7F800000u) return 0;
    if (b == 0x7F800000u) return 127;
    const int x = (int)(b >> 23);
    const int e = x == 0 ? -126 : x - 135 + ((b & 0x7FFFFFu) > 0x600000u ? 1 : 0);
    return min(127, max(-126, e));
}

// 2^-e as a float for e in [-126, 127] (e = 127: the subnormal 2^-127).
__device__ __forceinline__ float mx_pow2_neg(int e) {
    return e == 127 ? __uint_as_float(0x00400000u) : __uint_as_float((uint32_t)(127 - e) << 23);
}

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kMxThreads, 1) ffn_mx_tcgen05_kernel(
    const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_t,
    const __grid_constant__ CUtensorMap tmap_tm, const __grid_constant__ CUtensorMap tmap_ts,
    const MxParams P, uint32_t *__restrict__ work_counter) {
    constexpr bool kG1 = MODE == kMxSwiGLUQuant;
    // queue consumers per entry: the leader's MMA thread and operand producer, the
    // follower's operand producer, scale gatherer and forwarder, and every epilogue
    // warp of both CTAs (GEMM1: the gate warps); the leader's scale warp publishes
    constexpr uint32_t kQueueConsumers = 5 + 2 * (kG1 ? kMxEpiWarps / 2 : kMxEpiWarps);
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // 1024-byte alignment for the swizzled tiles (same offsets in both CTAs of the pair)
    unsigned char *base = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char *ring = base;                                       // [stages][W | T]
    unsigned char *sf_ring = base + kMxRingBytes;                     // [scale stages][6 atoms]
    float *xchg = reinterpret_cast<float *>(sf_ring + kMxSfRingBytes);   // GEMM1 only
    MxSmem *S = reinterpret_cast<MxSmem *>(sf_ring + kMxSfRingBytes + (kG1 ? kMxXchgBytes : 0));
    int32_t *s_tpre = reinterpret_cast<int32_t *>(S + 1);            // [E + 1] tile prefix
    int32_t *s_tb = s_tpre + (P.E + 1);                               // [E] token blocks per expert

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();                          // 0: leader (issues the MMA)

    if (warp == 0) {
        int run = 0;
        for (int e0 = 0; e0 < P.E; e0 += 32) {
            const int e = e0 + lane;
            int tb = 0;
            if (e < P.E) {
                tb = (P.expert_offsets[e + 1] - P.expert_offsets[e] + kMxTileTok - 1) / kMxTileTok;
                s_tb[e] = tb;
            }
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
        for (int s = 0; s < kMxStages; ++s) {
            mbar_init(&S->full[s], 1);
            mbar_init(&S->empty[s], 1);
        }
        for (int s = 0; s < kMxSfStages; ++s) {
            mbar_init(&S->sf_full[s], rank == 0 ? 32 + 1 : 32);
            mbar_init(&S->sf_empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&S->tmem_full[a], 1);
            mbar_init(&S->tmem_empty[a], 2 * kMxEpiWarps);   // every epilogue warp of both CTAs
        }
        for (int i = 0; i < kQueue; ++i) { mbar_init(&S->q_full[i], 1); mbar_init(&S->q_empty[i], kQueueConsumers); }
        mbar_init(&S->mma_done, 1);
        S->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kMxProdWarp && lane == 0) {
        tma_prefetch_desc(&tmap_w);
        tma_prefetch_desc(&tmap_t);
        tma_prefetch_desc(&tmap_tm);
        tma_prefetch_desc(&tmap_ts);
    }
    if (warp == kMxMmaWarp) { tmem_alloc_pair(&S->tmem_base, kMxTmemCols); tmem_relinquish_pair(); }
    tc_fence_before();
    cluster_sync_all();      // barriers of both CTAs initialised, TMEM allocated
    tc_fence_after();

    const int total = S->total_slices;
    const uint32_t tmem_base = S->tmem_base;
    const int kwords = P.K / 128;                             // scale words per row
    const int num_k = (P.K + 128 * kMxKS - 1) / (128 * kMxKS);   // ring stages per tile (a last
                                                              // chunk past K loads zeros, scale words 0)
    volatile int *abort_flag = &S->abort_flag;

    if (warp == kMxProdWarp) {
        // ------------------------------------------------ TMA producer (one lane, both CTAs)
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            bool ok = true;
            SliceReader reader;
            int slice;
            while (ok) {
                if (!reader.next(S, abort_flag, true, slice)) { ok = false; break; }
                if (slice < 0) break;
                int se, sfb, t_blk;
                decode_tile(slice, s_tpre, s_tb, P.E, se, sfb, t_blk);
                const MxTile ti = mx_tile_info(se, sfb, t_blk, P);
                // this CTA's weight rows and its half of the tile's tokens
                const int f0 = (sfb * 2 + (int)rank) * P.feat_per_cta;
                const int tok_row = ti.p0 + (int)rank * (ti.n_mma / 2);
                // the smallest token box that holds this CTA's n_mma / 2 rows: fewer bytes
                // through L2 for the same stage slot
                const int box = mx_token_box(ti.n_mma);
                const CUtensorMap *tmap_tok = box == kMxSmallBox ? &tmap_ts : box == kMxMidBox ? &tmap_tm : &tmap_t;
                const uint32_t stage_tx = kMxKS * (kMxWChunk + (uint32_t)box * 128);
                for (int kb = 0; kb < num_k; ++kb) {
                    if (!mbar_wait_bounded(&S->empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
                    unsigned char *st = ring + stage * kMxStageBytes;
                    const int ch = kb * kMxKS;   // first k-chunk of the stage
                    const uint32_t full_leader = mapa_shared(smem_u32(&S->full[stage]), 0);
                    if (rank == 0) mbar_arrive_expect_tx(&S->full[stage], 2 * stage_tx);
                    if (kG1)
                        tma_load_4d_pair(st, &tmap_w, full_leader, 0, f0, 2 * se, ch);
                    else
                        tma_load_3d_pair(st, &tmap_w, full_leader, 0, se * P.w_rows_per_expert + f0, ch);
                    tma_load_3d_pair(st + kMxTOff, tmap_tok, full_leader, 0, tok_row, ch);
                    ++issued;
                    if (++stage == kMxStages) { stage = 0; phase ^= 1u; }
                }
            }
            if (!ok) {
                raise_status(P.status, MOE_DEV_WAIT_TIMEOUT);
                *abort_flag = 1;
            }
            // the leader's full barriers count both CTAs' bytes: let the last copies land
            if (rank == 0) {
                volatile int never = 0;
                const long long last = issued < kMxStages ? issued : kMxStages;
                int st = stage;
                uint32_t ph = phase;
                for (long long i = 0; i < last; ++i) {
                    if (--st < 0) { st = kMxStages - 1; ph ^= 1u; }
                    mbar_wait_bounded(&S->full[st], ph, &never);
                }
            }
        }
        __syncwarp();
    } else if (warp == kMxSfWarp) {
        // ------------------------------------------------ scale gather (whole warp, both CTAs);
        // the leader's also deals the tiles
        int sstage = 0;
        uint32_t sphase = 0;
        bool ok = true;
        int qi = 0;
        uint32_t qph = 0;
        SliceReader reader;
        // the leader holds one ticket ahead: the counter's round trip for the
        // next tile overlaps the gathers of the current one
        int ticket = (rank == 0 && lane == 0) ? (int)atomicAdd(work_counter, 1u) : 0;
        while (ok) {
            int slice = 0;
            bool got = true;
            if (lane == 0) {
                if (rank != 0) {
                    got = reader.next(S, abort_flag, true, slice);
                } else if ((got = mbar_wait_bounded(&S->q_empty[qi], qph ^ 1u, abort_flag))) {
                    slice = ticket < total ? ticket : -1;
                    S->q_slice[qi] = slice;
                    st_cluster_u32(mapa_shared(smem_u32(&S->q_slice[qi]), 1), (uint32_t)slice);
                    mbar_arrive(&S->q_full[qi]);
                    mbar_arrive_cluster_release(mapa_shared(smem_u32(&S->q_full[qi]), 1));
                    if (++qi == kQueue) { qi = 0; qph ^= 1u; }
                    if (slice >= 0) ticket = (int)atomicAdd(work_counter, 1u);
                }
            }
            if (!__shfl_sync(0xffffffffu, got ? 1 : 0, 0)) { ok = false; break; }
            slice = __shfl_sync(0xffffffffu, slice, 0);
            if (slice < 0) break;
            int se, sfb, t_blk;
            decode_tile(slice, s_tpre, s_tb, P.E, se, sfb, t_blk);
            const MxTile ti = mx_tile_info(se, sfb, t_blk, P);
            const int f0 = (sfb * 2 + (int)rank) * P.feat_per_cta;
            // the scale rows this lane gathers: weight rows r = lane + 32 i (-1: past
            // the expert's features) and the tile's tokens n = lane + 32 i (-1: past n_valid)
            int64_t wrow[4], trow[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = lane + 32 * i;
                const int64_t eb = (int64_t)se * P.w_rows_per_expert;
                if (kG1) {   // gate rows of 64 features, then their up rows
                    const int f = f0 + (r & 63);
                    wrow[i] = f < P.out_cols ? eb + (r < 64 ? 0 : P.out_cols) + f : -1;
                } else {
                    const int f = f0 + r;
                    wrow[i] = f < P.out_cols ? eb + f : -1;
                }
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int n = lane + 32 * i;
                trow[i] = n < ti.n_valid ? (int64_t)ti.p0 + n : -1;
            }
            for (int kb = 0; kb < num_k; ++kb) {
                const bool w_ok = lane == 0 ? mbar_wait_bounded(&S->sf_empty[sstage], sphase ^ 1u, abort_flag) : true;
                if (!__shfl_sync(0xffffffffu, w_ok ? 1 : 0, 0)) { ok = false; break; }
                const int ch = kb * kMxKS;
                // weight rows of chunk c at atom c, tokens 128 a .. 128 a + 127 of chunk c
                // at atom 2 + 2c + a; words past K or of rows past the tile are zeros
                const uint32_t sfs = smem_u32(sf_ring + sstage * kMxSfSlotBytes) + 16 * lane;
#pragma unroll
                for (int c = 0; c < kMxKS; ++c) {
                    const bool in_k = ch + c < kwords;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const bool ok_w = in_k && wrow[i] >= 0;
                        cp_async_4(sfs + c * kMxAtom + 4 * i, ok_w ? P.w_sf + wrow[i] * kwords + ch + c : P.w_sf,
                                   ok_w ? 4u : 0u);
                    }
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const bool ok_t = in_k && trow[i] >= 0;
                        cp_async_4(sfs + (kMxKS + 2 * c + (i >> 2)) * kMxAtom + 4 * (i & 3),
                                   ok_t ? P.t_sf + trow[i] * kwords + ch + c : P.t_sf, ok_t ? 4u : 0u);
                    }
                }
                cp_async_mbar_arrive_noinc(&S->sf_full[sstage]);
                if (++sstage == kMxSfStages) { sstage = 0; sphase ^= 1u; }
            }
        }
        if (!ok && lane == 0) {
            raise_status(P.status, MOE_DEV_WAIT_TIMEOUT);
            *abort_flag = 1;
        }
        cp_async_wait_all();   // this lane's scale copies have landed
        __syncwarp();
    } else if (warp == kMxMmaWarp) {
        if (lane == 0) {
            if (rank == 0) {
                // ------------------------------------------------ scale copies + MMA issuer (leader)
                int stage = 0, sstage = 0;
                uint32_t phase = 0, sphase = 0;
                int acc = 0;
                uint32_t acc_phase = 0;
                uint32_t slot = 0;     // TMEM scale columns alternate between two slots, stage by stage
                bool ok = true;
                SliceReader reader;
                int slice;
                while (ok) {
                    if (!reader.next(S, abort_flag, true, slice)) { ok = false; break; }
                    if (slice < 0) break;
                    int se, sfb, t_blk;
                    decode_tile(slice, s_tpre, s_tb, P.E, se, sfb, t_blk);
                    const MxTile ti = mx_tile_info(se, sfb, t_blk, P);
                    if (!mbar_wait_bounded(&S->tmem_empty[acc], acc_phase ^ 1u, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t d = tmem_base + (uint32_t)acc * kMxAccStride;
                    // k-chunk stride inside the stage's token box (32, 64 or 112 rows)
                    const uint32_t tchunk = (uint32_t)mx_token_box(ti.n_mma) * 128;
                    for (int kb = 0; kb < num_k; ++kb) {
                        // the stage's scales: both CTAs' atoms into TMEM, then the slot is free
                        if (!mbar_wait_bounded(&S->sf_full[sstage], sphase, abort_flag)) { ok = false; break; }
                        tc_fence_after();
                        fence_proxy_async_smem();   // the leader's cp.async scale words, before tcgen05.cp
                        const uint32_t sf = smem_u32(sf_ring + sstage * kMxSfSlotBytes);
                        const uint32_t tsf = tmem_base + kMxSfCol + kMxAccStride * slot;
                        // weight-row scales of chunk c at tsf + 4c, token scales at tsf + 8 + 8c
#pragma unroll
                        for (int a = 0; a < kMxSfAtoms; ++a)
                            tc_cp_sf_atom_pair(tsf + 4 * a, make_sf_atom_desc(sf + a * kMxAtom));
                        tc_commit_pair_mc(&S->sf_empty[sstage], 0x3);
                        if (++sstage == kMxSfStages) { sstage = 0; sphase ^= 1u; }
                        // the stage's operands
                        if (!mbar_wait_bounded(&S->full[stage], phase, abort_flag)) { ok = false; break; }
                        tc_fence_after();
                        const uint32_t st = smem_u32(ring + stage * kMxStageBytes);
#pragma unroll
                        for (int c = 0; c < kMxKS; ++c) {
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {   // 32-value K blocks of the chunk
                                const uint64_t wd = make_sw128_desc(st + c * kMxWChunk + kk * 32);
                                const uint64_t td = make_sw128_desc(st + kMxTOff + c * tchunk + kk * 32);
                                const uint32_t sel = (uint32_t)kk << 30;
                                tc_mma_mx_pair(d, wd, td, make_idesc_mx_e4m3(2 * kMxRows, ti.n_mma, kk),
                                               (tsf + 4 * c) | sel, (tsf + 4 * kMxKS + 8 * c) | sel,
                                               (kb > 0 || c > 0 || kk > 0) ? 1u : 0u);
                            }
                        }
                        tc_commit_pair_mc(&S->empty[stage], 0x3);   // frees the stage in both CTAs
                        slot ^= 1u;
                        if (++stage == kMxStages) { stage = 0; phase ^= 1u; }
                    }
                    if (!ok) break;
                    tc_commit_pair_mc(&S->tmem_full[acc], 0x3);    // accumulator ready in both CTAs
                    if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
                }
                if (!ok) {
                    raise_status(P.status, MOE_DEV_WAIT_TIMEOUT);
                    *abort_flag = 1;
                }
                tc_commit_pair_mc(&S->mma_done, 0x3);
            } else {
                // ------------------------------------------------ forwarder (follower)
                // each scale slot of this CTA, once its copies have landed, counted on
                // the leader's scale barrier
                int sstage = 0;
                uint32_t sphase = 0;
                bool ok = true;
                SliceReader reader;
                int slice;
                while (ok) {
                    if (!reader.next(S, abort_flag, true, slice)) { ok = false; break; }
                    if (slice < 0) break;
                    for (int kb = 0; kb < num_k; ++kb) {
                        if (!mbar_wait_bounded(&S->sf_full[sstage], sphase, abort_flag)) { ok = false; break; }
                        fence_proxy_async_smem();   // before the leader's tcgen05.cp reads them
                        mbar_arrive_cluster_release(mapa_shared(smem_u32(&S->sf_full[sstage]), 0));
                        if (++sstage == kMxSfStages) { sstage = 0; sphase ^= 1u; }
                    }
                }
                if (!ok) {
                    raise_status(P.status, MOE_DEV_WAIT_TIMEOUT);
                    *abort_flag = 1;
                }
            }
            // every MMA issued so far must finish before TMEM is released
            volatile int never = 0;
            mbar_wait_bounded(&S->mma_done, 0, &never);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue (warps 0-7 of both CTAs)
        // warp w drains TMEM lanes 32q .. 32q+31 (q = w % 4) for the 32-token
        // chunks of parity w / 4.  GEMM1: quadrants 0-1 hold gate, 2-3 the up rows
        // of the same features; GEMM2: quadrant q holds features 32q .. 32q+31.
        const int q = warp & 3, half = warp >> 2;
        const int feat_lane = kG1 ? (q & 1) * 32 + lane : q * 32 + lane;
        const bool is_gate = q < 2;
        const int xpair = half * 2 + (q & 1);                 // gate/up warp pair (GEMM1)
        const uint32_t empty_leader[2] = {mapa_shared(smem_u32(&S->tmem_empty[0]), 0),
                                          mapa_shared(smem_u32(&S->tmem_empty[1]), 0)};
        int acc = 0;
        uint32_t acc_phase = 0;
        SliceReader reader;
        while (true) {
            int slice = -1;
            if (kG1) {
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
            int se, sfb, t_blk;
            decode_tile(slice, s_tpre, s_tb, P.E, se, sfb, t_blk);
            const MxTile ti = mx_tile_info(se, sfb, t_blk, P);
            const int f = (sfb * 2 + (int)rank) * P.feat_per_cta + feat_lane;   // output feature
            const bool f_ok = f < P.out_cols;
            bool go;
            if (kG1) {
                if (is_gate) {
                    go = mbar_wait_bounded(&S->tmem_full[acc], acc_phase, abort_flag);
                    if (lane == 0) S->go_flag[xpair] = go ? 1 : 0;
                }
                named_barrier_sync(1 + xpair, 64);
                if (!is_gate) go = *reinterpret_cast<volatile int *>(&S->go_flag[xpair]) != 0;
            } else {
                go = mbar_wait_bounded(&S->tmem_full[acc], acc_phase, abort_flag);
            }
            if (!go) {
                if (lane == 0) { raise_status(P.status, MOE_DEV_WAIT_TIMEOUT); *abort_flag = 1; }
                break;
            }
            tc_fence_after();
            const uint32_t tbase = tmem_base + (uint32_t)acc * kMxAccStride + ((uint32_t)(q * 32) << 16);
            for (int c0 = half * 32; c0 < ti.n_mma; c0 += 64) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tbase + c0, r);
                tc_wait_ld_regs(r);
                if (kG1) {
                    // exchange: gate warps hand over tokens 16..31, up warps tokens 0..15
                    float *mine = xchg + (xpair * 2 + (is_gate ? 0 : 1)) * 512;
                    float *theirs = xchg + (xpair * 2 + (is_gate ? 1 : 0)) * 512;
#pragma unroll
                    for (int j = 0; j < 16; ++j) mine[j * 32 + lane] = __uint_as_float(r[is_gate ? 16 + j : j]);
                    named_barrier_sync(1 + xpair, 64);
                    float other[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) other[j] = theirs[j * 32 + lane];
                    named_barrier_sync(1 + xpair, 64);   // both read before the next chunk's writes
                    const int cbase = c0 + (is_gate ? 0 : 16);
                    const int nc = min(16, ti.n_valid - cbase);
                    // h of 16 tokens for this lane's feature, rounded to bf16; the warp's
                    // 32 features are one 32-value block of h: per token, the block's
                    // exponent from the warp's largest magnitude, then the E4M3 codes
                    float hv[16];
                    uint32_t amax[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float own = __uint_as_float(r[is_gate ? j : 16 + j]);
                        const float g = is_gate ? own : other[j], u = is_gate ? other[j] : own;
                        hv[j] = __bfloat162float(__float2bfloat16_rn(silu_f(g) * u));
                        amax[j] = __reduce_max_sync(0xffffffffu, f_ok ? __float_as_uint(fabsf(hv[j])) : 0u);
                    }
                    const size_t row0 = (size_t)(ti.p0 + cbase);
                    uint8_t *hq = P.h_q + row0 * P.out_cols + f;
                    uint8_t *hs = P.h_sf + row0 * (P.out_cols / 32) + (f - lane) / 32;
                    const bool blk_ok = f - lane < P.out_cols;
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int e = mx_exponent_bits(amax[j]);
                        const uint8_t code =
                            (uint8_t)__nv_cvt_float_to_fp8(hv[j] * mx_pow2_neg(e), __NV_SATFINITE, __NV_E4M3);
                        if (j < nc) {
                            if (f_ok) hq[(size_t)j * P.out_cols] = code;
                            if (lane == 0 && blk_ok) hs[(size_t)j * (P.out_cols / 32)] = (uint8_t)(e + 127);
                        }
                    }
                } else if (MODE == kMxStore) {
                    // one 64-byte warp store per token row, down a running row pointer
                    __nv_bfloat16 *y = P.y + (size_t)(ti.p0 + c0) * P.out_cols + f;
                    const int nc = f_ok ? min(32, ti.n_valid - c0) : 0;
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        if (j < nc) *y = __float2bfloat16_rn(__uint_as_float(r[j]));
                        y += P.out_cols;
                    }
                } else {   // kMxReduce: out_reduce[t] += w * y, one token column at a time
                    int my_t = 0;
                    float my_w = 0.0f;
                    const int nc = min(32, ti.n_valid - c0);
                    if (lane < nc) {
                        const int p = ti.p0 + c0 + lane;
                        my_t = P.recv_token[p];
                        my_w = P.topk_w[(size_t)my_t * P.k + P.recv_slot[p]];
                    }
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int t = __shfl_sync(0xffffffffu, my_t, j);
                        const float w = __shfl_sync(0xffffffffu, my_w, j);
                        if (j < nc && f_ok)
                            atomicAdd(P.out_reduce + (size_t)t * P.out_cols + f, w * __uint_as_float(r[j]));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(empty_leader[acc]);   // release the pair's accumulator
            if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        }
    }

    tc_fence_before();
    cluster_sync_all();      // both CTAs done: no MMA, copy or remote arrive in flight
    if (warp == kMxMmaWarp) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, kMxTmemCols);
    }
}

// ------------------------------------------------------------------ host side

static PFN_cuTensorMapEncodeTiled_v12000 mx_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// E4M3 rows [rows][K] as (128, rows, K / 128): boxes of box_rows rows and two k-chunks.
static bool mx_tmap_rows(CUtensorMap *m, const void *ptr, uint64_t rows, uint64_t K, uint32_t box_rows) {
    auto enc = mx_encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {128, rows, K / 128};
    const cuuint64_t strides[2] = {K, 128};
    const cuuint32_t box[3] = {128, box_rows, (cuuint32_t)kMxKS};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// W13 codes [E][2][I][H] as (128, I, 2E, H / 128): one box is 64 gate rows of a
// feature block and the 64 matching up rows, two k-chunks deep.
static bool mx_tmap_w13(CUtensorMap *m, const void *ptr, uint64_t E, uint64_t I, uint64_t H) {
    auto enc = mx_encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[4] = {128, I, 2 * E, H / 128};
    const cuuint64_t strides[3] = {H, I * H, 128};
    const cuuint32_t box[4] = {128, (cuuint32_t)kMxRows / 2, 2, (cuuint32_t)kMxKS};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t ffn_mx_smem(int E, bool g1) {
    return 1024 + (size_t)kMxRingBytes + kMxSfRingBytes + (g1 ? kMxXchgBytes : 0) + sizeof(MxSmem) +
           sizeof(int32_t) * (2 * (size_t)E + 1) + 64;
}

template <int MODE>
static cudaError_t launch_mx(const CUtensorMap &tw, const CUtensorMap &tt, const CUtensorMap &ttm,
                             const CUtensorMap &tts, const MxParams &P, int grid, uint32_t *counter,
                             cudaStream_t s) {
    const size_t smem = ffn_mx_smem(P.E, MODE == kMxSwiGLUQuant);
    static SmemOptIn opt_in;   // one per kernel instantiation
    cudaError_t err = opt_in.ensure(ffn_mx_tcgen05_kernel<MODE>, smem);
    if (err != cudaSuccess) return err;
    ffn_mx_tcgen05_kernel<MODE><<<grid, kMxThreads, smem, s>>>(tw, tt, ttm, tts, P, counter);
    return cudaGetLastError();
}

// CTA pairs: an upper bound on the pair tiles is (n_rows / 224 + E) * n_fblocks
static int mx_grid(const moe_config &c, int64_t n_rows, const MxParams &P, int num_sms) {
    const long long max_pairs = num_sms / 2;
    const long long g = (n_rows / kMxTileTok + c.E) * (long long)P.n_fblocks;
    return 2 * (int)(g < max_pairs ? g : max_pairs);
}

// The block-scaled FP8 FFN: GEMM1 (SwiGLU, h quantised by 32-value blocks) then
// GEMM2.  Scale arrays are bytes, one per row and 32 K values (read as words of
// four).  counters: two work counters.  Returns cudaErrorNotSupported when the
// tensor-map encoder is unavailable or E exceeds the tile table's room.
cudaError_t launch_ffn_mx(const moe_config &c, int64_t n_rows, const uint8_t *xr_q, const uint8_t *xr_sf,
                          const int32_t *expert_offsets, const uint8_t *w13_q, const uint8_t *w13_sf,
                          const uint8_t *w2_q, const uint8_t *w2_sf, uint8_t *h_q, uint8_t *h_sf, void *y,
                          const int32_t *recv_token, const int32_t *recv_slot, const float *topk_w,
                          float *out_reduce, uint32_t *status, uint32_t *counters, cudaStream_t s,
                          int num_sms) {
    if (n_rows <= 0) return cudaSuccess;
    if (c.E > kMxMaxExperts) return cudaErrorNotSupported;
    cudaError_t cerr = cudaMemsetAsync(counters, 0, 2 * sizeof(uint32_t), s);
    if (cerr != cudaSuccess) return cerr;
    const uint64_t n = (uint64_t)n_rows;
    CUtensorMap tw1, tx, txm, txs, tw2, th, thm, ths;
    if (!mx_tmap_w13(&tw1, w13_q, c.E, c.I, c.H) || !mx_tmap_rows(&tx, xr_q, n, c.H, kMxBoxTok) ||
        !mx_tmap_rows(&txs, xr_q, n, c.H, kMxSmallBox) || !mx_tmap_rows(&txm, xr_q, n, c.H, kMxMidBox) ||
        !mx_tmap_rows(&thm, h_q, n, c.I, kMxMidBox) ||
        !mx_tmap_rows(&tw2, w2_q, (uint64_t)c.E * c.H, c.I, kMxRows) ||
        !mx_tmap_rows(&th, h_q, n, c.I, kMxBoxTok) || !mx_tmap_rows(&ths, h_q, n, c.I, kMxSmallBox))
        return cudaErrorNotSupported;
    MxParams P{};
    P.expert_offsets = expert_offsets;
    P.E = c.E;
    P.k = c.k;
    P.status = status;
    P.recv_token = recv_token;
    P.recv_slot = recv_slot;
    P.topk_w = topk_w;
    // GEMM1: each CTA's 128 rows are the gate and up rows of 64 features
    MxParams P1 = P;
    P1.K = c.H;
    P1.feat_per_cta = kMxRows / 2;
    P1.n_fblocks = c.I / (2 * P1.feat_per_cta);   // I is a multiple of 128
    P1.w_rows_per_expert = 2 * c.I;
    P1.out_cols = c.I;
    P1.w_sf = reinterpret_cast<const uint32_t *>(w13_sf);
    P1.t_sf = reinterpret_cast<const uint32_t *>(xr_sf);
    P1.h_q = h_q;
    P1.h_sf = h_sf;
    cudaError_t err = launch_mx<kMxSwiGLUQuant>(tw1, tx, txm, txs, P1, mx_grid(c, n_rows, P1, num_sms), counters, s);
    if (err != cudaSuccess) return err;
    MxParams P2 = P;
    P2.K = c.I;
    P2.feat_per_cta = kMxRows;
    P2.n_fblocks = (c.H + 2 * kMxRows - 1) / (2 * kMxRows);
    P2.w_rows_per_expert = c.H;
    P2.out_cols = c.H;
    P2.w_sf = reinterpret_cast<const uint32_t *>(w2_sf);
    P2.t_sf = reinterpret_cast<const uint32_t *>(h_sf);
    P2.y = static_cast<__nv_bfloat16 *>(y);
    P2.out_reduce = out_reduce;
    const int grid2 = mx_grid(c, n_rows, P2, num_sms);
    if (c.reduce_dense) return launch_mx<kMxReduce>(tw2, th, thm, ths, P2, grid2, counters + 1, s);
    return launch_mx<kMxStore>(tw2, th, thm, ths, P2, grid2, counters + 1, s);
}

}  // namespace moe
