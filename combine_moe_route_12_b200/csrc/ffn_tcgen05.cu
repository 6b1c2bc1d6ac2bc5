// Step 5 (bf16): grouped SwiGLU expert FFN on the expert-contiguous receive
// rows (LightLLM PR 1687: contiguous "psum" grouped GEMM, silu_and_mul, second
// grouped GEMM; decode reduces w*y straight into a dense output).
//
// Two launches of one persistent, warp-specialised tcgen05 kernel:
//   GEMM1  gate|up = W13[e] . xr^T, epilogue h = silu(gate) * up (bf16)
//   GEMM2  y = W2[e] . h^T (bf16), or in decode form
//          out_reduce[t] += w * y in fp32.
//
// Operands are swapped relative to the row-major product: the weights are the
// 128-row MMA operand (A) and the expert's tokens are the N operand (B), so a
// tile is (expert, 128 output features, up to 128 / 256 tokens) and the
// token count is only rounded up to the MMA's N granularity of 16.  A ragged
// expert segment of M_e rows wastes < 16 rows instead of up to 127.  In
// GEMM1 the gate rows and the up rows of the same 128 features are two MMAs
// into two TMEM accumulators, so TMEM lane i holds gate_i and up_i of every
// token and the SwiGLU is lane-local.
//
// CTA = 6 warps.  Warp 4 (one lane) streams weight and token tiles with TMA
// into a 4-stage ring of 128B-swizzled shared-memory buffers; warp 5 (one
// lane) issues tcgen05.mma (M=128, N=16..256, K=16, bf16 -> fp32) into one of
// two TMEM accumulator buffers, so the epilogue of tile i overlaps the main
// loop of tile i+1; warps 0-3 drain TMEM (warp q owns features 32q..32q+31 of
// the tile) and write h / y one token row at a time (each warp store covers
// 32 consecutive features).  Tiles run expert by expert, feature block by
// feature block, token block innermost, so the CTAs that share a weight slice
// run together and read it from DRAM once.
//
// Every mbarrier wait is bounded (2 s); a timeout raises MOE_DEV_WAIT_TIMEOUT,
// stops the other roles, lets in-flight copies and MMAs land, frees TMEM and
// returns.
#include <cudaTypedefs.h>

#include "moe_common.cuh"

namespace moe {

constexpr int kBK = 64, kStages = 4;
constexpr int kFeat = 128;                           // weight rows (output features) per tile
constexpr int kTokRows = 32;                         // rows per token TMA box
constexpr int kFfnThreads = 192;
constexpr uint32_t kWBytes = kFeat * kBK * 2;        // 16 KiB: one 128-row weight box
constexpr uint32_t kTokBoxBytes = kTokRows * kBK * 2;  // 4 KiB
constexpr uint32_t kStageBytes = 48 * 1024;
constexpr uint32_t kTmemCols = 512;                  // two 256-column accumulator buffers

enum EpiMode : int { kEpiSwiGLU = 0, kEpiStore = 1, kEpiReduce = 2 };

struct FfnGemmParams {
    const int32_t *expert_offsets;
    int E;
    int K;                 // reduction length (H for GEMM1, I for GEMM2)
    int n_fblocks;         // 128-feature blocks per expert (I/128 or H/128, rounded up)
    int w_rows_per_expert; // 2I for GEMM1, H for GEMM2
    int up_offset;         // GEMM1: rows from a gate row to its up row (I)
    int tok_block;         // tokens per tile: 128 (GEMM1) or 256 (GEMM2)
    int out_cols;          // row length of the output (I for h, H for y / out_reduce)
    void *out;             // h or y
    float *out_reduce;
    const int32_t *recv_token;
    const int32_t *recv_slot;
    const float *topk_w;
    int k;
    uint32_t *status;
};

struct FfnSmem {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t tmem_full[2];
    uint64_t tmem_empty[2];
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort_flag;
    int total_tiles;
};

struct TileInfo {
    int e, f_blk, p0, n_valid, n_mma;
};

__device__ __forceinline__ TileInfo decode_tile(int tile, const int32_t *s_tpre, const int32_t *s_tb,
                                                const FfnGemmParams &P) {
    int lo = 0, hi = P.E - 1;  // last e with s_tpre[e] <= tile (it owns >= 1 tile)
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_tpre[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    TileInfo t;
    t.e = lo;
    const int local = tile - s_tpre[lo];
    const int tb = s_tb[lo];
    t.f_blk = local / tb;
    const int t_blk = local - t.f_blk * tb;
    const int off = P.expert_offsets[lo];
    const int m_e = P.expert_offsets[lo + 1] - off;
    t.p0 = off + t_blk * P.tok_block;
    t.n_valid = min(P.tok_block, m_e - t_blk * P.tok_block);
    t.n_mma = (t.n_valid + 15) & ~15;
    return t;
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + __expf(-g)); }

template <int MODE>
__global__ void __launch_bounds__(kFfnThreads, 1) ffn_gemm_tcgen05_kernel(
    const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
    const FfnGemmParams P) {
    constexpr bool kSwiGLU = MODE == kEpiSwiGLU;
    // weight boxes at the start of a stage (gate + up for GEMM1), token rows after
    constexpr uint32_t kTokOff = kSwiGLU ? 2 * kWBytes : kWBytes;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // 1024-byte alignment for the swizzled tiles
    unsigned char *base = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char *tiles = base;
    FfnSmem *S = reinterpret_cast<FfnSmem *>(base + kStages * kStageBytes);
    int32_t *s_tpre = reinterpret_cast<int32_t *>(S + 1);   // [E + 1] tile prefix
    int32_t *s_tb = s_tpre + (P.E + 1);                       // [E] token blocks per expert

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // --- tile table (every CTA builds the same one from the expert offsets)
    if (warp == 0) {
        int run = 0;
        for (int e0 = 0; e0 < P.E; e0 += 32) {
            const int e = e0 + lane;
            int tb = 0;
            if (e < P.E) {
                const int m = P.expert_offsets[e + 1] - P.expert_offsets[e];
                tb = (m + P.tok_block - 1) / P.tok_block;
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
        if (lane == 0) { s_tpre[P.E] = run; S->total_tiles = run; }
    }
    if (threadIdx.x == 32) {
        for (int s = 0; s < kStages; ++s) { mbar_init(&S->full[s], 1); mbar_init(&S->empty[s], 1); }
        for (int a = 0; a < 2; ++a) { mbar_init(&S->tmem_full[a], 1); mbar_init(&S->tmem_empty[a], 4); }
        mbar_init(&S->mma_done, 1);
        S->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 4 && lane == 0) { tma_prefetch_desc(&tmap_w); tma_prefetch_desc(&tmap_x); }
    if (warp == 5) { tmem_alloc(&S->tmem_base, kTmemCols); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const int total = S->total_tiles;
    const uint32_t tmem_base = S->tmem_base;
    const int num_k = (P.K + kBK - 1) / kBK;
    volatile int *abort_flag = &S->abort_flag;

    if (warp == 4) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                const TileInfo ti = decode_tile(tile, s_tpre, s_tb, P);
                const int w_row = ti.e * P.w_rows_per_expert + ti.f_blk * kFeat;
                const int n_box = (ti.n_mma + kTokRows - 1) / kTokRows;
                const uint32_t bytes = (kSwiGLU ? 2 : 1) * kWBytes + n_box * kTokBoxBytes;
                for (int kb = 0; kb < num_k; ++kb) {
                    if (!mbar_wait_bounded(&S->empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
                    unsigned char *st = tiles + stage * kStageBytes;
                    const int kx = kb * kBK;
                    mbar_arrive_expect_tx(&S->full[stage], bytes);
                    tma_load_2d(st, &tmap_w, &S->full[stage], kx, w_row);
                    if (kSwiGLU) tma_load_2d(st + kWBytes, &tmap_w, &S->full[stage], kx, w_row + P.up_offset);
                    for (int b = 0; b < n_box; ++b)
                        tma_load_2d(st + kTokOff + b * kTokBoxBytes, &tmap_x, &S->full[stage], kx,
                                    ti.p0 + b * kTokRows);
                    ++issued;
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                }
            }
            if (!ok) {
                raise_status(P.status, MOE_DEV_WAIT_TIMEOUT);
                *abort_flag = 1;
            }
            // let the last copies land before the CTA can exit
            volatile int never = 0;
            const long long last = issued < kStages ? issued : kStages;
            int st = stage;
            uint32_t ph = phase;
            for (long long i = 0; i < last; ++i) {
                if (--st < 0) { st = kStages - 1; ph ^= 1u; }
                mbar_wait_bounded(&S->full[st], ph, &never);
            }
        }
    } else if (warp == 5) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                const TileInfo ti = decode_tile(tile, s_tpre, s_tb, P);
                const uint32_t idesc = make_idesc_bf16_f32(kFeat, ti.n_mma);
                if (!mbar_wait_bounded(&S->tmem_empty[acc], acc_phase ^ 1u, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d0 = tmem_base + (uint32_t)(acc * 256);
                for (int kb = 0; kb < num_k; ++kb) {
                    if (!mbar_wait_bounded(&S->full[stage], phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t st = smem_u32(tiles + stage * kStageBytes);
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        const uint32_t acc_in = (kb > 0 || kk > 0) ? 1u : 0u;
                        const uint64_t xdesc = make_sw128_desc(st + kTokOff + kk * 32);
                        tc_mma_f16(d0, make_sw128_desc(st + kk * 32), xdesc, idesc, acc_in);
                        if (kSwiGLU)
                            tc_mma_f16(d0 + 128, make_sw128_desc(st + kWBytes + kk * 32), xdesc, idesc, acc_in);
                    }
                    tc_commit(&S->empty[stage]);   // frees the stage once these MMAs finish
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                tc_commit(&S->tmem_full[acc]);     // accumulator ready for the epilogue
                if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
            }
            if (!ok) {
                raise_status(P.status, MOE_DEV_WAIT_TIMEOUT);
                *abort_flag = 1;
            }
            // every MMA issued so far must finish before TMEM is released
            volatile int never = 0;
            tc_commit(&S->mma_done);
            mbar_wait_bounded(&S->mma_done, 0, &never);
        }
    } else {
        // ------------------------------------------------ epilogue (warps 0-3)
        const int q = warp;  // TMEM lanes 32q .. 32q+31 = features 32q .. 32q+31 of the tile
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
            if (!mbar_wait_bounded(&S->tmem_full[acc], acc_phase, abort_flag)) {
                if (lane == 0) { raise_status(P.status, MOE_DEV_WAIT_TIMEOUT); *abort_flag = 1; }
                break;
            }
            tc_fence_after();
            const TileInfo ti = decode_tile(tile, s_tpre, s_tb, P);
            const int f = ti.f_blk * kFeat + q * 32 + lane;       // this thread's output feature
            const bool f_ok = f < P.out_cols;
            const uint32_t tbase = tmem_base + (uint32_t)(acc * 256) + ((uint32_t)(q * 32) << 16);

            for (int c0 = 0; c0 < ti.n_mma; c0 += 32) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tbase + c0, r);
                if (kSwiGLU) {
                    uint32_t u[32];
                    tmem_ld_32x32b_x32(tbase + 128 + c0, u);
                    tc_wait_ld();
                    __nv_bfloat16 *h = static_cast<__nv_bfloat16 *>(P.out) + (size_t)ti.p0 * P.out_cols + f;
                    const int nc = min(32, ti.n_valid - c0);
                    if (f_ok) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            if (j < nc) {
                                const float hv = silu_f(__uint_as_float(r[j])) * __uint_as_float(u[j]);
                                h[(size_t)(c0 + j) * P.out_cols] = __float2bfloat16_rn(hv);
                            }
                        }
                    }
                } else if (MODE == kEpiStore) {
                    tc_wait_ld();
                    __nv_bfloat16 *y = static_cast<__nv_bfloat16 *>(P.out) + (size_t)ti.p0 * P.out_cols + f;
                    const int nc = min(32, ti.n_valid - c0);
                    if (f_ok) {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (j < nc) y[(size_t)(c0 + j) * P.out_cols] = __float2bfloat16_rn(__uint_as_float(r[j]));
                    }
                } else {  // kEpiReduce: out_reduce[t] += w * y, one token column at a time
                    tc_wait_ld();
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
            if (lane == 0) mbar_arrive(&S->tmem_empty[acc]);
            if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
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

// 2-D bf16 tensor map over a row-major [rows, cols] matrix, box 64 cols x box_rows,
// 128-byte swizzle, zero fill outside the matrix.
static bool make_tmap_bf16(CUtensorMap *m, const void *ptr, uint64_t rows, uint64_t cols,
                           uint32_t box_rows) {
    auto enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {(cuuint32_t)kBK, box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

size_t ffn_tcgen05_smem(int E) {
    return 1024 + (size_t)kStages * kStageBytes + sizeof(FfnSmem) + sizeof(int32_t) * (2 * (size_t)E + 1) + 64;
}

template <int MODE>
static cudaError_t launch_gemm(const CUtensorMap &tw, const CUtensorMap &tx,
                               const FfnGemmParams &P, int grid, cudaStream_t s) {
    const size_t smem = ffn_tcgen05_smem(P.E);
    static size_t configured = 0;   // largest dynamic smem this kernel was opened up to
    if (smem > configured) {
        cudaError_t err = cudaFuncSetAttribute(ffn_gemm_tcgen05_kernel<MODE>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
        configured = smem;
    }
    ffn_gemm_tcgen05_kernel<MODE><<<grid, kFfnThreads, smem, s>>>(tw, tx, P);
    return cudaGetLastError();
}

// Returns cudaErrorNotSupported when the tensor-map encoder is unavailable.
cudaError_t launch_ffn_tcgen05(const moe_config &c, int64_t n_rows, const void *xr,
                               const int32_t *expert_offsets, const void *w13, const void *w2,
                               void *h, void *y, const int32_t *recv_token,
                               const int32_t *recv_slot, const float *topk_w, float *out_reduce,
                               uint32_t *status, cudaStream_t s, int num_sms) {
    if (n_rows <= 0) return cudaSuccess;
    CUtensorMap tw1, tx1, tw2, tx2;
    if (!make_tmap_bf16(&tw1, w13, (uint64_t)c.E * 2 * c.I, (uint64_t)c.H, kFeat) ||
        !make_tmap_bf16(&tx1, xr, (uint64_t)n_rows, (uint64_t)c.H, kTokRows) ||
        !make_tmap_bf16(&tw2, w2, (uint64_t)c.E * c.H, (uint64_t)c.I, kFeat) ||
        !make_tmap_bf16(&tx2, h, (uint64_t)n_rows, (uint64_t)c.I, kTokRows))
        return cudaErrorNotSupported;

    FfnGemmParams P1{};
    P1.expert_offsets = expert_offsets;
    P1.E = c.E;
    P1.K = c.H;
    P1.n_fblocks = (c.I + kFeat - 1) / kFeat;
    P1.w_rows_per_expert = 2 * c.I;
    P1.up_offset = c.I;
    P1.tok_block = 128;
    P1.out_cols = c.I;
    P1.out = h;
    P1.k = c.k;
    P1.status = status;
    // an upper bound on the tiles: sum_e ceil(M_e / tok) <= n_rows / tok + E
    long long g1 = (n_rows / P1.tok_block + c.E) * (long long)P1.n_fblocks;
    int grid1 = (int)(g1 < num_sms ? g1 : num_sms);
    cudaError_t err = launch_gemm<kEpiSwiGLU>(tw1, tx1, P1, grid1, s);
    if (err != cudaSuccess) return err;

    FfnGemmParams P2 = P1;
    P2.K = c.I;
    P2.n_fblocks = (c.H + kFeat - 1) / kFeat;
    P2.w_rows_per_expert = c.H;
    P2.up_offset = 0;
    P2.tok_block = 256;
    P2.out_cols = c.H;
    P2.out = y;
    P2.out_reduce = out_reduce;
    P2.recv_token = recv_token;
    P2.recv_slot = recv_slot;
    P2.topk_w = topk_w;
    long long g2 = (n_rows / P2.tok_block + c.E) * (long long)P2.n_fblocks;
    int grid2 = (int)(g2 < num_sms ? g2 : num_sms);
    if (c.reduce_dense) return launch_gemm<kEpiReduce>(tw2, tx2, P2, grid2, s);
    return launch_gemm<kEpiStore>(tw2, tx2, P2, grid2, s);
}

}  // namespace moe
