// Step 5 (bf16): grouped SwiGLU expert FFN on the expert-contiguous receive
// rows (LightLLM PR 1687: contiguous "psum" grouped GEMM, silu_and_mul, second
// grouped GEMM; decode reduces w*y straight into a dense output).
//
// Two launches of one persistent, warp-specialised tcgen05 kernel:
//   GEMM1  [M_e, H] x W13[e]^T -> gate | up, epilogue h = silu(gate) * up (bf16)
//   GEMM2  [M_e, I] x W2[e]^T  -> y (bf16), or in decode form
//          out_reduce[t] += w * y in fp32 (vector red.add).
//
// CTA = 6 warps.  Warp 4 (one lane) streams A and B tiles with TMA into a
// 4-stage ring of 128B-swizzled shared-memory buffers; warp 5 (one lane)
// issues tcgen05.mma (M=128, N=256, K=16, bf16 -> fp32) into one of two TMEM
// accumulators (2 x 256 columns), so the epilogue of tile i overlaps the
// main loop of tile i+1; warps 0-3 drain TMEM (warp q owns rows 32q..32q+31)
// and write the outputs.  Tiles are (expert, n block, m block), m innermost
// so the CTAs working on one weight slice run together and share it in L2.
// The M dimension follows the device-side expert offsets: a tile's rows
// past its expert are computed and discarded, never stored.
//
// Every mbarrier wait is bounded (2 s); a timeout raises MOE_DEV_WAIT_TIMEOUT,
// stops the other roles, lets in-flight copies and MMAs land, frees TMEM and
// returns.
#include <cudaTypedefs.h>

#include "moe_common.cuh"

namespace moe {

constexpr int kBM = 128, kBN = 256, kBK = 64, kStages = 4;
constexpr int kFfnThreads = 192;
constexpr uint32_t kABytes = kBM * kBK * 2;          // 16 KiB
constexpr uint32_t kBHalfBytes = 128 * kBK * 2;      // 16 KiB
constexpr uint32_t kBBytes = kBN * kBK * 2;          // 32 KiB
constexpr uint32_t kStageBytes = kABytes + kBBytes;  // 48 KiB
constexpr uint32_t kTmemCols = 2 * kBN;              // two fp32 accumulators

enum EpiMode : int { kEpiSwiGLU = 0, kEpiStore = 1, kEpiReduce = 2 };

struct FfnGemmParams {
    const int32_t *expert_offsets;
    int E;
    int K;                 // reduction length (H for GEMM1, I for GEMM2)
    int n_blocks;          // N tiles per expert
    int b_rows_per_expert; // rows of one expert's B matrix (2I or H)
    int b_block_stride;    // B rows per N tile (128 gate rows, or 256 output rows)
    int b_second;          // offset of the second 128-row B box (I: the up half, or 128)
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

__device__ __forceinline__ void decode_tile(int tile, const int32_t *s_tpre, const int32_t *s_mb,
                                            int E, int n_blocks, int &e, int &m_blk, int &n_blk) {
    int lo = 0, hi = E - 1;  // last e with s_tpre[e] <= tile
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_tpre[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    e = lo;
    const int local = tile - s_tpre[e];
    const int mb = s_mb[e];
    n_blk = local / mb;
    m_blk = local - n_blk * mb;
}

__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi) {
    const __nv_bfloat16 l = __float2bfloat16_rn(lo), h = __float2bfloat16_rn(hi);
    return (uint32_t)__bfloat16_as_ushort(l) | ((uint32_t)__bfloat16_as_ushort(h) << 16);
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + __expf(-g)); }

template <int MODE>
__global__ void __launch_bounds__(kFfnThreads, 1) ffn_gemm_tcgen05_kernel(
    const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
    const FfnGemmParams P) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // 1024-byte alignment for the swizzled tiles
    unsigned char *base = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char *tiles = base;
    FfnSmem *S = reinterpret_cast<FfnSmem *>(base + kStages * kStageBytes);
    int32_t *s_tpre = reinterpret_cast<int32_t *>(S + 1);   // [E + 1] tile prefix
    int32_t *s_mb = s_tpre + (P.E + 1);                       // [E] m blocks per expert

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // --- tile table (every CTA builds the same one from the expert offsets)
    if (warp == 0) {
        int run = 0;
        for (int e0 = 0; e0 < P.E; e0 += 32) {
            const int e = e0 + lane;
            int mb = 0;
            if (e < P.E) {
                const int m = P.expert_offsets[e + 1] - P.expert_offsets[e];
                mb = (m + kBM - 1) / kBM;
                s_mb[e] = mb;
            }
            const int t = mb * P.n_blocks;
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
    if (warp == 4 && lane == 0) { tma_prefetch_desc(&tmap_a); tma_prefetch_desc(&tmap_b); }
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
                int e, m_blk, n_blk;
                decode_tile(tile, s_tpre, s_mb, P.E, P.n_blocks, e, m_blk, n_blk);
                const int a_row = P.expert_offsets[e] + m_blk * kBM;
                const int b_row0 = e * P.b_rows_per_expert + n_blk * P.b_block_stride;
                const int b_row1 = b_row0 + P.b_second;
                for (int kb = 0; kb < num_k; ++kb) {
                    if (!mbar_wait_bounded(&S->empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
                    unsigned char *sa = tiles + stage * kStageBytes;
                    unsigned char *sb = sa + kABytes;
                    mbar_arrive_expect_tx(&S->full[stage], kStageBytes);
                    tma_load_2d(sa, &tmap_a, &S->full[stage], kb * kBK, a_row);
                    tma_load_2d(sb, &tmap_b, &S->full[stage], kb * kBK, b_row0);
                    tma_load_2d(sb + kBHalfBytes, &tmap_b, &S->full[stage], kb * kBK, b_row1);
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
            const uint32_t idesc = make_idesc_bf16_f32(kBM, kBN);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                if (!mbar_wait_bounded(&S->tmem_empty[acc], acc_phase ^ 1u, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * kBN);
                for (int kb = 0; kb < num_k; ++kb) {
                    if (!mbar_wait_bounded(&S->full[stage], phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(tiles + stage * kStageBytes);
                    const uint32_t b_addr = a_addr + kABytes;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        tc_mma_f16(d_tmem, make_sw128_desc(a_addr + kk * 32),
                                   make_sw128_desc(b_addr + kk * 32), idesc,
                                   (kb > 0 || kk > 0) ? 1u : 0u);
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
        const int q = warp;  // TMEM lanes 32q .. 32q+31
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
            if (!mbar_wait_bounded(&S->tmem_full[acc], acc_phase, abort_flag)) {
                if (lane == 0) { raise_status(P.status, MOE_DEV_WAIT_TIMEOUT); *abort_flag = 1; }
                break;
            }
            tc_fence_after();
            int e, m_blk, n_blk;
            decode_tile(tile, s_tpre, s_mb, P.E, P.n_blocks, e, m_blk, n_blk);
            const int off_e = P.expert_offsets[e];
            const int m_e = P.expert_offsets[e + 1] - off_e;
            const int row = m_blk * kBM + q * 32 + lane;
            const bool valid = row < m_e;
            const long long p = (long long)off_e + row;
            const uint32_t tbase = tmem_base + (uint32_t)(acc * kBN) + ((uint32_t)(q * 32) << 16);

            if (MODE == kEpiSwiGLU) {
                __nv_bfloat16 *h = static_cast<__nv_bfloat16 *>(P.out);
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t g[32], u[32];
                    tmem_ld_32x32b_x32(tbase + c * 32, g);
                    tmem_ld_32x32b_x32(tbase + 128 + c * 32, u);
                    tc_wait_ld();
                    const int col = n_blk * 128 + c * 32;
                    if (valid && col < P.out_cols) {
                        uint4 *dst = reinterpret_cast<uint4 *>(h + p * P.out_cols + col);
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            float hv[8];
#pragma unroll
                            for (int z = 0; z < 8; ++z)
                                hv[z] = silu_f(__uint_as_float(g[8 * v + z])) * __uint_as_float(u[8 * v + z]);
                            uint4 o;
                            o.x = pack2_bf16(hv[0], hv[1]);
                            o.y = pack2_bf16(hv[2], hv[3]);
                            o.z = pack2_bf16(hv[4], hv[5]);
                            o.w = pack2_bf16(hv[6], hv[7]);
                            dst[v] = o;
                        }
                    }
                }
            } else if (MODE == kEpiStore) {
                __nv_bfloat16 *y = static_cast<__nv_bfloat16 *>(P.out);
#pragma unroll 1
                for (int c = 0; c < 8; ++c) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(tbase + c * 32, r);
                    tc_wait_ld();
                    const int col = n_blk * kBN + c * 32;
                    if (valid && col < P.out_cols) {
                        uint4 *dst = reinterpret_cast<uint4 *>(y + p * P.out_cols + col);
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            uint4 o;
                            o.x = pack2_bf16(__uint_as_float(r[8 * v + 0]), __uint_as_float(r[8 * v + 1]));
                            o.y = pack2_bf16(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3]));
                            o.z = pack2_bf16(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5]));
                            o.w = pack2_bf16(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7]));
                            dst[v] = o;
                        }
                    }
                }
            } else {  // kEpiReduce
                int t = 0;
                float w = 0.0f;
                if (valid) {
                    t = P.recv_token[p];
                    w = P.topk_w[(size_t)t * P.k + P.recv_slot[p]];
                }
#pragma unroll 1
                for (int c = 0; c < 8; ++c) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(tbase + c * 32, r);
                    tc_wait_ld();
                    const int col = n_blk * kBN + c * 32;
                    if (valid && col < P.out_cols) {
                        float4 *dst = reinterpret_cast<float4 *>(P.out_reduce + (size_t)t * P.out_cols + col);
#pragma unroll
                        for (int v = 0; v < 8; ++v) {
                            const float4 a = make_float4(w * __uint_as_float(r[4 * v + 0]),
                                                         w * __uint_as_float(r[4 * v + 1]),
                                                         w * __uint_as_float(r[4 * v + 2]),
                                                         w * __uint_as_float(r[4 * v + 3]));
                            atomicAdd(dst + v, a);
                        }
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

// 2-D bf16 tensor map over a row-major [rows, cols] matrix, box 64 cols x 128 rows,
// 128-byte swizzle, zero fill outside the matrix.
static bool make_tmap_bf16(CUtensorMap *m, const void *ptr, uint64_t rows, uint64_t cols) {
    auto enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {(cuuint32_t)kBK, 128u};
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
static cudaError_t launch_gemm(const CUtensorMap &ta, const CUtensorMap &tb,
                               const FfnGemmParams &P, int grid, cudaStream_t s) {
    const size_t smem = ffn_tcgen05_smem(P.E);
    cudaError_t err = cudaFuncSetAttribute(ffn_gemm_tcgen05_kernel<MODE>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    ffn_gemm_tcgen05_kernel<MODE><<<grid, kFfnThreads, smem, s>>>(ta, tb, P);
    return cudaGetLastError();
}

// Returns cudaErrorNotSupported when the tensor-map encoder is unavailable.
cudaError_t launch_ffn_tcgen05(const moe_config &c, int64_t n_rows, const void *xr,
                               const int32_t *expert_offsets, const void *w13, const void *w2,
                               void *h, void *y, const int32_t *recv_token,
                               const int32_t *recv_slot, const float *topk_w, float *out_reduce,
                               uint32_t *status, cudaStream_t s, int num_sms) {
    if (n_rows <= 0) return cudaSuccess;
    CUtensorMap ta1, tb1, ta2, tb2;
    if (!make_tmap_bf16(&ta1, xr, (uint64_t)n_rows, (uint64_t)c.H) ||
        !make_tmap_bf16(&tb1, w13, (uint64_t)c.E * 2 * c.I, (uint64_t)c.H) ||
        !make_tmap_bf16(&ta2, h, (uint64_t)n_rows, (uint64_t)c.I) ||
        !make_tmap_bf16(&tb2, w2, (uint64_t)c.E * c.H, (uint64_t)c.I))
        return cudaErrorNotSupported;
    // an upper bound on the tiles: sum_e ceil(M_e / 128) <= n_rows / 128 + E
    const long long mblk_bound = n_rows / kBM + c.E;

    FfnGemmParams P1{};
    P1.expert_offsets = expert_offsets;
    P1.E = c.E;
    P1.K = c.H;
    P1.n_blocks = (c.I + 127) / 128;
    P1.b_rows_per_expert = 2 * c.I;
    P1.b_block_stride = 128;
    P1.b_second = c.I;
    P1.out_cols = c.I;
    P1.out = h;
    P1.k = c.k;
    P1.status = status;
    long long g1 = mblk_bound * P1.n_blocks;
    int grid1 = (int)(g1 < num_sms ? g1 : num_sms);
    cudaError_t err = launch_gemm<kEpiSwiGLU>(ta1, tb1, P1, grid1, s);
    if (err != cudaSuccess) return err;

    FfnGemmParams P2 = P1;
    P2.K = c.I;
    P2.n_blocks = (c.H + kBN - 1) / kBN;
    P2.b_rows_per_expert = c.H;
    P2.b_block_stride = kBN;
    P2.b_second = 128;
    P2.out_cols = c.H;
    P2.out = y;
    P2.out_reduce = out_reduce;
    P2.recv_token = recv_token;
    P2.recv_slot = recv_slot;
    P2.topk_w = topk_w;
    long long g2 = mblk_bound * P2.n_blocks;
    int grid2 = (int)(g2 < num_sms ? g2 : num_sms);
    if (c.reduce_dense) return launch_gemm<kEpiReduce>(ta2, tb2, P2, grid2, s);
    return launch_gemm<kEpiStore>(ta2, tb2, P2, grid2, s);
}

}  // namespace moe
