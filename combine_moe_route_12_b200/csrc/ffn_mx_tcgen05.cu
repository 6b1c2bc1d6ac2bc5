// Step 5 in FP8 with K-blocked UE8M0 scales (LightLLM PR 1687: the FP8 grouped
// GEMM over the psum layout with UE8M0 scales packed four to an int32, and
// silu_and_mul followed by the quantisation of h).  Every operand row carries
// one UE8M0 scale per 32 K values: x's receive rows, h's rows, and each weight
// row of W13 and W2; four consecutive block scales of a row read as an int32
// (block 4i in the low byte) are one 128-value k-chunk's scales.
//
// Two launches of one persistent, warp-specialised single-CTA kernel with the
// block-scaled tensor-core MMA (tcgen05.mma kind::mxf8f6f4.block_scale, M = 128
// weight rows, N <= 128 tokens, K = 32 per instruction, fp32 in TMEM):
//   GEMM1  gate|up = W13[e] . xr^T; epilogue h = silu(gate) * up rounded to
//          bf16, then quantised by 32-feature blocks: E4M3 codes h_q [n, I]
//          and scales h_sf [n, I/32] (no bf16 h is stored);
//   GEMM2  y = W2[e] . h_q^T (bf16), or in decode form out_reduce += w * y.
//
// A tile is (expert, 128 weight rows, 128 tokens): in GEMM1 the gate rows of
// 64 features followed by their 64 up rows (TMEM lanes i and 64 + i), in GEMM2
// 128 output features.  Warp 8 streams each ring stage (two 128-value
// k-chunks: 32 KiB of weight rows and 32 KiB of token rows, one TMA box each)
// and, with all its lanes, gathers the stage's scale words - 128 weight rows
// and 128 token rows, two words each - into four 512-byte scale atoms in shared
// memory (row r's word at byte 16 (r % 32) + 4 (r / 32), the layout tcgen05.cp
// spreads over the four TMEM lane quadrants).  Warp 9 (one lane) copies the
// atoms to TMEM with tcgen05.cp and issues the stage's eight MMAs, each reading
// its block's scale byte.  Warps 0-7 drain TMEM (warps q and q + 4 share lane
// quadrant q and take alternate 32-token chunks): GEMM1's gate and up warps
// swap half their tokens through shared memory as in the bf16 kernel; each
// warp then holds 32 features (one 32-value block of h) of 16 tokens and
// quantises them with a warp max per token.
//
// Every wait is bounded (2 s); a timeout raises MOE_DEV_WAIT_TIMEOUT, stops the
// other roles, lets in-flight copies and MMAs land, frees TMEM and returns.
#include <cfloat>
#include <cudaTypedefs.h>
#include <cuda_fp8.h>

#include "moe_common.cuh"

namespace moe {

constexpr int kMxTile = 128;                                 // weight rows and tokens per tile
constexpr int kMxStages = 3;
constexpr uint32_t kMxChunkBytes = 128 * 128;                 // 128 rows x one 128-value k-chunk
constexpr uint32_t kMxOpBytes = 2 * kMxChunkBytes;            // one operand of a stage (32 KiB)
constexpr uint32_t kMxAtomBytes = 512;                       // 128 rows x 4 block scales
constexpr uint32_t kMxStageBytes = 2 * kMxOpBytes + 4 * kMxAtomBytes;   // 66 KiB
constexpr int kMxEpiWarps = 8;
constexpr int kMxProdWarp = kMxEpiWarps, kMxMmaWarp = kMxEpiWarps + 1;
constexpr int kMxThreads = 32 * (kMxEpiWarps + 2);
constexpr uint32_t kMxTmemCols = 512;                        // accumulators 0-255, scales from 256
constexpr uint32_t kMxSfaCol = 256, kMxSfbCol = 264;         // 8 columns each (two atoms)
constexpr uint32_t kMxXchgBytes = 16 * 1024;                 // GEMM1 gate / up exchange
constexpr int kMxMaxExperts = 512;

enum MxMode : int { kMxSwiGLUQuant = 0, kMxStore = 1, kMxReduce = 2 };

struct MxParams {
    const int32_t *expert_offsets;
    int E;
    int K;                  // H (GEMM1) or I (GEMM2)
    int n_fblocks;          // weight-row tiles per expert: I/64 (GEMM1) or H/128 (GEMM2)
    int w_rows_per_expert;  // 2I or H
    int half_rows;          // GEMM1: I (the up rows start there)
    int out_cols;           // I (h) or H (y)
    const uint32_t *w_sf;   // [E * w_rows_per_expert, K/128] scale words
    const uint32_t *t_sf;   // [n_rows, K/128] scale words of the token rows
    int64_t n_rows;
    uint8_t *h_q;           // GEMM1: [n_rows, I] codes
    uint8_t *h_sf;          // GEMM1: [n_rows, I/32] scale bytes
    void *y;                // GEMM2: [n_rows, H] bf16
    float *out_reduce;      // GEMM2 decode form: [T, H]
    const int32_t *recv_token;
    const int32_t *recv_slot;
    const float *topk_w;
    int k;
    uint32_t *status;
};

struct MxSmem {
    uint64_t full[kMxStages];
    uint64_t empty[kMxStages];
    uint64_t tmem_full[2];
    uint64_t tmem_empty[2];
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort_flag;
    int total;
    int pair_go[4];        // GEMM1: did the gate warp of each warp pair get its accumulator
};

struct MxTile {
    int e, fb, p0, n_valid, n_mma;
};

__device__ __forceinline__ MxTile mx_tile(int t, const int32_t *s_tpre, const int32_t *s_tb,
                                          const MxParams &P) {
    int lo = 0, hi = P.E - 1;   // last e with s_tpre[e] <= t
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_tpre[mid] <= t) lo = mid; else hi = mid - 1;
    }
    MxTile w;
    w.e = lo;
    const int local = t - s_tpre[lo];
    w.fb = local / s_tb[lo];
    const int tb = local - w.fb * s_tb[lo];
    const int off = P.expert_offsets[lo];
    w.p0 = off + tb * kMxTile;
    w.n_valid = min(kMxTile, P.expert_offsets[lo + 1] - w.p0);
    w.n_mma = (w.n_valid + 15) & ~15;
    return w;
}

__device__ __forceinline__ int mx_exponent(float amax) {
    // the smallest e with amax <= 448 * 2^e (amax = m 2^x, m in [0.5, 1), 448 = 0.875 2^9)
    if (!(amax > 0.0f)) return 0;
    if (amax > FLT_MAX) return 127;
    int x;
    const float m = frexpf(amax, &x);
    const int e = m <= 0.875f ? x - 9 : x - 8;
    return min(127, max(-126, e));
}

__device__ __forceinline__ float mx_pow2_neg(int e) {
    return e == 127 ? __uint_as_float(0x00400000u) : __uint_as_float((uint32_t)(127 - e) << 23);
}

__device__ __forceinline__ void mx_named_barrier(uint32_t id, uint32_t nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

template <int MODE>
__global__ void __launch_bounds__(kMxThreads, 1) ffn_mx_tcgen05_kernel(
    const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_t,
    const MxParams P) {
    constexpr bool kG1 = MODE == kMxSwiGLUQuant;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *base = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char *ring = base;                                       // [stages][A | B | SFA | SFB]
    float *xchg = reinterpret_cast<float *>(base + kMxStages * kMxStageBytes);   // GEMM1
    MxSmem *S = reinterpret_cast<MxSmem *>(base + kMxStages * kMxStageBytes + (kG1 ? kMxXchgBytes : 0));
    int32_t *s_tpre = reinterpret_cast<int32_t *>(S + 1);           // [E + 1] tile prefix
    int32_t *s_tb = s_tpre + (P.E + 1);                              // [E] token blocks per expert

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp == 0) {
        int run = 0;
        for (int e0 = 0; e0 < P.E; e0 += 32) {
            const int e = e0 + lane;
            int tb = 0;
            if (e < P.E) {
                tb = (P.expert_offsets[e + 1] - P.expert_offsets[e] + kMxTile - 1) / kMxTile;
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
        if (lane == 0) { s_tpre[P.E] = run; S->total = run; }
    }
    if (threadIdx.x == 32) {
        for (int s = 0; s < kMxStages; ++s) {
            mbar_init(&S->full[s], 2);       // the TMA bytes' arrival and the scale atoms' arrival
            mbar_init(&S->empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&S->tmem_full[a], 1);
            mbar_init(&S->tmem_empty[a], kMxEpiWarps);
        }
        mbar_init(&S->mma_done, 1);
        S->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kMxProdWarp && lane == 0) { tma_prefetch_desc(&tmap_w); tma_prefetch_desc(&tmap_t); }
    if (warp == kMxMmaWarp) { tmem_alloc_1(&S->tmem_base, kMxTmemCols); tmem_relinquish_1(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const int total = S->total;
    const uint32_t tmem_base = S->tmem_base;
    volatile int *abort_flag = &S->abort_flag;
    const int kwords = P.K / 128;          // scale words per row
    const int num_k = (P.K + 255) / 256;   // ring stages per tile (two k-chunks each; a last
                                           // stage past K loads zeros and scale words 0)

    if (warp == kMxProdWarp) {
        // ------------------------------------------------ TMA + scale gather (whole warp)
        int stage = 0;
        uint32_t phase = 0;
        long long issued = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
            const MxTile w = mx_tile(t, s_tpre, s_tb, P);
            // this lane's four weight rows and four token rows (r = lane + 32 i)
            int64_t wrow[4], trow[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = lane + 32 * i;
                if (kG1)   // gate rows of 64 features, then their up rows
                    wrow[i] = (int64_t)w.e * P.w_rows_per_expert + (r < 64 ? 0 : P.half_rows) + w.fb * 64 + (r & 63);
                else
                    wrow[i] = (int64_t)w.e * P.w_rows_per_expert + w.fb * 128 + r;
                trow[i] = r < w.n_valid ? (int64_t)w.p0 + r : -1;
            }
            for (int kb = 0; kb < num_k; ++kb) {
                bool got = lane == 0 ? mbar_wait_bounded(&S->empty[stage], phase ^ 1u, abort_flag) : true;
                if (!__shfl_sync(0xffffffffu, got ? 1 : 0, 0)) { ok = false; break; }
                unsigned char *st = ring + stage * kMxStageBytes;
                const int ch = 2 * kb;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&S->full[stage], 2 * kMxOpBytes);
                    if (kG1)
                        tma_load_4d(st, &tmap_w, &S->full[stage], 0, w.fb * 64, 2 * w.e, ch);
                    else
                        tma_load_3d(st, &tmap_w, &S->full[stage], 0, w.e * P.w_rows_per_expert + w.fb * 128, ch);
                    tma_load_3d(st + kMxOpBytes, &tmap_t, &S->full[stage], 0, w.p0, ch);
                }
                // scale atoms: atom a (a = 0, 1) holds word ch + a of each row; row r's
                // word at byte 16 (r % 32) + 4 (r / 32), so lane's four rows are one uint4
#pragma unroll
                for (int a = 0; a < 2; ++a) {
                    uint4 wa, ta;
                    uint32_t *pw = &wa.x, *pt = &ta.x;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const bool in_k = ch + a < kwords;
                        pw[i] = in_k ? __ldg(P.w_sf + wrow[i] * kwords + ch + a) : 0u;
                        pt[i] = in_k && trow[i] >= 0 ? __ldg(P.t_sf + trow[i] * kwords + ch + a) : 0u;
                    }
                    *reinterpret_cast<uint4 *>(st + 2 * kMxOpBytes + a * kMxAtomBytes + 16 * lane) = wa;
                    *reinterpret_cast<uint4 *>(st + 2 * kMxOpBytes + (2 + a) * kMxAtomBytes + 16 * lane) = ta;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&S->full[stage]);
                ++issued;
                if (++stage == kMxStages) { stage = 0; phase ^= 1u; }
            }
        }
        if (!ok && lane == 0) {
            raise_status(P.status, MOE_DEV_WAIT_TIMEOUT);
            *abort_flag = 1;
        }
        if (lane == 0) {
            // let the last copies land before the CTA can leave
            volatile int never = 0;
            const long long last = issued < kMxStages ? issued : kMxStages;
            int st = stage;
            uint32_t ph = phase;
            for (long long i = 0; i < last; ++i) {
                if (--st < 0) { st = kMxStages - 1; ph ^= 1u; }
                mbar_wait_bounded(&S->full[st], ph, &never);
            }
        }
        __syncwarp();
    } else if (warp == kMxMmaWarp) {
        // ------------------------------------------------ scale copies + MMA issuer (one lane)
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                const MxTile w = mx_tile(t, s_tpre, s_tb, P);
                if (!mbar_wait_bounded(&S->tmem_empty[acc], acc_phase ^ 1u, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d = tmem_base + (uint32_t)(acc * kMxTile);
                for (int kb = 0; kb < num_k; ++kb) {
                    if (!mbar_wait_bounded(&S->full[stage], phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t st = smem_u32(ring + stage * kMxStageBytes);
                    const uint32_t sf = st + 2 * kMxOpBytes;
#pragma unroll
                    for (int a = 0; a < 2; ++a) {
                        tc_cp_sf_atom(tmem_base + kMxSfaCol + 4 * a, make_sf_atom_desc(sf + a * kMxAtomBytes));
                        tc_cp_sf_atom(tmem_base + kMxSfbCol + 4 * a, make_sf_atom_desc(sf + (2 + a) * kMxAtomBytes));
                    }
#pragma unroll
                    for (int blk = 0; blk < 8; ++blk) {   // 32-value K blocks of the stage
                        const int c = blk >> 2, kk = blk & 3;
                        const uint64_t ad = make_sw128_desc(st + c * kMxChunkBytes + kk * 32);
                        const uint64_t bd = make_sw128_desc(st + kMxOpBytes + c * kMxChunkBytes + kk * 32);
                        const uint32_t sel = (uint32_t)kk << 30;
                        tc_mma_mx_1(d, ad, bd, make_idesc_mx_e4m3(kMxTile, w.n_mma, kk),
                                    (tmem_base + kMxSfaCol + 4 * c) | sel, (tmem_base + kMxSfbCol + 4 * c) | sel,
                                    (kb > 0 || blk > 0) ? 1u : 0u);
                    }
                    tc_commit_1(&S->empty[stage]);    // frees the stage (and its scale atoms)
                    if (++stage == kMxStages) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                tc_commit_1(&S->tmem_full[acc]);
                if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
            }
            if (!ok) {
                raise_status(P.status, MOE_DEV_WAIT_TIMEOUT);
                *abort_flag = 1;
            }
            tc_commit_1(&S->mma_done);
            volatile int never = 0;
            mbar_wait_bounded(&S->mma_done, 0, &never);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue (warps 0-7)
        const int q = warp & 3, half = warp >> 2;
        const bool is_gate = q < 2;
        const int xpair = half * 2 + (q & 1);
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x) {
            const MxTile w = mx_tile(t, s_tpre, s_tb, P);
            // GEMM1: features fb*64 + (q & 1)*32 + lane; GEMM2: fb*128 + q*32 + lane
            const int f = kG1 ? w.fb * 64 + (q & 1) * 32 + lane : w.fb * 128 + q * 32 + lane;
            const bool f_ok = f < P.out_cols;
            bool go;
            if (kG1) {
                // the gate warp waits and tells its up partner, so that both pass the
                // same exchange barriers or both leave
                if (is_gate) {
                    const bool g = lane == 0 ? mbar_wait_bounded(&S->tmem_full[acc], acc_phase, abort_flag) : true;
                    go = __shfl_sync(0xffffffffu, g ? 1 : 0, 0) != 0;
                    if (lane == 0) S->pair_go[xpair] = go ? 1 : 0;
                }
                mx_named_barrier(1 + xpair, 64);
                if (!is_gate) go = *reinterpret_cast<volatile int *>(&S->pair_go[xpair]) != 0;
            } else {
                const bool g = lane == 0 ? mbar_wait_bounded(&S->tmem_full[acc], acc_phase, abort_flag) : true;
                go = __shfl_sync(0xffffffffu, g ? 1 : 0, 0) != 0;
            }
            if (!go) {
                if (lane == 0) { raise_status(P.status, MOE_DEV_WAIT_TIMEOUT); *abort_flag = 1; }
                break;
            }
            tc_fence_after();
            const uint32_t tbase = tmem_base + (uint32_t)(acc * kMxTile) + ((uint32_t)(q * 32) << 16);
            for (int c0 = half * 32; c0 < w.n_mma; c0 += 64) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tbase + c0, r);
                tc_wait_ld_regs(r);
                if (kG1) {
                    // exchange: gate warps hand over tokens 16..31, up warps tokens 0..15
                    float *mine = xchg + (xpair * 2 + (is_gate ? 0 : 1)) * 512;
                    float *theirs = xchg + (xpair * 2 + (is_gate ? 1 : 0)) * 512;
#pragma unroll
                    for (int j = 0; j < 16; ++j) mine[j * 32 + lane] = __uint_as_float(r[is_gate ? 16 + j : j]);
                    mx_named_barrier(1 + xpair, 64);
                    float other[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) other[j] = theirs[j * 32 + lane];
                    mx_named_barrier(1 + xpair, 64);
                    const int cbase = c0 + (is_gate ? 0 : 16);
                    const int nc = min(16, w.n_valid - cbase);
                    // h of 16 tokens for this lane's feature; the warp's 32 features are
                    // one 32-value block of h: scale per token by the warp's maximum
                    const size_t row0 = (size_t)(w.p0 + cbase);
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float own = __uint_as_float(r[is_gate ? j : 16 + j]);
                        const float g = is_gate ? own : other[j], u = is_gate ? other[j] : own;
                        const float hv = __bfloat162float(__float2bfloat16_rn(__fdividef(g, 1.0f + __expf(-g)) * u));
                        const float a = f_ok ? fabsf(hv) : 0.0f;
                        const uint32_t amax_bits = __reduce_max_sync(0xffffffffu, __float_as_uint(a));
                        const int e = mx_exponent(__uint_as_float(amax_bits));
                        const float sc = hv * mx_pow2_neg(e);
                        const uint8_t code = (uint8_t)(__nv_cvt_float_to_fp8(sc, __NV_SATFINITE, __NV_E4M3));
                        if (j < nc) {
                            if (f_ok) P.h_q[(row0 + j) * P.out_cols + f] = code;
                            if (lane == 0 && f - lane < P.out_cols)
                                P.h_sf[(row0 + j) * (P.out_cols / 32) + f / 32] = (uint8_t)(e + 127);
                        }
                    }
                } else if (MODE == kMxStore) {
                    __nv_bfloat16 *y = static_cast<__nv_bfloat16 *>(P.y) + (size_t)w.p0 * P.out_cols + f;
                    const int nc = min(32, w.n_valid - c0);
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (f_ok && j < nc) y[(size_t)(c0 + j) * P.out_cols] = __float2bfloat16_rn(__uint_as_float(r[j]));
                } else {
                    int my_t = 0;
                    float my_w = 0.0f;
                    const int nc = min(32, w.n_valid - c0);
                    if (lane < nc) {
                        const int p = w.p0 + c0 + lane;
                        my_t = P.recv_token[p];
                        my_w = P.topk_w[(size_t)my_t * P.k + P.recv_slot[p]];
                    }
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int tt = __shfl_sync(0xffffffffu, my_t, j);
                        const float ww = __shfl_sync(0xffffffffu, my_w, j);
                        if (j < nc && f_ok)
                            atomicAdd(P.out_reduce + (size_t)tt * P.out_cols + f, ww * __uint_as_float(r[j]));
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
    if (warp == kMxMmaWarp) {
        tc_fence_after();
        tmem_dealloc_1(tmem_base, kMxTmemCols);
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

// E4M3 rows [rows][K] as (128, rows, K / 128): 128-row boxes of two k-chunks.
static bool mx_tmap_rows(CUtensorMap *m, const void *ptr, uint64_t rows, uint64_t K) {
    auto enc = mx_encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {128, rows, K / 128};
    const cuuint64_t strides[2] = {K, 128};
    const cuuint32_t box[3] = {128, 128, 2};
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
    const cuuint32_t box[4] = {128, 64, 2, 2};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t ffn_mx_smem(int E, bool g1) {
    return 1024 + (size_t)kMxStages * kMxStageBytes + (g1 ? kMxXchgBytes : 0) + sizeof(MxSmem) +
           sizeof(int32_t) * (2 * (size_t)E + 1) + 64;
}

template <int MODE>
static cudaError_t launch_mx(const CUtensorMap &tw, const CUtensorMap &tt, const MxParams &P, int grid,
                             cudaStream_t s) {
    const size_t smem = ffn_mx_smem(P.E, MODE == kMxSwiGLUQuant);
    static SmemOptIn opt_in;
    cudaError_t err = opt_in.ensure(ffn_mx_tcgen05_kernel<MODE>, smem);
    if (err != cudaSuccess) return err;
    ffn_mx_tcgen05_kernel<MODE><<<grid, kMxThreads, smem, s>>>(tw, tt, P);
    return cudaGetLastError();
}

// The block-scaled FP8 FFN: GEMM1 (SwiGLU, h quantised by 32-value blocks) then
// GEMM2.  Scale arrays are bytes, one per row and 32 K values (read as words of
// four).  Returns cudaErrorNotSupported when the tensor-map encoder is
// unavailable or E exceeds the tile table's room.
cudaError_t launch_ffn_mx(const moe_config &c, int64_t n_rows, const uint8_t *xr_q, const uint8_t *xr_sf,
                          const int32_t *expert_offsets, const uint8_t *w13_q, const uint8_t *w13_sf,
                          const uint8_t *w2_q, const uint8_t *w2_sf, uint8_t *h_q, uint8_t *h_sf, void *y,
                          const int32_t *recv_token, const int32_t *recv_slot, const float *topk_w,
                          float *out_reduce, uint32_t *status, cudaStream_t s, int num_sms) {
    if (n_rows <= 0) return cudaSuccess;
    if (c.E > kMxMaxExperts) return cudaErrorNotSupported;
    CUtensorMap tw1, tx, tw2, th;
    if (!mx_tmap_w13(&tw1, w13_q, c.E, c.I, c.H) || !mx_tmap_rows(&tx, xr_q, n_rows, c.H) ||
        !mx_tmap_rows(&tw2, w2_q, (uint64_t)c.E * c.H, c.I) || !mx_tmap_rows(&th, h_q, n_rows, c.I))
        return cudaErrorNotSupported;
    MxParams P{};
    P.expert_offsets = expert_offsets;
    P.E = c.E;
    P.n_rows = n_rows;
    P.k = c.k;
    P.status = status;
    P.recv_token = recv_token;
    P.recv_slot = recv_slot;
    P.topk_w = topk_w;
    // GEMM1: 128 rows = the gate and up rows of 64 features
    MxParams P1 = P;
    P1.K = c.H;
    P1.n_fblocks = c.I / 64;
    P1.w_rows_per_expert = 2 * c.I;
    P1.half_rows = c.I;
    P1.out_cols = c.I;
    P1.w_sf = reinterpret_cast<const uint32_t *>(w13_sf);
    P1.t_sf = reinterpret_cast<const uint32_t *>(xr_sf);
    P1.h_q = h_q;
    P1.h_sf = h_sf;
    const long long cap = num_sms;
    long long g1 = (n_rows / kMxTile + c.E) * (long long)P1.n_fblocks;
    cudaError_t err = launch_mx<kMxSwiGLUQuant>(tw1, tx, P1, (int)(g1 < cap ? g1 : cap), s);
    if (err != cudaSuccess) return err;
    MxParams P2 = P;
    P2.K = c.I;
    P2.n_fblocks = c.H / 128;
    P2.w_rows_per_expert = c.H;
    P2.out_cols = c.H;
    P2.w_sf = reinterpret_cast<const uint32_t *>(w2_sf);
    P2.t_sf = reinterpret_cast<const uint32_t *>(h_sf);
    P2.y = y;
    P2.out_reduce = out_reduce;
    long long g2 = (n_rows / kMxTile + c.E) * (long long)P2.n_fblocks;
    const int grid2 = (int)(g2 < cap ? g2 : cap);
    if (c.reduce_dense) return launch_mx<kMxReduce>(tw2, th, P2, grid2, s);
    return launch_mx<kMxStore>(tw2, th, P2, grid2, s);
}

}  // namespace moe
