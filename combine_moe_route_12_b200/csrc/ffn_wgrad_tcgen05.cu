// Weight gradients of the grouped SwiGLU FFN (the backward of the expert
// GEMMs; axolotl ExpertParallelArgs, expert_parallel_save_dispatch: the
// layer's backward under activation checkpointing).  For every expert e and
// its receive rows in each of n_seg segments (the token chunks of a layer
// pass: segment s holds rows [s * seg_rows + off_s[e], s * seg_rows +
// off_s[e+1])):
//   dW2[e]  [H, I]  = sum over its rows p of dy[p] (x) h[p]
//   dW13[e] [2I, H] = sum over its rows p of [dg | du][p] (x) xr[p]
// i.e. out[e] = A_e^T B_e with A = the row-major [rows, M] operand and B the
// row-major [rows, N] operand restricted to the expert's rows.  One pass over
// all segments writes each fp32 gradient once.  The reduction runs over token
// rows, so both operands are read MN-major: a ring stage holds 128 token rows
// of 128 output rows (A) and of 128 output columns (B), each as two 64-element
// blocks of 128-byte rows brought by one 3-D TMA box.
//
// One CTA per SM, tiles (expert, 128 output rows, 128 output columns) dealt
// round-robin (tile = CTA + i * grid), expert by expert, so the tiles that
// read one expert's rows run side by side and share them through L2.  Warp 8
// (one lane) streams the ring with TMA; warp 9 waits for each stage and issues
// the single-CTA tcgen05.mma (bf16 -> fp32, M = N = 128) into one of two TMEM
// accumulators.  An expert's rows rarely fill a segment's last stage: the MMA
// stops at the last 16-row k-step that holds a row of the expert, and the warp
// first zeroes that step's rows past the expert (they belong to the next
// expert, or lie past the valid rows) in both operands.  Warps 0-7 drain TMEM
// (warps q and q + 4 share lane quadrant q and take alternate 64-column
// halves), turn each 32 x 32 block around through shared memory with 16-byte
// accesses (chunk c of row r stored at chunk c ^ (r % 8): no bank conflicts) and
// write it as 16-byte stores, eight lanes per 128-byte row piece of the fp32
// output (or add to it).
//
// Every wait is bounded (2 s); a timeout raises MOE_DEV_WAIT_TIMEOUT, stops the
// other roles, lets in-flight copies and MMAs land, frees TMEM and returns.
#include <cudaTypedefs.h>

#include "moe_common.cuh"

namespace moe {

constexpr int kWgStages = 3;                             // 3 x 64 KiB + 33 KiB staging fits the 227 KiB limit
constexpr int kWgTile = 128;                              // output rows / columns per tile
constexpr int kWgRows = 128;                              // token rows per ring stage
constexpr uint32_t kWgBlockBytes = kWgRows * 128;         // 64 elements x 128 rows (16 KiB)
constexpr uint32_t kWgOpBytes = 2 * kWgBlockBytes;        // one operand of a stage (32 KiB)
constexpr uint32_t kWgStageBytes = 2 * kWgOpBytes;        // 64 KiB
constexpr int kWgEpiWarps = 8;
constexpr int kWgProdWarp = kWgEpiWarps, kWgMmaWarp = kWgEpiWarps + 1;
constexpr int kWgThreads = 32 * (kWgEpiWarps + 2);
constexpr uint32_t kWgTmemCols = 2 * kWgTile;             // two 128-column accumulators
constexpr int kWgPad = 32;                                // staging row stride in floats (16-byte chunks XOR-swizzled by row)

struct WgradParams {
    const int32_t *expert_offsets;   // [n_seg][E + 1]
    int n_seg;
    long long seg_rows;              // row distance between the segments' buffers
    int E;
    int M, N;              // out[e] is [M, N], row-major
    int m_blocks, n_blocks;
    float *out;            // [E, M, N]
    int accumulate;        // 1: out += the gradient, 0: out = the gradient
    uint32_t *status;
};

struct WgSmem {
    uint64_t full[kWgStages];
    uint64_t empty[kWgStages];
    uint64_t tmem_full[2];
    uint64_t tmem_empty[2];
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort_flag;
};

struct WgTile {
    int e, mb, nb, rows;   // rows: the expert's rows over all segments
};

__device__ __forceinline__ WgTile wg_tile(int t, const WgradParams &P) {
    WgTile w;
    const int per_e = P.m_blocks * P.n_blocks;
    w.e = t / per_e;
    const int r = t - w.e * per_e;
    w.mb = r / P.n_blocks;
    w.nb = r - w.mb * P.n_blocks;
    w.rows = 0;
    for (int sg = 0; sg < P.n_seg; ++sg) {
        const int32_t *o = P.expert_offsets + (size_t)sg * (P.E + 1) + w.e;
        w.rows += o[1] - o[0];
    }
    return w;
}

// First row and row count of the expert's part of segment sg.
__device__ __forceinline__ void wg_segment(const WgradParams &P, int e, int sg, int &p0, int &rows) {
    const int32_t *o = P.expert_offsets + (size_t)sg * (P.E + 1) + e;
    p0 = (int)(sg * P.seg_rows) + o[0];
    rows = o[1] - o[0];
}

__global__ void __launch_bounds__(kWgThreads, 1) wgrad_tcgen05_kernel(
    const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
    const WgradParams P) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *base = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char *ring = base;                                            // [stages][A | B]
    float *stg = reinterpret_cast<float *>(base + kWgStages * kWgStageBytes);   // [8][32][33]
    WgSmem *S = reinterpret_cast<WgSmem *>(stg + kWgEpiWarps * 32 * kWgPad);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kWgStages; ++s) { mbar_init(&S->full[s], 1); mbar_init(&S->empty[s], 1); }
        for (int a = 0; a < 2; ++a) { mbar_init(&S->tmem_full[a], 1); mbar_init(&S->tmem_empty[a], kWgEpiWarps); }
        mbar_init(&S->mma_done, 1);
        S->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kWgProdWarp && lane == 0) { tma_prefetch_desc(&tmap_a); tma_prefetch_desc(&tmap_b); }
    if (warp == kWgMmaWarp) { tmem_alloc_1(&S->tmem_base, kWgTmemCols); tmem_relinquish_1(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const int total = P.E * P.m_blocks * P.n_blocks;
    const uint32_t tmem_base = S->tmem_base;
    volatile int *abort_flag = &S->abort_flag;

    if (warp == kWgProdWarp) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                const WgTile w = wg_tile(t, P);
                for (int sg = 0; sg < P.n_seg && ok; ++sg) {
                    int p0, rows;
                    wg_segment(P, w.e, sg, p0, rows);
                    const int nk = (rows + kWgRows - 1) / kWgRows;
                    for (int kb = 0; kb < nk; ++kb) {
                        if (!mbar_wait_bounded(&S->empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
                        unsigned char *st = ring + stage * kWgStageBytes;
                        mbar_arrive_expect_tx(&S->full[stage], kWgStageBytes);
                        const int row = p0 + kb * kWgRows;
                        tma_load_3d(st, &tmap_a, &S->full[stage], 0, row, w.mb * 2);
                        tma_load_3d(st + kWgOpBytes, &tmap_b, &S->full[stage], 0, row, w.nb * 2);
                        ++issued;
                        if (++stage == kWgStages) { stage = 0; phase ^= 1u; }
                    }
                }
            }
            if (!ok) {
                raise_status(P.status, MOE_DEV_WAIT_TIMEOUT);
                *abort_flag = 1;
            }
            // let the last copies land before the CTA can leave
            volatile int never = 0;
            const long long last = issued < kWgStages ? issued : kWgStages;
            int st = stage;
            uint32_t ph = phase;
            for (long long i = 0; i < last; ++i) {
                if (--st < 0) { st = kWgStages - 1; ph ^= 1u; }
                mbar_wait_bounded(&S->full[st], ph, &never);
            }
        }
    } else if (warp == kWgMmaWarp) {
        // ------------------------------------------------ MMA issuer (lane 0), tail fix-up (all lanes)
        const uint32_t idesc = make_idesc_bf16_f32_major(kWgTile, kWgTile, true, true);
        int stage = 0;
        uint32_t phase = 0;
        int acc = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
            const WgTile w = wg_tile(t, P);
            // lane 0 waits and tells the warp, so that the lanes stay together
            bool got = lane == 0 ? mbar_wait_bounded(&S->tmem_empty[acc], acc_phase ^ 1u, abort_flag) : true;
            if (!__shfl_sync(0xffffffffu, got ? 1 : 0, 0)) { ok = false; break; }
            tc_fence_after();
            const uint32_t d = tmem_base + (uint32_t)(acc * kWgTile);
            bool first = true;   // the tile's first MMA overwrites the accumulator
            for (int sg = 0; sg < P.n_seg && ok; ++sg) {
                int p0, rows;
                wg_segment(P, w.e, sg, p0, rows);
                const int nk = (rows + kWgRows - 1) / kWgRows;
                for (int kb = 0; kb < nk; ++kb) {
                    got = lane == 0 ? mbar_wait_bounded(&S->full[stage], phase, abort_flag) : true;
                    if (!__shfl_sync(0xffffffffu, got ? 1 : 0, 0)) { ok = false; break; }
                    tc_fence_after();
                    unsigned char *st = ring + stage * kWgStageBytes;
                    const int v = min(kWgRows, rows - kb * kWgRows);   // rows of the expert in the stage
                    const int ksteps = (v + 15) >> 4;
                    if (v & 15) {
                        // zero rows [v, 16 * ksteps) of both operands' two blocks (128 bytes a row)
                        const int nz = 16 * ksteps - v;
                        for (int i = lane; i < 4 * nz * 8; i += 32) {
                            const int region = i / (nz * 8), rem = i - region * nz * 8;
                            const int row = v + rem / 8, chunk = rem & 7;
                            uint4 *dst = reinterpret_cast<uint4 *>(st + region * kWgBlockBytes + row * 128) + chunk;
                            *dst = make_uint4(0u, 0u, 0u, 0u);
                        }
                        fence_proxy_async_smem();
                    }
                    __syncwarp();
                    if (lane == 0) {
                        const uint32_t a0 = smem_u32(st), b0 = smem_u32(st + kWgOpBytes);
                        for (int ks = 0; ks < ksteps; ++ks) {
                            const uint64_t ad = make_sw128_desc_mn(a0 + ks * 2048, kWgBlockBytes);
                            const uint64_t bd = make_sw128_desc_mn(b0 + ks * 2048, kWgBlockBytes);
                            tc_mma_f16_1(d, ad, bd, idesc, (first && ks == 0) ? 0u : 1u);
                        }
                        tc_commit_1(&S->empty[stage]);   // frees the stage once these MMAs are done
                    }
                    __syncwarp();
                    first = false;
                    if (++stage == kWgStages) { stage = 0; phase ^= 1u; }
                }
            }
            if (!ok) break;
            if (lane == 0) tc_commit_1(&S->tmem_full[acc]);   // accumulator ready (or untouched: no rows)
            __syncwarp();
            if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        }
        if (!ok && lane == 0) {
            raise_status(P.status, MOE_DEV_WAIT_TIMEOUT);
            *abort_flag = 1;
        }
        if (lane == 0) {
            tc_commit_1(&S->mma_done);
            volatile int never = 0;
            mbar_wait_bounded(&S->mma_done, 0, &never);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue (warps 0-7)
        const int q = warp & 3, half = warp >> 2;
        float *my = stg + warp * 32 * kWgPad;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x) {
            const WgTile w = wg_tile(t, P);
            const bool got = lane == 0 ? mbar_wait_bounded(&S->tmem_full[acc], acc_phase, abort_flag) : true;
            if (!__shfl_sync(0xffffffffu, got ? 1 : 0, 0)) {
                if (lane == 0) { raise_status(P.status, MOE_DEV_WAIT_TIMEOUT); *abort_flag = 1; }
                break;
            }
            tc_fence_after();
            const bool write = w.rows > 0 || !P.accumulate;   // no rows: zeros, or nothing to add
            const uint32_t tbase = tmem_base + (uint32_t)(acc * kWgTile) + ((uint32_t)(q * 32) << 16);
            const int row0 = w.mb * kWgTile + q * 32;
            for (int ch = 0; ch < 2 && write; ++ch) {
                const int c0 = half * 64 + ch * 32;
                uint32_t r[32];
                if (w.rows > 0) {
                    tmem_ld_32x32b_x32(tbase + c0, r);
                    tc_wait_ld_regs(r);
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) r[j] = 0u;
                }
                // row (row0 + lane), columns c0..c0+31, as eight 16-byte stores into
                // its staging row (chunk j/4 at chunk (j/4) ^ (lane % 8): the eight
                // lanes of a store phase hit all 32 banks once)
#pragma unroll
                for (int j = 0; j < 32; j += 4)
                    *reinterpret_cast<float4 *>(my + lane * kWgPad + 4 * ((j >> 2) ^ (lane & 7))) =
                        make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                                    __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
                __syncwarp();
                // read back four rows per pass: lane -> row rr0 + lane / 8, columns
                // 4 (lane % 8) .. +3; each row's 32 columns leave as one 128-byte piece
                const int sub = lane >> 3, cq = (lane & 7) * 4;
                const int col = w.nb * kWgTile + c0 + cq;
                const bool full = row0 + 32 <= P.M && w.nb * kWgTile + c0 + 32 <= P.N;
                float *obase = P.out + ((size_t)w.e * P.M + row0) * P.N + col;
#pragma unroll
                for (int rr0 = 0; rr0 < 32; rr0 += 4) {
                    const int rr = rr0 + sub;
                    if (full || (row0 + rr < P.M && col < P.N)) {
                        float4 v = *reinterpret_cast<const float4 *>(my + rr * kWgPad + 4 * ((cq >> 2) ^ (rr & 7)));
                        float4 *o = reinterpret_cast<float4 *>(obase + (size_t)rr * P.N);
                        if (P.accumulate) {
                            const float4 a = *o;
                            v.x += a.x; v.y += a.y; v.z += a.z; v.w += a.w;
                        }
                        *o = v;
                    }
                }
                __syncwarp();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&S->tmem_empty[acc]);
            if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kWgMmaWarp) {
        tc_fence_after();
        tmem_dealloc_1(tmem_base, kWgTmemCols);
    }
}

size_t wgrad_tcgen05_smem() {
    return 1024 + (size_t)kWgStages * kWgStageBytes + sizeof(float) * kWgEpiWarps * 32 * kWgPad +
           sizeof(WgSmem) + 64;
}

// out[e] (+)= A_e^T B_e over the expert's rows in n_seg segments (segment s:
// expert offsets expert_offsets + s * (E + 1), rows seg_rows * s further on);
// tmap_a and tmap_b view A [rows, M] and B [rows, N] as (64, rows, M/64) with
// 128-row boxes of two 64-element blocks (make_tmap_mn).
cudaError_t launch_wgrad_tcgen05(const CUtensorMap &tmap_a, const CUtensorMap &tmap_b,
                                 const int32_t *expert_offsets, int n_seg, long long seg_rows, int E,
                                 int M, int N, float *out, int accumulate, uint32_t *status,
                                 cudaStream_t s, int num_sms) {
    WgradParams P{};
    P.expert_offsets = expert_offsets;
    P.n_seg = n_seg;
    P.seg_rows = seg_rows;
    P.E = E;
    P.M = M;
    P.N = N;
    P.m_blocks = (M + kWgTile - 1) / kWgTile;
    P.n_blocks = (N + kWgTile - 1) / kWgTile;
    P.out = out;
    P.accumulate = accumulate;
    P.status = status;
    const long long tiles = (long long)E * P.m_blocks * P.n_blocks;
    if (tiles <= 0) return cudaSuccess;
    const int grid = (int)(tiles < num_sms ? tiles : num_sms);
    const size_t smem = wgrad_tcgen05_smem();
    static SmemOptIn opt_in;
    cudaError_t err = opt_in.ensure(wgrad_tcgen05_kernel, smem);
    if (err != cudaSuccess) return err;
    wgrad_tcgen05_kernel<<<grid, kWgThreads, smem, s>>>(tmap_a, tmap_b, P);
    return cudaGetLastError();
}

}  // namespace moe
