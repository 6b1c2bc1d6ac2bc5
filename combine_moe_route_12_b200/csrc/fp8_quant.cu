// FP8 quantisation by rows (LightLLM PR 1687: UE8M0 FP8 quantisation of the
// dispatch input and of h after silu_and_mul): E4M3 codes and one UE8M0
// (power-of-two) scale per row.  Used on x per chunk, on h between the two
// grouped GEMMs, and once on the expert weights.
//
// One warp per row, 16-byte loads.  Rows of up to 256 vectors (2048 bf16 or
// 1024 fp32 values) stay in registers between the maximum and the codes;
// longer rows take a second pass over the row (from L1).  HBM-bound: rows *
// cols * (element + 1) bytes.
#include <cfloat>
#include <cuda_fp8.h>

#include "moe_common.cuh"

namespace moe {

constexpr int kQuantWarps = 8;

// The scale exponent: the smallest e with amax <= 448 * 2^e.  With amax =
// m * 2^x, m in [0.5, 1), and 448 = 0.875 * 2^9, that is e = x - 9 when
// m <= 0.875 and x - 8 otherwise; clamped to the UE8M0 range used here.
__device__ __forceinline__ int ue8m0_exponent(float amax) {
    if (!(amax > 0.0f)) return 0;
    if (amax > FLT_MAX) return 127;
    int x;
    const float m = frexpf(amax, &x);
    const int e = m <= 0.875f ? x - 9 : x - 8;
    return min(127, max(-126, e));
}

// 2^-e for e in [-126, 127] (2^-127 is an fp32 subnormal).
__device__ __forceinline__ float pow2_neg(int e) {
    return e == 127 ? __uint_as_float(0x00400000u) : __uint_as_float((uint32_t)(127 - e) << 23);
}

__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
    // the first value lands in the low byte (memory order)
    return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

template <bool BF16>
__device__ __forceinline__ float vec_amax(const uint4 &q) {
    if (BF16)
        return fmaxf(fmaxf(fmaxf(fabsf(bf16_lo(q.x)), fabsf(bf16_hi(q.x))),
                           fmaxf(fabsf(bf16_lo(q.y)), fabsf(bf16_hi(q.y)))),
                     fmaxf(fmaxf(fabsf(bf16_lo(q.z)), fabsf(bf16_hi(q.z))),
                           fmaxf(fabsf(bf16_lo(q.w)), fabsf(bf16_hi(q.w)))));
    return fmaxf(fmaxf(fabsf(__uint_as_float(q.x)), fabsf(__uint_as_float(q.y))),
                 fmaxf(fabsf(__uint_as_float(q.z)), fabsf(__uint_as_float(q.w))));
}

// The 8 codes of one 16-byte vector of 8 bf16 values.
__device__ __forceinline__ uint2 bf16_vec_codes(const uint4 &q, float inv) {
    uint2 o;
    o.x = e4m3x2(bf16_lo(q.x) * inv, bf16_hi(q.x) * inv) |
          e4m3x2(bf16_lo(q.y) * inv, bf16_hi(q.y) * inv) << 16;
    o.y = e4m3x2(bf16_lo(q.z) * inv, bf16_hi(q.z) * inv) |
          e4m3x2(bf16_lo(q.w) * inv, bf16_hi(q.w) * inv) << 16;
    return o;
}

// The codes of one 16-byte vector (8 bf16 or 4 fp32 values) at vector v of dst.
template <bool BF16>
__device__ __forceinline__ void vec_store_codes(uint8_t *dst, int v, const uint4 &q, float inv) {
    if (BF16) {
        reinterpret_cast<uint2 *>(dst)[v] = bf16_vec_codes(q, inv);
    } else {
        reinterpret_cast<uint32_t *>(dst)[v] =
            e4m3x2(__uint_as_float(q.x) * inv, __uint_as_float(q.y) * inv) |
            e4m3x2(__uint_as_float(q.z) * inv, __uint_as_float(q.w) * inv) << 16;
    }
}

// rows: allocated rows; n_dev (optional): the device-side row count, rows
// past it are left untouched.  kRegVecs > 0: every lane holds its (at most
// kRegVecs) vectors of the row in registers; 0: two passes over the row.
template <bool BF16, int kRegVecs>
__global__ void __launch_bounds__(32 * kQuantWarps) quant_rows_kernel(
    int64_t rows, int cols, const void *__restrict__ in, uint8_t *__restrict__ codes,
    uint8_t *__restrict__ scales, const int32_t *__restrict__ n_dev) {
    int64_t n = rows;
    if (n_dev) n = min(n, (int64_t)max(*n_dev, 0));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int kVecElems = BF16 ? 8 : 4;
    const int nv = cols / kVecElems;
    for (int64_t r = (int64_t)blockIdx.x * kQuantWarps + warp; r < n;
         r += (int64_t)gridDim.x * kQuantWarps) {
        const uint4 *src = reinterpret_cast<const uint4 *>(
            static_cast<const char *>(in) + (size_t)r * cols * (BF16 ? 2 : 4));
        uint8_t *dst = codes + (size_t)r * cols;
        float amax = 0.0f;
        uint4 q[kRegVecs > 0 ? kRegVecs : 1];
        if (kRegVecs > 0) {
#pragma unroll
            for (int i = 0; i < kRegVecs; ++i) {
                const int v = lane + 32 * i;
                q[i] = v < nv ? src[v] : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int i = 0; i < kRegVecs; ++i) amax = fmaxf(amax, vec_amax<BF16>(q[i]));
        } else {
            for (int v = lane; v < nv; v += 32) amax = fmaxf(amax, vec_amax<BF16>(src[v]));
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        const int e = ue8m0_exponent(amax);
        const float inv = pow2_neg(e);      // exact: the scaled values are x / 2^e
        if (lane == 0) scales[r] = (uint8_t)(e + 127);
        if (kRegVecs > 0) {
#pragma unroll
            for (int i = 0; i < kRegVecs; ++i) {
                const int v = lane + 32 * i;
                if (v < nv) vec_store_codes<BF16>(dst, v, q[i], inv);
            }
        } else {
            for (int v = lane; v < nv; v += 32) vec_store_codes<BF16>(dst, v, src[v], inv);
        }
    }
}

// Quantise-and-permute of a chunk's bf16 token rows (the forward's FP8 path):
// one CTA per token; the row is read once into registers (VPT 16-byte vectors
// per thread), its scale taken over the CTA, and its codes written straight to
// each kept receive row; a token with every slot dropped is not read.  The
// codes equal those of quant_rows_kernel followed by the permute.
constexpr int kPqThreads = 128;

template <int VPT>
__global__ void __launch_bounds__(kPqThreads) permute_quant_kernel(
    int tb, int k, int row_vecs, const uint4 *__restrict__ x, const int32_t *__restrict__ pos,
    uint8_t *__restrict__ xr_q, uint8_t *__restrict__ x_scale) {
    grid_dependency_wait();
    grid_dependents_launch();
    __shared__ int32_t s_pos[kMaxTopK];
    __shared__ float s_red[kPqThreads / 32];
    __shared__ int s_any;
    const int i = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp == 0) {
        const int p = lane < k ? pos[(size_t)i * k + lane] : -1;
        if (lane < k) s_pos[lane] = p;
        const uint32_t any = __ballot_sync(0xffffffffu, p >= 0);
        if (lane == 0) s_any = any != 0u;
    }
    __syncthreads();
    if (!s_any) return;                         // every slot dropped: x[t] is not needed
    const uint4 *src = x + (size_t)(tb + i) * row_vecs;
    uint4 q[VPT];
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
        const int v = threadIdx.x + kPqThreads * j;
        q[j] = v < row_vecs ? __ldg(src + v) : make_uint4(0u, 0u, 0u, 0u);
        amax = fmaxf(amax, vec_amax<true>(q[j]));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if (lane == 0) s_red[warp] = amax;
    __syncthreads();
#pragma unroll
    for (int w = 0; w < kPqThreads / 32; ++w) amax = fmaxf(amax, s_red[w]);
    const int e = ue8m0_exponent(amax);
    const float inv = pow2_neg(e);
    if (threadIdx.x == 0) x_scale[tb + i] = (uint8_t)(e + 127);
    const size_t row_bytes = (size_t)row_vecs * 8;
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
        const int v = threadIdx.x + kPqThreads * j;
        if (v >= row_vecs) continue;
        const uint2 c = bf16_vec_codes(q[j], inv);
        for (int jj = 0; jj < k; ++jj) {
            const int p = s_pos[jj];
            if (p >= 0) reinterpret_cast<uint2 *>(xr_q + (size_t)p * row_bytes)[v] = c;
        }
    }
}

// Returns cudaErrorNotSupported for rows longer than 1024 vectors (8192 values).
cudaError_t launch_permute_quant(const moe_config &c, const void *x, const int32_t *pos, int tb,
                                 int tc, uint8_t *xr_q, uint8_t *x_scale, cudaStream_t s) {
    if (tc == 0) return cudaSuccess;
    const int row_vecs = c.H / 8;
    const uint4 *xv = static_cast<const uint4 *>(x);
    if (row_vecs <= 2 * kPqThreads)
        return launch_dependent(permute_quant_kernel<2>, tc, kPqThreads, 0, s, tb, c.k, row_vecs, xv, pos, xr_q, x_scale);
    if (row_vecs <= 8 * kPqThreads)
        return launch_dependent(permute_quant_kernel<8>, tc, kPqThreads, 0, s, tb, c.k, row_vecs, xv, pos, xr_q, x_scale);
    return cudaErrorNotSupported;
}

// ------------------------------------------------------------------ K-blocked scales
// One UE8M0 scale per 32 consecutive values of a row (the MX block of the
// block-scaled tensor-core MMA): a row-major [rows, cols] array with cols % 32 ==
// 0 is a flat run of 32-value blocks.  LPB consecutive lanes take one block (4
// bf16 or 8 fp32 vectors of 16 bytes), its maximum by shuffles among them; the
// codes as in the row form; scales[b] for block b (row-major [rows, cols / 32]).
template <bool BF16>
__global__ void __launch_bounds__(256) quant_blocks_kernel(int64_t n_blocks, const uint4 *__restrict__ src,
                                                           uint8_t *__restrict__ codes,
                                                           uint8_t *__restrict__ scales) {
    constexpr int LPB = BF16 ? 4 : 8;      // lanes per block
    const int64_t n_vec = n_blocks * LPB;
    const int64_t step = (int64_t)gridDim.x * blockDim.x;
    // every lane of a warp runs the same trips (the shuffles need them all)
    for (int64_t v0 = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31); v0 < n_vec; v0 += step) {
        const int64_t v = v0 + (threadIdx.x & 31);
        const bool live = v < n_vec;
        const uint4 q = live ? __ldg(src + v) : make_uint4(0u, 0u, 0u, 0u);
        float amax = vec_amax<BF16>(q);
#pragma unroll
        for (int off = 1; off < LPB; off <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        if (!live) continue;
        const int e = ue8m0_exponent(amax);
        const float inv = pow2_neg(e);
        if (BF16) {
            reinterpret_cast<uint2 *>(codes)[v] = bf16_vec_codes(q, inv);
        } else {
            reinterpret_cast<uint32_t *>(codes)[v] =
                e4m3x2(__uint_as_float(q.x) * inv, __uint_as_float(q.y) * inv) |
                e4m3x2(__uint_as_float(q.z) * inv, __uint_as_float(q.w) * inv) << 16;
        }
        if ((v & (LPB - 1)) == 0) scales[v / LPB] = (uint8_t)(e + 127);
    }
}

cudaError_t launch_quant_blocks(int64_t rows, int cols, bool bf16, const void *in, uint8_t *codes,
                                uint8_t *scales, cudaStream_t s, int num_sms) {
    const int64_t n_blocks = rows * (int64_t)(cols / 32);
    if (n_blocks <= 0) return cudaSuccess;
    const int64_t n_vec = n_blocks * (bf16 ? 4 : 8);
    long long grid = (n_vec + 255) / 256;
    const long long cap = (long long)num_sms * 8;
    if (grid > cap) grid = cap;
    if (bf16)
        quant_blocks_kernel<true><<<(unsigned)grid, 256, 0, s>>>(n_blocks, static_cast<const uint4 *>(in),
                                                                codes, scales);
    else
        quant_blocks_kernel<false><<<(unsigned)grid, 256, 0, s>>>(n_blocks, static_cast<const uint4 *>(in),
                                                                 codes, scales);
    return cudaGetLastError();
}

// Quantise-and-permute with K-blocked scales: one CTA per token of the chunk;
// thread t holds vectors t, t + 128, ... of the bf16 row (a 32-value block is
// four consecutive vectors, so four consecutive lanes), the block maximum by two
// shuffles; each kept receive row p gets the codes and the row's block scales
// (xr_sf [N_max, H / 32]).  A token with every slot dropped is not read.
template <int VPT>
__global__ void __launch_bounds__(kPqThreads) permute_quant_blocks_kernel(
    int tb, int k, int row_vecs, const uint4 *__restrict__ x, const int32_t *__restrict__ pos,
    uint8_t *__restrict__ xr_q, uint8_t *__restrict__ xr_sf) {
    grid_dependency_wait();
    grid_dependents_launch();
    __shared__ int32_t s_pos[kMaxTopK];
    __shared__ int s_any;
    const int i = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp == 0) {
        const int p = lane < k ? pos[(size_t)i * k + lane] : -1;
        if (lane < k) s_pos[lane] = p;
        const uint32_t any = __ballot_sync(0xffffffffu, p >= 0);
        if (lane == 0) s_any = any != 0u;
    }
    __syncthreads();
    if (!s_any) return;
    const uint4 *src = x + (size_t)(tb + i) * row_vecs;
    const size_t row_bytes = (size_t)row_vecs * 8, sf_bytes = (size_t)row_vecs / 4;
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
        const int v = threadIdx.x + kPqThreads * j;
        const uint4 q = v < row_vecs ? __ldg(src + v) : make_uint4(0u, 0u, 0u, 0u);
        float amax = vec_amax<true>(q);
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        if (v >= row_vecs) continue;
        const int e = ue8m0_exponent(amax);
        const uint2 c = bf16_vec_codes(q, pow2_neg(e));
        for (int jj = 0; jj < k; ++jj) {
            const int p = s_pos[jj];
            if (p < 0) continue;
            reinterpret_cast<uint2 *>(xr_q + (size_t)p * row_bytes)[v] = c;
            if ((v & 3) == 0) xr_sf[(size_t)p * sf_bytes + v / 4] = (uint8_t)(e + 127);
        }
    }
}

// Returns cudaErrorNotSupported for rows longer than 1024 vectors (8192 values).
cudaError_t launch_permute_quant_blocks(const moe_config &c, const void *x, const int32_t *pos, int tb,
                                        int tc, uint8_t *xr_q, uint8_t *xr_sf, cudaStream_t s) {
    if (tc == 0) return cudaSuccess;
    const int row_vecs = c.H / 8;
    const uint4 *xv = static_cast<const uint4 *>(x);
    if (row_vecs <= 2 * kPqThreads)
        return launch_dependent(permute_quant_blocks_kernel<2>, tc, kPqThreads, 0, s, tb, c.k, row_vecs, xv, pos, xr_q, xr_sf);
    if (row_vecs <= 8 * kPqThreads)
        return launch_dependent(permute_quant_blocks_kernel<8>, tc, kPqThreads, 0, s, tb, c.k, row_vecs, xv, pos, xr_q, xr_sf);
    return cudaErrorNotSupported;
}

cudaError_t launch_quant_rows(int64_t rows, int cols, bool bf16, const void *in, uint8_t *codes,
                              uint8_t *scales, const int32_t *n_dev, cudaStream_t s, int num_sms) {
    if (rows <= 0) return cudaSuccess;
    long long blocks = (rows + kQuantWarps - 1) / kQuantWarps;
    const long long cap = (long long)num_sms * 16;
    if (blocks > cap) blocks = cap;
    const int nv = cols / (bf16 ? 8 : 4);
    const dim3 g((unsigned)blocks), b(32 * kQuantWarps);
    if (bf16) {
        if (nv <= 32 * 8) quant_rows_kernel<true, 8><<<g, b, 0, s>>>(rows, cols, in, codes, scales, n_dev);
        else quant_rows_kernel<true, 0><<<g, b, 0, s>>>(rows, cols, in, codes, scales, n_dev);
    } else {
        if (nv <= 32 * 8) quant_rows_kernel<false, 8><<<g, b, 0, s>>>(rows, cols, in, codes, scales, n_dev);
        else quant_rows_kernel<false, 0><<<g, b, 0, s>>>(rows, cols, in, codes, scales, n_dev);
    }
    return cudaGetLastError();
}

}  // namespace moe
