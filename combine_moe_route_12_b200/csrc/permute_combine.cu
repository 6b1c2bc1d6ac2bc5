// Steps 4 and 6: the row permutation into the receive layout and the weighted
// combine back to token order (axolotl ExpertParallelArgs: dispatch / combine
// all_to_all_single outputs; LightLLM PR 1687: decode reduce into a dense
// output).  Both are HBM-bound row copies with 16-byte vector loads and stores,
// each source row read once.  A CTA takes tpc <= kTokPerCta consecutive
// tokens: their pos (and weights) arrive with one load round and one barrier.
// Large chunks take several tokens per CTA, so that a token with one kept row
// or none is not dominated by the CTA's start-up; chunks that would then leave
// SMs idle take one (tok_per_cta).
//
//   permute:  x[t] is read once and written to each of its kept receive rows;
//             a token with no kept row is not read at all.
//   combine:  out[t] = sum_j w[t, j] * y[pos[t, j]] in fp32, slot order,
//             rounded once to the storage type.
#include "moe_common.cuh"

namespace moe {

constexpr int kRowThreads = 128;
constexpr int kTokPerCta = 4;                 // kTokPerCta * kMaxTopK <= kRowThreads
static_assert(kTokPerCta * kMaxTopK <= kRowThreads, "one pos per thread");

// Tokens per CTA: as many (up to kTokPerCta) as still leave about 27 CTAs per
// SM (1.7 waves of 16 resident): 16384 tokens take 4 per CTA on 148 SMs, 4096
// take 1 (measured: 4 per CTA there left SMs idle and slowed the permute).
static int tok_per_cta(int tc) {
    int dev = 0, nsm = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    const int t = tc / (nsm * 27);
    return t < 1 ? 1 : (t > kTokPerCta ? kTokPerCta : t);
}

// pos (and topk_w; unit weights when it is NULL, the permute's backward) of the
// CTA's tokens [i0, i0 + n) into shared memory.
__device__ __forceinline__ void load_slots(int tb, int i0, int n, int k, const int32_t *pos,
                                           const float *topk_w, int32_t (*s_pos)[kMaxTopK],
                                           float (*s_w)[kMaxTopK]) {
    const int a = threadIdx.x / k, j = threadIdx.x - a * k;
    if (a < n) {
        s_pos[a][j] = pos[(size_t)(i0 + a) * k + j];
        if (s_w) s_w[a][j] = topk_w ? topk_w[(size_t)(tb + i0 + a) * k + j] : 1.0f;
    }
}

__global__ void __launch_bounds__(kRowThreads) permute_rows_kernel(
    int tb, int tc, int tpc, int k, int row_vecs, const uint4 *__restrict__ x, const int32_t *__restrict__ pos,
    uint4 *__restrict__ xr) {
    grid_dependency_wait();
    grid_dependents_launch();
    __shared__ int32_t s_pos[kTokPerCta][kMaxTopK];
    const int i0 = blockIdx.x * tpc;
    const int n = min(tpc, tc - i0);
    load_slots(tb, i0, n, k, pos, nullptr, s_pos, nullptr);
    __syncthreads();
    for (int a = 0; a < n; ++a) {
        bool any = false;
        for (int j = 0; j < k; ++j) any |= s_pos[a][j] >= 0;
        if (!any) continue;                   // every slot dropped: x[t] is not needed
        const uint4 *src = x + (size_t)(tb + i0 + a) * row_vecs;
        for (int v = threadIdx.x; v < row_vecs; v += kRowThreads) {
            const uint4 d = __ldg(src + v);
            for (int j = 0; j < k; ++j) {
                const int p = s_pos[a][j];
                if (p >= 0) xr[(size_t)p * row_vecs + v] = d;
            }
        }
    }
}

__device__ __forceinline__ void unpack8(const uint4 &u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        f[2 * q] = __uint_as_float(w[q] << 16);
        f[2 * q + 1] = __uint_as_float(w[q] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat16 l = __float2bfloat16_rn(lo), h = __float2bfloat16_rn(hi);
    return (uint32_t)__bfloat16_as_ushort(l) | ((uint32_t)__bfloat16_as_ushort(h) << 16);
}

constexpr int kCombineBatch = 4;   // expert rows of a token loaded together

// bf16 storage: one uint4 = 8 elements.
__global__ void __launch_bounds__(kRowThreads) combine_rows_bf16_kernel(
    int tb, int tc, int tpc, int k, int row_vecs, const uint4 *__restrict__ y, const int32_t *__restrict__ pos,
    const float *__restrict__ topk_w, const uint4 *__restrict__ y_shared, uint4 *__restrict__ out) {
    grid_dependency_wait();
    grid_dependents_launch();
    __shared__ int32_t s_pos_all[kTokPerCta][kMaxTopK];
    __shared__ float s_w_all[kTokPerCta][kMaxTopK];
    const int i0 = blockIdx.x * tpc;
    const int n = min(tpc, tc - i0);
    load_slots(tb, i0, n, k, pos, topk_w, s_pos_all, s_w_all);
    __syncthreads();
    for (int a = 0; a < n; ++a) {
    const int i = i0 + a;
    const int t = tb + i;
    const int32_t *s_pos = s_pos_all[a];
    const float *s_w = s_w_all[a];
    // two 16-byte columns per pass, all their row loads issued before any add or
    // store: a token with one or two kept rows still has several loads in flight
    for (int v0 = threadIdx.x; v0 < row_vecs; v0 += 2 * kRowThreads) {
        const int v1 = v0 + kRowThreads;
        const bool has1 = v1 < row_vecs;
        float acc0[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        float acc1[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (y_shared) {   // the shared expert's row
            unpack8(__ldg(y_shared + (size_t)i * row_vecs + v0), acc0);
            if (has1) unpack8(__ldg(y_shared + (size_t)i * row_vecs + v1), acc1);
        }
        for (int j0 = 0; j0 < k; j0 += kCombineBatch) {
            // the adds keep slot order
            uint4 u0[kCombineBatch], u1[kCombineBatch];
#pragma unroll
            for (int jj = 0; jj < kCombineBatch; ++jj) {
                const int p = j0 + jj < k ? s_pos[j0 + jj] : -1;
                const uint4 *row = y + (size_t)(p >= 0 ? p : 0) * row_vecs;
                u0[jj] = p >= 0 ? __ldg(row + v0) : make_uint4(0u, 0u, 0u, 0u);
                u1[jj] = (p >= 0 && has1) ? __ldg(row + v1) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int jj = 0; jj < kCombineBatch; ++jj) {
                if (j0 + jj >= k || s_pos[j0 + jj] < 0) continue;
                const float w = s_w[j0 + jj];
                float f[8];
                unpack8(u0[jj], f);
#pragma unroll
                for (int q = 0; q < 8; ++q) acc0[q] = __fmaf_rn(w, f[q], acc0[q]);
                unpack8(u1[jj], f);
#pragma unroll
                for (int q = 0; q < 8; ++q) acc1[q] = __fmaf_rn(w, f[q], acc1[q]);
            }
        }
        uint4 o;
        o.x = pack_bf16x2(acc0[0], acc0[1]);
        o.y = pack_bf16x2(acc0[2], acc0[3]);
        o.z = pack_bf16x2(acc0[4], acc0[5]);
        o.w = pack_bf16x2(acc0[6], acc0[7]);
        out[(size_t)t * row_vecs + v0] = o;
        if (has1) {
            o.x = pack_bf16x2(acc1[0], acc1[1]);
            o.y = pack_bf16x2(acc1[2], acc1[3]);
            o.z = pack_bf16x2(acc1[4], acc1[5]);
            o.w = pack_bf16x2(acc1[6], acc1[7]);
            out[(size_t)t * row_vecs + v1] = o;
        }
    }
    }
}

// fp32 storage: one float4 = 4 elements.
__global__ void __launch_bounds__(kRowThreads) combine_rows_f32_kernel(
    int tb, int tc, int tpc, int k, int row_vecs, const float4 *__restrict__ y, const int32_t *__restrict__ pos,
    const float *__restrict__ topk_w, const float4 *__restrict__ y_shared, float4 *__restrict__ out) {
    grid_dependency_wait();
    grid_dependents_launch();
    __shared__ int32_t s_pos_all[kTokPerCta][kMaxTopK];
    __shared__ float s_w_all[kTokPerCta][kMaxTopK];
    const int i0 = blockIdx.x * tpc;
    const int n = min(tpc, tc - i0);
    load_slots(tb, i0, n, k, pos, topk_w, s_pos_all, s_w_all);
    __syncthreads();
    for (int a = 0; a < n; ++a) {
    const int i = i0 + a;
    const int t = tb + i;
    const int32_t *s_pos = s_pos_all[a];
    const float *s_w = s_w_all[a];
    for (int v = threadIdx.x; v < row_vecs; v += kRowThreads) {
        float4 acc = y_shared ? __ldg(y_shared + (size_t)i * row_vecs + v) : make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < k; ++j) {
            const int p = s_pos[j];
            if (p < 0) continue;
            const float4 f = __ldg(y + (size_t)p * row_vecs + v);
            const float w = s_w[j];
            acc.x = __fmaf_rn(w, f.x, acc.x);
            acc.y = __fmaf_rn(w, f.y, acc.y);
            acc.z = __fmaf_rn(w, f.z, acc.z);
            acc.w = __fmaf_rn(w, f.w, acc.w);
        }
        out[(size_t)t * row_vecs + v] = acc;
    }
    }
}

// Decode form: out[t] = round(out_reduce[t]) for the chunk's tokens.
__global__ void reduce_finalize_kernel(int tb, int tc, int H, int dtype,
                                       const float4 *__restrict__ red, const void *__restrict__ y_shared,
                                       void *__restrict__ out) {
    grid_dependency_wait();
    grid_dependents_launch();
    const size_t n4 = (size_t)tc * H / 4;
    const size_t base4 = (size_t)tb * H / 4;
    for (size_t q = (size_t)blockIdx.x * blockDim.x + threadIdx.x; q < n4;
         q += (size_t)gridDim.x * blockDim.x) {
        float4 v = red[base4 + q];
        if (y_shared) {   // the shared expert's row (chunk-relative), added before the rounding
            float s[4];
            if (dtype == MOE_F32) {
                const float4 f = reinterpret_cast<const float4 *>(y_shared)[q];
                s[0] = f.x; s[1] = f.y; s[2] = f.z; s[3] = f.w;
            } else {
                const uint2 u = reinterpret_cast<const uint2 *>(y_shared)[q];
                s[0] = __uint_as_float(u.x << 16); s[1] = __uint_as_float(u.x & 0xFFFF0000u);
                s[2] = __uint_as_float(u.y << 16); s[3] = __uint_as_float(u.y & 0xFFFF0000u);
            }
            v.x = __fadd_rn(s[0], v.x); v.y = __fadd_rn(s[1], v.y);
            v.z = __fadd_rn(s[2], v.z); v.w = __fadd_rn(s[3], v.w);
        }
        if (dtype == MOE_F32) {
            reinterpret_cast<float4 *>(out)[base4 + q] = v;
        } else {
            uint2 o;
            o.x = pack_bf16x2(v.x, v.y);
            o.y = pack_bf16x2(v.z, v.w);
            reinterpret_cast<uint2 *>(out)[base4 + q] = o;
        }
    }
}

// Warp-per-token permute for large chunks of rows of at most 32 * kWarpVecs
// 16-byte vectors (2048 bf16 values): four independent warps per CTA, no
// barrier; a warp reads its token's pos once (a lane per slot) and then has the
// whole row in flight, kWarpVecs loads per lane, instead of a chain of
// dependent rounds per token.  (The same form of the combine measured slower
// than four tokens per CTA and is not used.)
constexpr int kWarpVecs = 8;

__global__ void __launch_bounds__(kRowThreads) permute_rows_warp_kernel(
    int tb, int tc, int k, int row_vecs, const uint4 *__restrict__ x, const int32_t *__restrict__ pos,
    uint4 *__restrict__ xr) {
    grid_dependency_wait();
    grid_dependents_launch();
    const int lane = threadIdx.x & 31;
    const int i = blockIdx.x * (kRowThreads / 32) + (threadIdx.x >> 5);
    if (i >= tc) return;
    const int my_p = lane < k ? pos[(size_t)i * k + lane] : -1;
    uint32_t kept = __ballot_sync(0xffffffffu, my_p >= 0);
    if (!kept) return;                        // every slot dropped: x[t] is not needed
    const uint4 *src = x + (size_t)(tb + i) * row_vecs;
    uint4 d[kWarpVecs];
#pragma unroll
    for (int q = 0; q < kWarpVecs; ++q) {
        const int v = lane + 32 * q;
        if (v < row_vecs) d[q] = __ldg(src + v);
    }
    while (kept) {
        const int j = __ffs(kept) - 1;
        kept &= kept - 1;
        const int p = __shfl_sync(0xffffffffu, my_p, j);
        uint4 *dst = xr + (size_t)p * row_vecs;
#pragma unroll
        for (int q = 0; q < kWarpVecs; ++q) {
            const int v = lane + 32 * q;
            if (v < row_vecs) dst[v] = d[q];
        }
    }
}

cudaError_t launch_permute(const moe_config &c, const void *x, const int32_t *pos, int tb,
                           int tc, void *xr, cudaStream_t s) {
    if (tc == 0) return cudaSuccess;
    // row bytes: E4M3 codes when the FFN runs in FP8, else the layer dtype
    const int row_vecs = (int)((size_t)c.H * (c.ffn_fp8 ? 1 : c.dtype == MOE_F32 ? 4 : 2) / 16);
    const int tpc = tok_per_cta(tc);
    if (tpc > 1 && row_vecs <= 32 * kWarpVecs) {
        return launch_dependent(permute_rows_warp_kernel, (tc + 3) / 4, kRowThreads, 0, s,
                                tb, tc, c.k, row_vecs, static_cast<const uint4 *>(x), pos, static_cast<uint4 *>(xr));
    }
    return launch_dependent(permute_rows_kernel, (tc + tpc - 1) / tpc, kRowThreads, 0, s,
                            tb, tc, tpc, c.k, row_vecs, static_cast<const uint4 *>(x), pos, static_cast<uint4 *>(xr));
}

cudaError_t launch_combine(const moe_config &c, const void *y, const int32_t *pos,
                           const float *topk_w, int tb, int tc, const void *y_shared, void *out,
                           cudaStream_t s) {
    if (tc == 0) return cudaSuccess;
    const int tpc = tok_per_cta(tc);
    if (c.dtype == MOE_F32) {
        const int row_vecs = c.H / 4;
        return launch_dependent(combine_rows_f32_kernel, (tc + tpc - 1) / tpc, kRowThreads, 0, s,
                                tb, tc, tpc, c.k, row_vecs, static_cast<const float4 *>(y), pos, topk_w,
                                static_cast<const float4 *>(y_shared), static_cast<float4 *>(out));
    } else {
        const int row_vecs = c.H / 8;
        return launch_dependent(combine_rows_bf16_kernel, (tc + tpc - 1) / tpc, kRowThreads, 0, s,
                                tb, tc, tpc, c.k, row_vecs, static_cast<const uint4 *>(y), pos, topk_w,
                                static_cast<const uint4 *>(y_shared), static_cast<uint4 *>(out));
    }
}

cudaError_t launch_reduce_finalize(const moe_config &c, const float *red, int tb, int tc,
                                   const void *y_shared, void *out, cudaStream_t s, int num_sms) {
    if (tc == 0) return cudaSuccess;
    const size_t n4 = (size_t)tc * c.H / 4;
    int blocks = (int)((n4 + 255) / 256);
    if (blocks > num_sms * 8) blocks = num_sms * 8;
    return launch_dependent(reduce_finalize_kernel, blocks, 256, 0, s, tb, tc, c.H, c.dtype,
                            reinterpret_cast<const float4 *>(red), y_shared, out);
}

// Expert offsets {0, rows} of the shared expert's one-expert FFN launch.
__global__ void shared_offsets_kernel(int32_t *off, int rows) {
    off[0] = 0;
    off[1] = rows;
}
cudaError_t launch_shared_offsets(int32_t *off, int rows, cudaStream_t s) {
    shared_offsets_kernel<<<1, 1, 0, s>>>(off, rows);
    return cudaGetLastError();
}

}  // namespace moe
