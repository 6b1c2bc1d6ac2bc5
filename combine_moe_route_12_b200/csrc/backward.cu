// Backward steps of the layer that are row passes over HBM (axolotl
// ExpertParallelArgs, expert_parallel_save_dispatch: the layer's backward, with
// the routing top-k and the split counts saved from the forward).
//
//   combine:  dy[p] = w[t,j] dout[t] for each kept slot (its receive row p),
//             dw[t,j] = <dout[t], y[p]> (fp32, reduced over the CTA)
//   routing:  dz[t,j] = w[t,j] (dw[t,j] - sum_i w[t,i] dw[t,i]) at the selected
//             experts of dlogits[t, :], 0 elsewhere; dbias = the column sums of
//             dlogits, in a fixed order (no atomics)
//   permute:  the combine with unit weights (permute_combine.cu)
#include "moe_common.cuh"

namespace moe {

constexpr int kBwdThreads = 128;

__device__ __forceinline__ void unpack_vec(const uint4 &u, bool bf16, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    if (bf16) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            f[2 * q] = __uint_as_float(w[q] << 16);
            f[2 * q + 1] = __uint_as_float(w[q] & 0xFFFF0000u);
        }
    } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) f[q] = __uint_as_float(w[q]);
    }
}

__device__ __forceinline__ uint4 pack_vec(const float (&f)[8], bool bf16) {
    uint4 o;
    if (bf16) {
        auto p2 = [](float lo, float hi) {
            return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo)) |
                   ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi)) << 16);
        };
        o.x = p2(f[0], f[1]);
        o.y = p2(f[2], f[3]);
        o.z = p2(f[4], f[5]);
        o.w = p2(f[6], f[7]);
    } else {
        o.x = __float_as_uint(f[0]);
        o.y = __float_as_uint(f[1]);
        o.z = __float_as_uint(f[2]);
        o.w = __float_as_uint(f[3]);
    }
    return o;
}

// One CTA per token of the chunk.  Each thread takes 16-byte columns of dout[t];
// for every kept slot it writes w * dout to the slot's receive row and adds its
// share of <dout[t], y[p]>; the shares are reduced over the CTA at the end.
template <bool BF16>
__global__ void __launch_bounds__(kBwdThreads) combine_bwd_kernel(
    int tb, int k, int row_vecs, const uint4 *__restrict__ dout, const uint4 *__restrict__ y,
    const int32_t *__restrict__ pos, const float *__restrict__ topk_w, uint4 *__restrict__ dy,
    float *__restrict__ dw) {
    constexpr int kVE = BF16 ? 8 : 4;          // values per 16-byte vector
    __shared__ int32_t s_pos[kMaxTopK];
    __shared__ float s_w[kMaxTopK];
    __shared__ float s_part[kBwdThreads / 32][kMaxTopK];
    const int i = blockIdx.x, t = tb + i;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x < k) {
        s_pos[threadIdx.x] = pos[(size_t)i * k + threadIdx.x];
        s_w[threadIdx.x] = topk_w[(size_t)t * k + threadIdx.x];
    }
    __syncthreads();
    float dot[kMaxTopK];
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) dot[j] = 0.0f;
    for (int v = threadIdx.x; v < row_vecs; v += kBwdThreads) {
        float d[8];
        unpack_vec(dout[(size_t)t * row_vecs + v], BF16, d);
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j) {
            if (j < k && s_pos[j] >= 0) {
                const size_t p = (size_t)s_pos[j];
                float yf[8], o[8];
                unpack_vec(y[p * row_vecs + v], BF16, yf);
                float acc = 0.0f;
#pragma unroll
                for (int e = 0; e < kVE; ++e) {
                    acc = __fmaf_rn(d[e], yf[e], acc);
                    o[e] = s_w[j] * d[e];
                }
                dot[j] += acc;
                dy[p * row_vecs + v] = pack_vec(o, BF16);
            }
        }
    }
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
        if (j < k) {                            // k is uniform: every lane shuffles
            float s = dot[j];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
            if (lane == 0) s_part[warp][j] = s;
        }
    }
    __syncthreads();
    if (threadIdx.x < k) {
        float s = 0.0f;
#pragma unroll
        for (int w = 0; w < kBwdThreads / 32; ++w) s += s_part[w][threadIdx.x];
        dw[(size_t)t * k + threadIdx.x] = s_pos[threadIdx.x] >= 0 ? s : 0.0f;
    }
}

// One warp per token: lane j < k holds slot j.  The row of dlogits is cleared,
// then each selected expert gets its slot's dz (experts of a token are distinct).
__global__ void __launch_bounds__(256) route_bwd_kernel(int T, int E, int k,
                                                        const int32_t *__restrict__ topk_idx,
                                                        const float *__restrict__ topk_w,
                                                        const float *__restrict__ dw,
                                                        float *__restrict__ dlogits,
                                                        uint32_t *__restrict__ status) {
    const int t = (int)(((size_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5);
    const int lane = threadIdx.x & 31;
    if (t >= T) return;                         // whole warps
    float w = 0.0f, d = 0.0f;
    int e = -1;
    if (lane < k) {
        w = topk_w[(size_t)t * k + lane];
        d = dw[(size_t)t * k + lane];
        e = topk_idx[(size_t)t * k + lane];
    }
    float sw = w * d;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sw += __shfl_xor_sync(0xffffffffu, sw, off);
    float *row = dlogits + (size_t)t * E;
    for (int c = lane; c < E; c += 32) row[c] = 0.0f;
    __syncwarp();
    if (lane < k) {
        if (e >= 0 && e < E) row[e] = w * (d - sw);
        else raise_status(status, MOE_DEV_BAD_INDEX);
    }
}

// dbias[e] = sum over t of dlogits[t, e]: 8 warps per 32 experts, each warp a
// fixed stride of tokens, then the 8 partial sums in warp order.
__global__ void __launch_bounds__(256) column_sum_kernel(int T, int E, const float *__restrict__ dlogits,
                                                         float *__restrict__ dbias) {
    __shared__ float s[8][32];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int e = blockIdx.x * 32 + lane;
    float acc = 0.0f;
    if (e < E)
        for (int t = w; t < T; t += 8) acc += dlogits[(size_t)t * E + e];
    s[w][lane] = acc;
    __syncthreads();
    if (w == 0 && e < E) {
        float tot = 0.0f;
#pragma unroll
        for (int q = 0; q < 8; ++q) tot += s[q][lane];
        dbias[e] = tot;
    }
}

cudaError_t launch_combine_bwd(const moe_config &c, const void *dout, const void *y,
                               const int32_t *pos, const float *topk_w, int tb, int tc, void *dy,
                               float *dw, cudaStream_t s) {
    if (tc == 0) return cudaSuccess;
    const bool bf16 = c.dtype == MOE_BF16;
    const int row_vecs = c.H / (bf16 ? 8 : 4);
    if (bf16)
        combine_bwd_kernel<true><<<tc, kBwdThreads, 0, s>>>(
            tb, c.k, row_vecs, static_cast<const uint4 *>(dout), static_cast<const uint4 *>(y), pos,
            topk_w, static_cast<uint4 *>(dy), dw);
    else
        combine_bwd_kernel<false><<<tc, kBwdThreads, 0, s>>>(
            tb, c.k, row_vecs, static_cast<const uint4 *>(dout), static_cast<const uint4 *>(y), pos,
            topk_w, static_cast<uint4 *>(dy), dw);
    return cudaGetLastError();
}

cudaError_t launch_route_bwd(const moe_config &c, const int32_t *topk_idx, const float *topk_w,
                             const float *dw, float *dlogits, float *dbias, uint32_t *status,
                             cudaStream_t s) {
    if (c.T == 0) return cudaSuccess;
    const int warps_per_block = 256 / 32;
    const int blocks = (c.T + warps_per_block - 1) / warps_per_block;
    route_bwd_kernel<<<blocks, 256, 0, s>>>(c.T, c.E, c.k, topk_idx, topk_w, dw, dlogits, status);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess || !dbias) return err;
    if (c.bias_select_only)       // the bias steers the selection only: no gradient reaches it
        return cudaMemsetAsync(dbias, 0, sizeof(float) * (size_t)c.E, s);
    column_sum_kernel<<<(c.E + 31) / 32, 256, 0, s>>>(c.T, c.E, dlogits, dbias);
    return cudaGetLastError();
}

}  // namespace moe
