// Step 5 (fp32): grouped SwiGLU expert FFN with fp32 FMA on the CUDA cores.
// The fp32 layer keeps fp32 end to end; tf32 tensor-core inputs (10-bit
// mantissa) would miss a 1e-4 absolute error budget at |y| ~ 1, so this
// dtype does not use the tensor cores.
//
// One CTA per receive row p (rows >= N exit at once).  The CTA keeps the row
// in shared memory; each warp computes whole dot products with lane-strided,
// coalesced weight reads and a shuffle reduction.
#include "moe_common.cuh"

namespace moe {

constexpr int kSimtThreads = 256;

__device__ __forceinline__ int expert_of_row(const int32_t *offs, int E, int p) {
    int lo = 0, hi = E - 1;  // last e with offs[e] <= p
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (offs[mid] <= p) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

__global__ void __launch_bounds__(kSimtThreads) ffn_simt_gemm1_kernel(
    int E, int H, int I, const int32_t *__restrict__ offs, const float *__restrict__ xr,
    const float *__restrict__ w13, float *__restrict__ h) {
    extern __shared__ float s_row[];  // [H]
    const int p = blockIdx.x;
    if (p >= offs[E]) return;
    const int e = expert_of_row(offs, E, p);
    for (int c = threadIdx.x; c < H; c += blockDim.x) s_row[c] = xr[(size_t)p * H + c];
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const float *wg = w13 + (size_t)e * 2 * I * H;
    for (int i = warp; i < I; i += nw) {
        const float *rg = wg + (size_t)i * H;
        const float *ru = wg + (size_t)(I + i) * H;
        float g = 0.f, u = 0.f;
        for (int c = lane; c < H; c += 32) {
            g = __fmaf_rn(__ldg(rg + c), s_row[c], g);
            u = __fmaf_rn(__ldg(ru + c), s_row[c], u);
        }
        g = warp_sum(g);
        u = warp_sum(u);
        if (lane == 0) h[(size_t)p * I + i] = g / (1.0f + expf(-g)) * u;
    }
}

__global__ void __launch_bounds__(kSimtThreads) ffn_simt_gemm2_kernel(
    int E, int H, int I, int k, const int32_t *__restrict__ offs, const float *__restrict__ h,
    const float *__restrict__ w2, float *__restrict__ y, const int32_t *__restrict__ recv_token,
    const int32_t *__restrict__ recv_slot, const float *__restrict__ topk_w,
    float *__restrict__ out_reduce) {
    extern __shared__ float s_row[];  // [I]
    const int p = blockIdx.x;
    if (p >= offs[E]) return;
    const int e = expert_of_row(offs, E, p);
    for (int c = threadIdx.x; c < I; c += blockDim.x) s_row[c] = h[(size_t)p * I + c];
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const float *we = w2 + (size_t)e * H * I;
    int t = 0;
    float w = 0.f;
    if (out_reduce) {
        t = recv_token[p];
        w = topk_w[(size_t)t * k + recv_slot[p]];
    }
    for (int o = warp; o < H; o += nw) {
        const float *r = we + (size_t)o * I;
        float acc = 0.f;
        for (int c = lane; c < I; c += 32) acc = __fmaf_rn(__ldg(r + c), s_row[c], acc);
        acc = warp_sum(acc);
        if (lane == 0) {
            if (out_reduce) atomicAdd(out_reduce + (size_t)t * H + o, w * acc);
            else y[(size_t)p * H + o] = acc;
        }
    }
}

cudaError_t launch_ffn_simt(const moe_config &c, int64_t n_rows, const void *xr,
                            const int32_t *expert_offsets, const void *w13, const void *w2,
                            void *h, void *y, const int32_t *recv_token, const int32_t *recv_slot,
                            const float *topk_w, float *out_reduce, cudaStream_t s) {
    if (n_rows <= 0) return cudaSuccess;
    if (n_rows > 0x7fffffffLL) return cudaErrorInvalidValue;
    ffn_simt_gemm1_kernel<<<(int)n_rows, kSimtThreads, sizeof(float) * c.H, s>>>(
        c.E, c.H, c.I, expert_offsets, static_cast<const float *>(xr),
        static_cast<const float *>(w13), static_cast<float *>(h));
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    ffn_simt_gemm2_kernel<<<(int)n_rows, kSimtThreads, sizeof(float) * c.I, s>>>(
        c.E, c.H, c.I, c.k, expert_offsets, static_cast<const float *>(h),
        static_cast<const float *>(w2), static_cast<float *>(y), recv_token, recv_slot, topk_w,
        c.reduce_dense ? out_reduce : nullptr);
    return cudaGetLastError();
}

}  // namespace moe
