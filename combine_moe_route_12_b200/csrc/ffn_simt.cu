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

// ------------------------------------------------------------------ backward (fp32)
// The same backward as the tcgen05 path (gate / up recomputed, dh, the SwiGLU
// backward, dxr, the weight gradients), in fp32 FMA.  One CTA per receive row
// for the data gradients; one CTA per (expert, output row) for the weights.

// g, u of the row (warp per feature, coalesced W13 rows), then per feature
// (thread per feature, coalesced W2 reads across features) dh = W2[:, i] . dy,
// h = silu(g) u, dg = dh u s (1 + g (1 - s)), du = dh silu(g).
__global__ void __launch_bounds__(kSimtThreads) ffn_simt_bwd_rows_kernel(
    int E, int H, int I, const int32_t *__restrict__ offs, const float *__restrict__ xr,
    const float *__restrict__ dy, const float *__restrict__ w13, const float *__restrict__ w2,
    float *__restrict__ h, float *__restrict__ dgu) {
    extern __shared__ float sm[];   // x [H], dy [H], g [I], u [I]
    float *s_x = sm, *s_dy = sm + H, *s_g = sm + 2 * H, *s_u = s_g + I;
    const int p = blockIdx.x;
    if (p >= offs[E]) return;
    const int e = expert_of_row(offs, E, p);
    for (int c = threadIdx.x; c < H; c += blockDim.x) {
        s_x[c] = xr[(size_t)p * H + c];
        s_dy[c] = dy[(size_t)p * H + c];
    }
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const float *wg = w13 + (size_t)e * 2 * I * H;
    for (int i = warp; i < I; i += nw) {
        const float *rg = wg + (size_t)i * H;
        const float *ru = wg + (size_t)(I + i) * H;
        float g = 0.f, u = 0.f;
        for (int c = lane; c < H; c += 32) {
            g = __fmaf_rn(__ldg(rg + c), s_x[c], g);
            u = __fmaf_rn(__ldg(ru + c), s_x[c], u);
        }
        g = warp_sum(g);
        u = warp_sum(u);
        if (lane == 0) { s_g[i] = g; s_u[i] = u; }
    }
    __syncthreads();
    const float *we = w2 + (size_t)e * H * I;
    for (int i = threadIdx.x; i < I; i += blockDim.x) {
        float dh = 0.f;
        for (int o = 0; o < H; ++o) dh = __fmaf_rn(__ldg(we + (size_t)o * I + i), s_dy[o], dh);
        const float g = s_g[i], u = s_u[i];
        const float sg = 1.0f / (1.0f + expf(-g));
        h[(size_t)p * I + i] = g * sg * u;
        dgu[(size_t)p * 2 * I + i] = dh * u * sg * (1.0f + g * (1.0f - sg));
        dgu[(size_t)p * 2 * I + I + i] = dh * g * sg;
    }
}

// dxr[p, c] = sum over j < 2I of W13[e][j, c] * dgu[p, j] (thread per c, coalesced)
__global__ void __launch_bounds__(kSimtThreads) ffn_simt_bwd_dx_kernel(
    int E, int H, int I, const int32_t *__restrict__ offs, const float *__restrict__ dgu,
    const float *__restrict__ w13, float *__restrict__ dxr) {
    extern __shared__ float s_d[];  // [2I]
    const int p = blockIdx.x;
    if (p >= offs[E]) return;
    const int e = expert_of_row(offs, E, p);
    for (int j = threadIdx.x; j < 2 * I; j += blockDim.x) s_d[j] = dgu[(size_t)p * 2 * I + j];
    __syncthreads();
    const float *we = w13 + (size_t)e * 2 * I * H;
    for (int c = threadIdx.x; c < H; c += blockDim.x) {
        float acc = 0.f;
        for (int j = 0; j < 2 * I; ++j) acc = __fmaf_rn(__ldg(we + (size_t)j * H + c), s_d[j], acc);
        dxr[(size_t)p * H + c] = acc;
    }
}

// out[e][m, n] (+)= sum over the expert's rows p of a[p, m] * b[p, n], over
// n_seg segments seg_rows rows apart (segment s: offsets offs + s * (E + 1))
__global__ void __launch_bounds__(kSimtThreads) ffn_simt_wgrad_kernel(
    int E, int M, int N, int n_seg, long long seg_rows, const int32_t *__restrict__ offs,
    const float *__restrict__ a, const float *__restrict__ b, float *__restrict__ out, int accumulate) {
    const int m = blockIdx.x, e = blockIdx.y;
    float *o = out + ((size_t)e * M + m) * N;
    for (int n = threadIdx.x; n < N; n += blockDim.x) {
        float acc = 0.f;
        for (int sg = 0; sg < n_seg; ++sg) {
            const int32_t *os = offs + (size_t)sg * (E + 1);
            const size_t base = (size_t)sg * seg_rows;
            for (int p = os[e]; p < os[e + 1]; ++p)
                acc = __fmaf_rn(a[(base + p) * M + m], b[(base + p) * N + n], acc);
        }
        o[n] = accumulate ? o[n] + acc : acc;
    }
}

cudaError_t launch_ffn_simt_wgrad(const moe_config &c, int n_seg, int64_t seg_rows,
                                  const int32_t *expert_offsets, const void *xr, const void *dy,
                                  const void *h, const void *dgu, float *dw13, float *dw2,
                                  int accumulate, cudaStream_t s) {
    ffn_simt_wgrad_kernel<<<dim3(c.H, c.E), kSimtThreads, 0, s>>>(
        c.E, c.H, c.I, n_seg, seg_rows, expert_offsets, static_cast<const float *>(dy),
        static_cast<const float *>(h), dw2, accumulate);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    ffn_simt_wgrad_kernel<<<dim3(2 * c.I, c.E), kSimtThreads, 0, s>>>(
        c.E, 2 * c.I, c.H, n_seg, seg_rows, expert_offsets, static_cast<const float *>(dgu),
        static_cast<const float *>(xr), dw13, accumulate);
    return cudaGetLastError();
}

cudaError_t launch_ffn_simt_dgrad(const moe_config &c, int64_t n_rows, const void *xr, const void *dy,
                                  const int32_t *expert_offsets, const void *w13, const void *w2,
                                  void *h, void *dgu, void *dxr, cudaStream_t s) {
    if (n_rows > 0x7fffffffLL) return cudaErrorInvalidValue;
    const float *x = static_cast<const float *>(xr), *d = static_cast<const float *>(dy);
    if (n_rows > 0) {
        ffn_simt_bwd_rows_kernel<<<(int)n_rows, kSimtThreads, sizeof(float) * (2 * (size_t)c.H + 2 * c.I), s>>>(
            c.E, c.H, c.I, expert_offsets, x, d, static_cast<const float *>(w13),
            static_cast<const float *>(w2), static_cast<float *>(h), static_cast<float *>(dgu));
        cudaError_t err = cudaGetLastError();
        if (err != cudaSuccess) return err;
        ffn_simt_bwd_dx_kernel<<<(int)n_rows, kSimtThreads, sizeof(float) * 2 * (size_t)c.I, s>>>(
            c.E, c.H, c.I, expert_offsets, static_cast<const float *>(dgu),
            static_cast<const float *>(w13), static_cast<float *>(dxr));
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
    }
    return cudaSuccess;
}

cudaError_t launch_ffn_simt_bwd(const moe_config &c, int64_t n_rows, const void *xr, const void *dy,
                                const int32_t *expert_offsets, const void *w13, const void *w2,
                                void *h, void *dgu, void *dxr, float *dw13, float *dw2,
                                int accumulate, cudaStream_t s) {
    cudaError_t err = launch_ffn_simt_dgrad(c, n_rows, xr, dy, expert_offsets, w13, w2, h, dgu, dxr, s);
    if (err != cudaSuccess) return err;
    // the weight gradients run whatever n_rows is: experts without rows get zeros
    return launch_ffn_simt_wgrad(c, 1, n_rows, expert_offsets, xr, dy, h, dgu, dw13, dw2, accumulate, s);
}

}  // namespace moe
