// Scheduling pieces shared by the CTA-pair grouped FFN kernels (bf16 / FP8 with
// row scales, and FP8 with K-blocked scales): the tile numbering, the slice
// queue through which the leader's producer publishes tiles to every role of
// both CTAs, and small epilogue helpers.
#pragma once

#include "moe_common.cuh"

namespace moe {

constexpr int kQueue = 8;   // slices published ahead of the slowest consumer

// Work is dealt out tile by tile from a global counter, so a pair that finishes
// early takes more.  Tiles are numbered expert by expert, weight slice (expert,
// pair feature block) by weight slice, token block innermost: the tiles of one
// slice are taken back to back and stream the same weights at the same time.
// s_tpre[e]: the first tile of expert e; s_tb[e]: its token blocks.
__device__ __forceinline__ void decode_tile(int tile, const int32_t *s_tpre, const int32_t *s_tb,
                                            int E, int &e, int &f_blk, int &t_blk) {
    int lo = 0, hi = E - 1;  // last e with s_tpre[e] <= tile (it owns >= 1 tile)
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_tpre[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    e = lo;
    const int local = tile - s_tpre[lo];
    f_blk = local / s_tb[lo];
    t_blk = local - f_blk * s_tb[lo];
}

// silu in the epilogues: the fast exponential and reciprocal-based divide (a
// few ulp in fp32) are far inside the bf16 rounding of h, and the IEEE divide
// made the epilogue instruction-bound.  For g -> -inf the quotient is -0.
__device__ __forceinline__ float silu_f(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

__device__ __forceinline__ void named_barrier_sync(uint32_t id, uint32_t nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// One consumer's position in the slice queue (q_full / q_slice in every CTA,
// q_empty in the leader's).  next() waits (bounded) for the next published
// slice, reads it and releases the entry on the leader's q_empty; it returns
// false on a timeout.  A slice of -1 ends the work.
struct SliceReader {
    int qi = 0;
    uint32_t qph = 0;
    template <class Smem>
    __device__ __forceinline__ bool next(Smem *S, volatile int *abort_flag, bool release, int &slice) {
        if (!mbar_wait_cluster_bounded(&S->q_full[qi], qph, abort_flag)) return false;
        slice = *reinterpret_cast<volatile int *>(&S->q_slice[qi]);
        if (release) mbar_arrive_cluster(mapa_shared(smem_u32(&S->q_empty[qi]), 0));
        if (++qi == kQueue) { qi = 0; qph ^= 1u; }
        return true;
    }
};

}  // namespace moe
