// C ABI of the MoE hot path: argument and topology checks, workspace carving,
// launches, and the two-stream chunked forward.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <vector>

#include "moe_common.cuh"

namespace moe {
cudaError_t launch_route_topk(const moe_config &c, const float *logits, const float *bias,
                              int32_t *topk_idx, float *topk_w, int32_t *counts,
                              uint32_t *status, cudaStream_t s, int num_sms);
cudaError_t launch_capacity_clip(const moe_config &c, const int32_t *topk_idx,
                                 const float *topk_w, const int32_t *counts, uint8_t *keep,
                                 int32_t *kept_counts, uint64_t *thr, int32_t *seg, uint64_t *keys,
                                 uint32_t *status, cudaStream_t s, int num_sms);
cudaError_t launch_dispatch_layout(const moe_config &c, int tb, int tc,
                                   const int32_t *topk_idx, const uint8_t *keep,
                                   int32_t *expert_offsets, int32_t *rank_offsets,
                                   int32_t *recv_token, int32_t *recv_slot, int32_t *pos,
                                   int32_t *send_splits, int32_t *splits_host, void *ws,
                                   int64_t n_rows_max, cudaStream_t s, int num_sms);
cudaError_t launch_permute(const moe_config &c, const void *x, const int32_t *pos, int tb,
                           int tc, void *xr, cudaStream_t s);
cudaError_t launch_combine(const moe_config &c, const void *y, const int32_t *pos,
                           const float *topk_w, int tb, int tc, const void *y_shared, void *out,
                           cudaStream_t s);
cudaError_t launch_reduce_finalize(const moe_config &c, const float *red, int tb, int tc,
                                   const void *y_shared, void *out, cudaStream_t s, int num_sms);
cudaError_t launch_shared_offsets(int32_t *off, int rows, cudaStream_t s);
cudaError_t launch_ffn_tcgen05(const moe_config &c, int64_t n_rows, const void *xr,
                               const int32_t *expert_offsets, const void *w13, const void *w2,
                               void *h, void *y, const int32_t *recv_token,
                               const int32_t *recv_slot, const float *topk_w, float *out_reduce,
                               uint32_t *status, uint32_t *counters, cudaStream_t s, int num_sms);
cudaError_t launch_ffn_tcgen05_fp8(const moe_config &c, int64_t n_rows, const uint8_t *xr_q,
                                   const uint8_t *x_scale, const int32_t *expert_offsets,
                                   const uint8_t *w13_q, const uint8_t *w13_scale,
                                   const uint8_t *w2_q, const uint8_t *w2_scale, void *h,
                                   uint8_t *h_q, uint8_t *h_scale, void *y,
                                   const int32_t *recv_token, const int32_t *recv_slot,
                                   const float *topk_w, float *out_reduce, uint32_t *status,
                                   uint32_t *counters, cudaStream_t s, int num_sms);
cudaError_t launch_quant_rows(int64_t rows, int cols, bool bf16, const void *in, uint8_t *codes,
                              uint8_t *scales, const int32_t *n_dev, cudaStream_t s, int num_sms);
cudaError_t launch_permute_quant(const moe_config &c, const void *x, const int32_t *pos, int tb,
                                 int tc, uint8_t *xr_q, uint8_t *x_scale, cudaStream_t s);
cudaError_t launch_quant_blocks(int64_t rows, int cols, bool bf16, const void *in, uint8_t *codes,
                                uint8_t *scales, cudaStream_t s, int num_sms);
cudaError_t launch_permute_quant_blocks(const moe_config &c, const void *x, const int32_t *pos, int tb,
                                        int tc, uint8_t *xr_q, uint8_t *xr_sf, cudaStream_t s);
cudaError_t launch_ffn_mx(const moe_config &c, int64_t n_rows, const uint8_t *xr_q, const uint8_t *xr_sf,
                          const int32_t *expert_offsets, const uint8_t *w13_q, const uint8_t *w13_sf,
                          const uint8_t *w2_q, const uint8_t *w2_sf, uint8_t *h_q, uint8_t *h_sf, void *y,
                          const int32_t *recv_token, const int32_t *recv_slot, const float *topk_w,
                          float *out_reduce, uint32_t *status, uint32_t *counters, cudaStream_t s,
                          int num_sms);
cudaError_t launch_ep_regroup(int n_src, int n_exp, const int32_t *counts, const void *in, void *out,
                              int64_t rows, int row_bytes, int inverse, int32_t *expert_offsets, uint32_t *status,
                              cudaStream_t s, int num_sms);
cudaError_t launch_combine_bwd(const moe_config &c, const void *dout, const void *y,
                               const int32_t *pos, const float *topk_w, int tb, int tc, void *dy,
                               float *dw, cudaStream_t s);
cudaError_t launch_route_bwd(const moe_config &c, const int32_t *topk_idx, const float *topk_w,
                             const float *dw, float *dlogits, float *dbias, uint32_t *status,
                             cudaStream_t s);
cudaError_t launch_ffn_tcgen05_bwd(const moe_config &c, int64_t n_rows, const void *xr, const void *dy,
                                   const int32_t *expert_offsets, const void *w13, const void *w2,
                                   void *gu, void *h, void *dgu, void *dxr, float *dw13, float *dw2,
                                   int accumulate, uint32_t *status, uint32_t *counters,
                                   cudaStream_t s, int num_sms);
cudaError_t launch_ffn_simt_bwd(const moe_config &c, int64_t n_rows, const void *xr, const void *dy,
                                const int32_t *expert_offsets, const void *w13, const void *w2,
                                void *h, void *dgu, void *dxr, float *dw13, float *dw2,
                                int accumulate, cudaStream_t s);
cudaError_t launch_ffn_tcgen05_dgrad(const moe_config &c, int64_t n_rows, const void *xr, const void *dy,
                                     const int32_t *expert_offsets, const void *w13, const void *w2,
                                     void *gu, void *h, void *dgu, void *dxr, uint32_t *status,
                                     uint32_t *counters, cudaStream_t s, int num_sms);
cudaError_t launch_ffn_tcgen05_wgrad(const moe_config &c, int n_seg, int64_t seg_rows,
                                     const int32_t *expert_offsets, const void *xr, const void *dy,
                                     const void *h, const void *dgu, float *dw13, float *dw2,
                                     int accumulate, uint32_t *status, cudaStream_t s, int num_sms);
cudaError_t launch_ffn_simt_dgrad(const moe_config &c, int64_t n_rows, const void *xr, const void *dy,
                                  const int32_t *expert_offsets, const void *w13, const void *w2,
                                  void *h, void *dgu, void *dxr, cudaStream_t s);
cudaError_t launch_ffn_simt_wgrad(const moe_config &c, int n_seg, int64_t seg_rows,
                                  const int32_t *expert_offsets, const void *xr, const void *dy,
                                  const void *h, const void *dgu, float *dw13, float *dw2,
                                  int accumulate, cudaStream_t s);
cudaError_t launch_ffn_simt(const moe_config &c, int64_t n_rows, const void *xr,
                            const int32_t *expert_offsets, const void *w13, const void *w2,
                            void *h, void *y, const int32_t *recv_token, const int32_t *recv_slot,
                            const float *topk_w, float *out_reduce, cudaStream_t s);
}  // namespace moe

using namespace moe;

namespace {

thread_local char g_detail[512] = "";

moe_status fail(moe_status st, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_detail, sizeof g_detail, fmt, ap);
    va_end(ap);
    return st;
}

moe_status cuda_fail(cudaError_t err, const char *where) {
    return fail(MOE_ERR_CUDA, "%s: %s", where, cudaGetErrorString(err));
}

int current_num_sms() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int64_t max_rows(const moe_config &c, int32_t tc) {
    int64_t n = (int64_t)tc * c.k;
    if (c.capacity >= 0) {
        const int64_t cap = (int64_t)c.E * c.capacity;
        if (cap < n) n = cap;
    }
    return n;
}

moe_status check_ws(void *ws) {
    if (!ws) return fail(MOE_ERR_WORKSPACE, "workspace is NULL");
    if (!aligned(ws, 256)) return fail(MOE_ERR_WORKSPACE, "workspace not 256-byte aligned");
    return MOE_OK;
}

moe_status check_range(const moe_config &c, int32_t tb, int32_t tc, bool need_ep) {
    if (tb < 0 || tc < 0 || (int64_t)tb + tc > c.T)
        return fail(MOE_ERR_INVALID_ARG, "token range [%d, %d+%d) outside [0, %d)", tb, tb, tc, c.T);
    if (need_ep && tc % c.ep != 0)
        return fail(MOE_ERR_INVALID_ARG, "tok_count %d not divisible by ep %d", tc, c.ep);
    return MOE_OK;
}

// The forward's FP8 path quantises x inside the permute for rows of up to 8192
// values; longer rows take a separate quantisation pass through x's codes.
bool fused_permute_quant(const moe_config &c) { return c.H <= 8192; }

// Forward workspace: scratch first, then saved counts, two chunk slots, and
// the dense fp32 reduce buffer (decode form).
struct Slot {
    size_t eoff, roff, recv_token, recv_slot, pos, splits, xr, h, y;
    size_t hs, ys;   // the shared expert's h and y for the chunk's rows (shared_I > 0)
    size_t hq, hsc;  // ffn_fp8: h's E4M3 codes and scales (one per row, or per 32 values: [nmax, I/32])
    size_t xsf;      // ffn_fp8 = 2: the receive rows' scales [nmax, H/32]
};
struct ForwardLayout {
    size_t counts, kept_counts;
    size_t xq, xsc;  // ffn_fp8: x's E4M3 codes [T, H] and row scales [T]
    Slot slot[2];
    size_t out_reduce;
    // device staging of the host-buffer entry point's activations (host_io only)
    size_t stage_logits, stage_bias, stage_x, stage_out;
    size_t total;
    int64_t nmax;
    int tc;
};

ForwardLayout forward_layout(const moe_config &c, bool host_io = false) {
    ForwardLayout F{};
    const ScratchLayout L = scratch_layout(c);
    size_t off = L.total;
    auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes, 256); return o; };
    F.tc = c.T / c.n_chunks;
    F.nmax = max_rows(c, F.tc);
    const size_t eb = c.dtype == MOE_F32 ? 4 : 2;
    F.counts = take(sizeof(int32_t) * c.E);
    F.kept_counts = take(sizeof(int32_t) * c.E);
    const int nslots = c.n_chunks > 1 ? 2 : 1;
    for (int s = 0; s < 2; ++s) {
        if (s >= nslots) { F.slot[s] = F.slot[0]; continue; }
        Slot &S = F.slot[s];
        S.eoff = take(sizeof(int32_t) * (c.E + 1));
        S.roff = take(sizeof(int32_t) * (c.ep + 1));
        S.recv_token = take(sizeof(int32_t) * (size_t)(F.nmax > 0 ? F.nmax : 1));
        S.recv_slot = take(sizeof(int32_t) * (size_t)(F.nmax > 0 ? F.nmax : 1));
        S.pos = take(sizeof(int32_t) * (size_t)F.tc * c.k);
        S.splits = take(sizeof(int32_t) * (size_t)c.ep * c.ep);
        S.xr = take((c.ffn_fp8 ? 1 : eb) * (size_t)F.nmax * c.H);   // codes when ffn_fp8
        S.h = take(eb * (size_t)F.nmax * c.I);
        S.y = c.reduce_dense ? 0 : take(eb * (size_t)F.nmax * c.H);
        S.hs = c.shared_I > 0 ? take(eb * (size_t)F.tc * c.shared_I) : 0;
        S.ys = c.shared_I > 0 ? take(eb * (size_t)F.tc * c.H) : 0;
        S.hq = c.ffn_fp8 ? take((size_t)(F.nmax > 0 ? F.nmax : 1) * c.I) : 0;
        S.hsc = c.ffn_fp8 ? take((size_t)(F.nmax > 0 ? F.nmax : 1) * (c.ffn_fp8 == 2 ? c.I / 32 : 1)) : 0;
        S.xsf = c.ffn_fp8 == 2 ? take((size_t)(F.nmax > 0 ? F.nmax : 1) * (c.H / 32)) : 0;
    }
    F.xq = c.ffn_fp8 == 1 && !fused_permute_quant(c) ? take((size_t)c.T * c.H) : 0;
    F.xsc = c.ffn_fp8 == 1 ? take((size_t)c.T) : 0;
    F.out_reduce = c.reduce_dense ? take(sizeof(float) * (size_t)c.T * c.H) : 0;
    if (host_io) {
        F.stage_logits = take(sizeof(float) * (size_t)c.T * c.E);
        F.stage_bias = take(sizeof(float) * (size_t)c.E);
        F.stage_x = take(eb * (size_t)c.T * c.H);
        F.stage_out = take(eb * (size_t)c.T * c.H);
    }
    F.total = off;
    return F;
}

// Backward workspace: scratch first; the rows the weight gradients read for
// every chunk (receive rows when recomputed, dy, h, dg | du; chunk c's at rows
// c * nmax), each chunk's expert offsets, one chunk slot of what is consumed
// within the chunk, and the fp32 slot gradients of all T tokens.  With a shared
// expert, its h and dg | du rows for all T tokens and a chunk slot of the rest.
struct BackwardLayout {
    size_t eoff;                          // int32 [n_chunks][E + 1]
    size_t roff, recv_token, recv_slot, pos, splits;
    size_t xr, h, dy, dgu;                // [n_chunks * nmax, .]
    size_t y, gu, dxr;                    // [nmax, .]
    size_t dw;                            // fp32 [T, k]
    size_t hs, dgus;                      // [T, .]
    size_t gus, dxs;                      // [tc, .]
    size_t total;
    int64_t nmax;
    int tc;
};

BackwardLayout backward_layout(const moe_config &c) {
    BackwardLayout B{};
    const ScratchLayout L = scratch_layout(c);
    size_t off = L.total;
    auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + (bytes ? bytes : 1), 256); return o; };
    B.tc = c.T / c.n_chunks;
    B.nmax = max_rows(c, B.tc);
    const size_t eb = c.dtype == MOE_F32 ? 4 : 2;
    const size_t n = (size_t)(B.nmax > 0 ? B.nmax : 1), nall = n * c.n_chunks;
    B.eoff = take(sizeof(int32_t) * (size_t)c.n_chunks * (c.E + 1));
    B.roff = take(sizeof(int32_t) * (c.ep + 1));
    B.recv_token = take(sizeof(int32_t) * n);
    B.recv_slot = take(sizeof(int32_t) * n);
    B.pos = take(sizeof(int32_t) * (size_t)B.tc * c.k);
    B.splits = take(sizeof(int32_t) * (size_t)c.ep * c.ep);
    B.xr = take(eb * nall * c.H);
    B.h = take(eb * nall * c.I);
    B.dy = take(eb * nall * c.H);
    B.dgu = take(eb * nall * 2 * c.I);
    B.y = take(eb * n * c.H);
    B.gu = take(eb * n * 2 * c.I);
    B.dxr = take(eb * n * c.H);
    B.dw = take(sizeof(float) * (size_t)c.T * c.k);
    if (c.shared_I > 0) {
        B.hs = take(eb * (size_t)c.T * c.shared_I);
        B.dgus = take(eb * (size_t)c.T * 2 * c.shared_I);
        B.gus = take(eb * (size_t)B.tc * 2 * c.shared_I);
        B.dxs = take(eb * (size_t)B.tc * c.H);
    }
    B.total = off;
    return B;
}

// Per-thread, per-device pool of timing-free events for the chunked forward,
// keyed by the device index and refilled when the device's context changed
// (events of a context that a device reset destroyed are gone with it).
struct EventPool {
    unsigned long long ctx = 0;
    std::vector<cudaEvent_t> ev;
};
thread_local std::map<int, EventPool> g_events;

cudaError_t get_events(int n, cudaEvent_t **out) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    EventPool &P = g_events[dev];
    const unsigned long long ctx = current_context_id();
    if (ctx != 0 && P.ctx != ctx) {
        if (P.ctx != 0) P.ev.clear();   // their context is gone: nothing to destroy
        P.ctx = ctx;
    }
    while ((int)P.ev.size() < n) {
        cudaEvent_t e;
        if ((err = cudaEventCreateWithFlags(&e, cudaEventDisableTiming)) != cudaSuccess) return err;
        P.ev.push_back(e);
    }
    *out = P.ev.data();
    return cudaSuccess;
}

}  // namespace

namespace moe {
// Used by entry points defined in other translation units.
moe_status report_error(moe_status st, const char *msg) { return fail(st, "%s", msg); }
int64_t max_recv_rows_of(const moe_config &c, int32_t tok_count) { return max_rows(c, tok_count); }
}  // namespace moe

extern "C" {

moe_status moe_config_check(const moe_config *cfg) {
    if (!cfg) return fail(MOE_ERR_INVALID_ARG, "cfg is NULL");
    const moe_config &c = *cfg;
    if (c.T < 0 || c.H < 1 || c.E < 1 || c.k < 1 || c.I < 1 || c.ep < 1 || c.n_chunks < 1)
        return fail(MOE_ERR_INVALID_ARG, "sizes must be positive (T >= 0)");
    if (c.dtype != MOE_F32 && c.dtype != MOE_BF16)
        return fail(MOE_ERR_INVALID_ARG, "unknown dtype %d", c.dtype);
    if (c.reduce_dense != 0 && c.reduce_dense != 1)
        return fail(MOE_ERR_INVALID_ARG, "reduce_dense must be 0 or 1");
    if (c.k > c.E) return fail(MOE_ERR_INVALID_ARG, "k=%d > E=%d", c.k, c.E);
    if (c.n_group < 0) return fail(MOE_ERR_INVALID_ARG, "n_group=%d < 0", c.n_group);
    if (c.bias_select_only != 0 && c.bias_select_only != 1)
        return fail(MOE_ERR_INVALID_ARG, "bias_select_only must be 0 or 1");
    if (c.shared_I < 0) return fail(MOE_ERR_INVALID_ARG, "shared_I=%d < 0", c.shared_I);
    if (c.ffn_fp8 < 0 || c.ffn_fp8 > 2) return fail(MOE_ERR_INVALID_ARG, "ffn_fp8 must be 0, 1 or 2");
    if (c.ffn_fp8) {
        if (c.dtype != MOE_BF16) return fail(MOE_ERR_UNSUPPORTED, "ffn_fp8 needs dtype MOE_BF16");
        if (c.H % 128 != 0 || c.I % 128 != 0)
            return fail(MOE_ERR_UNSUPPORTED, "ffn_fp8 needs H and I multiples of 128 (H=%d, I=%d)", c.H, c.I);
        if (c.shared_I != 0) return fail(MOE_ERR_UNSUPPORTED, "ffn_fp8 with a shared expert");
        if (c.ffn_fp8 == 2 && (c.E > 512 || c.H > 8192))
            return fail(MOE_ERR_UNSUPPORTED, "ffn_fp8 = 2 (K-blocked scales) needs E <= 512 and H <= 8192 "
                        "(E=%d, H=%d)", c.E, c.H);
    }
    if (c.shared_I > 0 && c.dtype == MOE_BF16 && c.shared_I % 64 != 0)
        return fail(MOE_ERR_UNSUPPORTED, "bf16 needs shared_I a multiple of 64 (got %d)", c.shared_I);
    if (c.shared_I > 0 && c.dtype == MOE_F32 && c.shared_I % 4 != 0)
        return fail(MOE_ERR_UNSUPPORTED, "fp32 needs shared_I a multiple of 4 (got %d)", c.shared_I);
    if (c.n_group > 1) {
        if (c.n_group > kMaxGroups) return fail(MOE_ERR_UNSUPPORTED, "n_group=%d > %d", c.n_group, kMaxGroups);
        if (c.E % c.n_group != 0)
            return fail(MOE_ERR_INVALID_ARG, "E=%d not divisible by n_group=%d", c.E, c.n_group);
        if (c.topk_group < 1 || c.topk_group > c.n_group)
            return fail(MOE_ERR_INVALID_ARG, "topk_group=%d outside [1, n_group=%d]", c.topk_group, c.n_group);
        if (c.k > c.topk_group * (c.E / c.n_group))
            return fail(MOE_ERR_INVALID_ARG, "k=%d > topk_group * E / n_group = %d", c.k,
                        c.topk_group * (c.E / c.n_group));
        if (c.group_score != 0 && c.group_score != 1)
            return fail(MOE_ERR_INVALID_ARG, "group_score must be 0 or 1");
        if (c.group_score == 1 && c.E / c.n_group < 2)
            return fail(MOE_ERR_INVALID_ARG, "group_score 1 needs groups of at least two experts");
    }
    if (c.E % c.ep != 0) return fail(MOE_ERR_INVALID_ARG, "E=%d not divisible by ep=%d", c.E, c.ep);
    if (c.T % c.n_chunks != 0)
        return fail(MOE_ERR_INVALID_ARG, "T=%d not divisible by n_chunks=%d", c.T, c.n_chunks);
    if ((c.T / c.n_chunks) % c.ep != 0)
        return fail(MOE_ERR_INVALID_ARG, "chunk of %d tokens not divisible by ep=%d",
                    c.T / c.n_chunks, c.ep);
    if (c.k > kMaxTopK) return fail(MOE_ERR_UNSUPPORTED, "k=%d > %d", c.k, kMaxTopK);
    if (c.E > kMaxExperts) return fail(MOE_ERR_UNSUPPORTED, "E=%d > %d", c.E, kMaxExperts);
    if ((int64_t)c.T * c.k >= (int64_t)1 << 30) return fail(MOE_ERR_UNSUPPORTED, "T*k >= 2^30");
    if (c.dtype == MOE_BF16 && (c.H % 64 != 0 || c.I % 64 != 0))
        return fail(MOE_ERR_UNSUPPORTED, "bf16 needs H and I multiples of 64 (H=%d, I=%d)", c.H, c.I);
    if (c.dtype == MOE_F32 && (c.H % 4 != 0 || c.I % 4 != 0))
        return fail(MOE_ERR_UNSUPPORTED, "fp32 needs H and I multiples of 4 (H=%d, I=%d)", c.H, c.I);
    return MOE_OK;
}

size_t moe_workspace_bytes(const moe_config *cfg) {
    if (moe_config_check(cfg) != MOE_OK) return 0;
    return scratch_layout(*cfg).total;
}

size_t moe_forward_workspace_bytes(const moe_config *cfg) {
    if (moe_config_check(cfg) != MOE_OK) return 0;
    return forward_layout(*cfg).total;
}

int64_t moe_max_recv_rows(const moe_config *cfg, int32_t tok_count) {
    if (moe_config_check(cfg) != MOE_OK || tok_count < 0) return -1;
    return max_rows(*cfg, tok_count);
}

moe_status moe_route_topk(const moe_config *cfg, const float *logits, const float *bias,
                          int32_t *topk_idx, float *topk_w, int32_t *counts, void *ws,
                          cudaStream_t stream) {
    moe_status st = moe_config_check(cfg);
    if (st != MOE_OK) return st;
    if ((st = check_ws(ws)) != MOE_OK) return st;
    const moe_config &c = *cfg;
    if ((c.T > 0 && (!logits || !topk_idx || !topk_w)) || !counts)
        return fail(MOE_ERR_INVALID_ARG, "NULL pointer argument");
    const ScratchLayout L = scratch_layout(c);
    cudaError_t err = launch_route_topk(c, logits, bias, topk_idx, topk_w, counts,
                                        ws_at<uint32_t>(ws, L.status), stream, current_num_sms());
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_route_topk");
}

moe_status moe_capacity_clip(const moe_config *cfg, const int32_t *topk_idx,
                             const float *topk_w, const int32_t *counts, uint8_t *keep,
                             int32_t *kept_counts, void *ws, cudaStream_t stream) {
    moe_status st = moe_config_check(cfg);
    if (st != MOE_OK) return st;
    if ((st = check_ws(ws)) != MOE_OK) return st;
    const moe_config &c = *cfg;
    if ((c.T > 0 && (!topk_idx || !topk_w || !keep)) || !counts || !kept_counts)
        return fail(MOE_ERR_INVALID_ARG, "NULL pointer argument");
    const ScratchLayout L = scratch_layout(c);
    cudaError_t err = launch_capacity_clip(c, topk_idx, topk_w, counts, keep, kept_counts,
                                           ws_at<uint64_t>(ws, L.clip_thr), ws_at<int32_t>(ws, L.clip_seg),
                                           ws_at<uint64_t>(ws, L.clip_keys),
                                           ws_at<uint32_t>(ws, L.status), stream,
                                           current_num_sms());
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_capacity_clip");
}

moe_status moe_dispatch_layout(const moe_config *cfg, int32_t tok_begin, int32_t tok_count,
                               const int32_t *topk_idx, const uint8_t *keep,
                               int32_t *expert_offsets, int32_t *rank_offsets,
                               int32_t *recv_token, int32_t *recv_slot, int32_t *pos,
                               int32_t *send_splits, int32_t *splits_host, void *ws,
                               cudaStream_t stream) {
    moe_status st = moe_config_check(cfg);
    if (st != MOE_OK) return st;
    if ((st = check_ws(ws)) != MOE_OK) return st;
    const moe_config &c = *cfg;
    if ((st = check_range(c, tok_begin, tok_count, true)) != MOE_OK) return st;
    if (!expert_offsets || !rank_offsets || !send_splits ||
        (tok_count > 0 && (!topk_idx || !keep || !recv_token || !recv_slot || !pos)))
        return fail(MOE_ERR_INVALID_ARG, "NULL pointer argument");
    cudaError_t err = launch_dispatch_layout(c, tok_begin, tok_count, topk_idx, keep,
                                             expert_offsets, rank_offsets, recv_token, recv_slot,
                                             pos, send_splits, splits_host, ws,
                                             max_rows(c, tok_count), stream, current_num_sms());
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_dispatch_layout");
}

moe_status moe_permute(const moe_config *cfg, const void *x, const int32_t *pos,
                       int32_t tok_begin, int32_t tok_count, void *xr, cudaStream_t stream) {
    moe_status st = moe_config_check(cfg);
    if (st != MOE_OK) return st;
    const moe_config &c = *cfg;
    if ((st = check_range(c, tok_begin, tok_count, false)) != MOE_OK) return st;
    if (tok_count > 0 && (!x || !pos || !xr)) return fail(MOE_ERR_INVALID_ARG, "NULL pointer argument");
    if (!aligned(x, 16) || !aligned(xr, 16)) return fail(MOE_ERR_INVALID_ARG, "x / xr not 16-byte aligned");
    cudaError_t err = launch_permute(c, x, pos, tok_begin, tok_count, xr, stream);
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_permute");
}

moe_status moe_grouped_swiglu_ffn(const moe_config *cfg, int64_t n_rows, const void *xr,
                                  const int32_t *expert_offsets, const void *w13,
                                  const void *w2, void *h, void *y, const int32_t *recv_token,
                                  const int32_t *recv_slot, const float *topk_w,
                                  float *out_reduce, void *ws, cudaStream_t stream) {
    moe_status st = moe_config_check(cfg);
    if (st != MOE_OK) return st;
    if ((st = check_ws(ws)) != MOE_OK) return st;
    const moe_config &c = *cfg;
    if (n_rows < 0) return fail(MOE_ERR_INVALID_ARG, "n_rows < 0");
    if (c.ffn_fp8) return fail(MOE_ERR_INVALID_ARG, "cfg->ffn_fp8 = %d: use moe_grouped_swiglu_ffn_%s",
                               c.ffn_fp8, c.ffn_fp8 == 2 ? "mxfp8" : "fp8");
    if (n_rows == 0) return MOE_OK;
    if (!xr || !expert_offsets || !w13 || !w2 || !h)
        return fail(MOE_ERR_INVALID_ARG, "NULL pointer argument");
    if (c.reduce_dense) {
        if (!recv_token || !recv_slot || !topk_w || !out_reduce)
            return fail(MOE_ERR_INVALID_ARG, "decode form needs recv_token, recv_slot, topk_w, out_reduce");
    } else if (!y) {
        return fail(MOE_ERR_INVALID_ARG, "y is NULL");
    }
    const void *ptrs[5] = {xr, w13, w2, h, y};
    for (const void *p : ptrs)
        if (p && !aligned(p, 16)) return fail(MOE_ERR_INVALID_ARG, "operand not 16-byte aligned");
    const ScratchLayout L = scratch_layout(c);
    uint32_t *status = ws_at<uint32_t>(ws, L.status);
    cudaError_t err;
    if (c.dtype == MOE_BF16) {
        int dev = 0, major = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        if (major != 10)
            return fail(MOE_ERR_UNSUPPORTED, "the bf16 FFN uses tcgen05 and needs sm_100 (got major %d)", major);
        err = launch_ffn_tcgen05(c, n_rows, xr, expert_offsets, w13, w2, h, y, recv_token,
                                 recv_slot, topk_w, out_reduce, status,
                                 ws_at<uint32_t>(ws, L.ffn_ctr), stream, current_num_sms());
        if (err == cudaErrorNotSupported)
            return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled unavailable or rejected a tensor map");
    } else {
        err = launch_ffn_simt(c, n_rows, xr, expert_offsets, w13, w2, h, y, recv_token,
                              recv_slot, topk_w, out_reduce, stream);
    }
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_grouped_swiglu_ffn");
}

moe_status moe_grouped_swiglu_ffn_backward(const moe_config *cfg, int64_t n_rows, const void *xr,
                                           const void *dy, const int32_t *expert_offsets,
                                           const void *w13, const void *w2, void *gu, void *h,
                                           void *dgu, void *dxr, float *dw13, float *dw2,
                                           int32_t accumulate, void *ws, cudaStream_t stream) {
    moe_status st = moe_config_check(cfg);
    if (st != MOE_OK) return st;
    if ((st = check_ws(ws)) != MOE_OK) return st;
    const moe_config &c = *cfg;
    if (n_rows < 0) return fail(MOE_ERR_INVALID_ARG, "n_rows < 0");
    if (accumulate != 0 && accumulate != 1) return fail(MOE_ERR_INVALID_ARG, "accumulate must be 0 or 1");
    if (c.ffn_fp8) return fail(MOE_ERR_UNSUPPORTED, "the FFN backward runs on bf16 or fp32 weights (ffn_fp8 = 0)");
    if (!expert_offsets || !w13 || !w2 || !dw13 || !dw2) return fail(MOE_ERR_INVALID_ARG, "NULL pointer argument");
    if (n_rows > 0 && (!xr || !dy || !h || !dgu || !dxr || (c.dtype == MOE_BF16 && !gu)))
        return fail(MOE_ERR_INVALID_ARG, "NULL pointer argument");
    const void *ptrs[9] = {xr, dy, w13, w2, gu, h, dgu, dxr, dw13};
    for (const void *p : ptrs)
        if (p && !aligned(p, 16)) return fail(MOE_ERR_INVALID_ARG, "operand not 16-byte aligned");
    if (!aligned(dw2, 16)) return fail(MOE_ERR_INVALID_ARG, "operand not 16-byte aligned");
    const ScratchLayout L = scratch_layout(c);
    cudaError_t err;
    if (c.dtype == MOE_BF16) {
        int dev = 0, major = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        if (major != 10)
            return fail(MOE_ERR_UNSUPPORTED, "the bf16 FFN backward uses tcgen05 and needs sm_100 (got major %d)", major);
        if (n_rows == 0) {
            // no rows: the weight gradients are zero (or unchanged when accumulating)
            err = cudaSuccess;
            if (!accumulate) {
                err = cudaMemsetAsync(dw13, 0, sizeof(float) * (size_t)c.E * 2 * c.I * c.H, stream);
                if (err == cudaSuccess)
                    err = cudaMemsetAsync(dw2, 0, sizeof(float) * (size_t)c.E * c.H * c.I, stream);
            }
        } else {
            err = launch_ffn_tcgen05_bwd(c, n_rows, xr, dy, expert_offsets, w13, w2, gu, h, dgu, dxr, dw13,
                                         dw2, accumulate, ws_at<uint32_t>(ws, L.status),
                                         ws_at<uint32_t>(ws, L.ffn_ctr), stream, current_num_sms());
            if (err == cudaErrorNotSupported)
                return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled unavailable or rejected a tensor map");
        }
    } else {
        err = launch_ffn_simt_bwd(c, n_rows, xr, dy, expert_offsets, w13, w2, h, dgu, dxr, dw13, dw2,
                                  accumulate, stream);
    }
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_grouped_swiglu_ffn_backward");
}

moe_status moe_quantize_fp8_rows(int64_t rows, int32_t cols, int32_t in_dtype, const void *in,
                                 uint8_t *codes, uint8_t *scales, cudaStream_t stream) {
    if (rows < 0 || cols < 1) return fail(MOE_ERR_INVALID_ARG, "rows < 0 or cols < 1");
    if (in_dtype != MOE_BF16 && in_dtype != MOE_F32)
        return fail(MOE_ERR_INVALID_ARG, "in_dtype must be MOE_BF16 or MOE_F32");
    const bool bf16 = in_dtype == MOE_BF16;
    if (cols % (bf16 ? 8 : 4) != 0)
        return fail(MOE_ERR_UNSUPPORTED, "cols %% %d != 0 (cols=%d)", bf16 ? 8 : 4, cols);
    if (rows == 0) return MOE_OK;
    if (!in || !codes || !scales) return fail(MOE_ERR_INVALID_ARG, "NULL pointer argument");
    if (!aligned(in, 16) || !aligned(codes, bf16 ? 8 : 4))
        return fail(MOE_ERR_INVALID_ARG, "in not 16-byte or codes not %d-byte aligned", bf16 ? 8 : 4);
    cudaError_t err = launch_quant_rows(rows, cols, bf16, in, codes, scales, nullptr, stream,
                                        current_num_sms());
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_quantize_fp8_rows");
}

moe_status moe_permute_quantize_fp8(const moe_config *cfg, const void *x, const int32_t *pos,
                                    int32_t tok_begin, int32_t tok_count, uint8_t *xr_q,
                                    uint8_t *x_scale, cudaStream_t stream) {
    moe_status st = moe_config_check(cfg);
    if (st != MOE_OK) return st;
    const moe_config &c = *cfg;
    if (c.ffn_fp8 != 1) return fail(MOE_ERR_INVALID_ARG, "cfg->ffn_fp8 = %d: use moe_permute%s", c.ffn_fp8,
                                    c.ffn_fp8 == 2 ? "_quantize_fp8_blocks" : "");
    if (!fused_permute_quant(c)) return fail(MOE_ERR_UNSUPPORTED, "H=%d > 8192", c.H);
    if ((st = check_range(c, tok_begin, tok_count, false)) != MOE_OK) return st;
    if (tok_count > 0 && (!x || !pos || !xr_q || !x_scale))
        return fail(MOE_ERR_INVALID_ARG, "NULL pointer argument");
    if (!aligned(x, 16) || !aligned(xr_q, 16)) return fail(MOE_ERR_INVALID_ARG, "x / xr_q not 16-byte aligned");
    cudaError_t err = launch_permute_quant(c, x, pos, tok_begin, tok_count, xr_q, x_scale, stream);
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_permute_quantize_fp8");
}

moe_status moe_grouped_swiglu_ffn_fp8(const moe_config *cfg, int64_t n_rows, const uint8_t *xr_q,
                                      const uint8_t *x_scale, const int32_t *expert_offsets,
                                      const uint8_t *w13_q, const uint8_t *w13_scale,
                                      const uint8_t *w2_q, const uint8_t *w2_scale, void *h,
                                      uint8_t *h_q, uint8_t *h_scale, void *y,
                                      const int32_t *recv_token, const int32_t *recv_slot,
                                      const float *topk_w, float *out_reduce, void *ws,
                                      cudaStream_t stream) {
    moe_status st = moe_config_check(cfg);
    if (st != MOE_OK) return st;
    if ((st = check_ws(ws)) != MOE_OK) return st;
    const moe_config &c = *cfg;
    if (c.ffn_fp8 != 1) return fail(MOE_ERR_INVALID_ARG, "cfg->ffn_fp8 = %d: use moe_grouped_swiglu_ffn%s",
                                    c.ffn_fp8, c.ffn_fp8 == 2 ? "_mxfp8" : "");
    if (n_rows < 0) return fail(MOE_ERR_INVALID_ARG, "n_rows < 0");
    if (n_rows == 0) return MOE_OK;
    if (!xr_q || !x_scale || !expert_offsets || !w13_q || !w13_scale || !w2_q || !w2_scale || !h ||
        !h_q || !h_scale || !recv_token)
        return fail(MOE_ERR_INVALID_ARG, "NULL pointer argument");
    if (c.reduce_dense) {
        if (!recv_slot || !topk_w || !out_reduce)
            return fail(MOE_ERR_INVALID_ARG, "decode form needs recv_slot, topk_w, out_reduce");
    } else if (!y) {
        return fail(MOE_ERR_INVALID_ARG, "y is NULL");
    }
    const void *ptrs[6] = {xr_q, w13_q, w2_q, h, h_q, y};
    for (const void *p : ptrs)
        if (p && !aligned(p, 16)) return fail(MOE_ERR_INVALID_ARG, "operand not 16-byte aligned");
    int dev = 0, major = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (major != 10)
        return fail(MOE_ERR_UNSUPPORTED, "the FP8 FFN uses tcgen05 and needs sm_100 (got major %d)", major);
    const ScratchLayout L = scratch_layout(c);
    cudaError_t err = launch_ffn_tcgen05_fp8(c, n_rows, xr_q, x_scale, expert_offsets, w13_q,
                                             w13_scale, w2_q, w2_scale, h, h_q, h_scale, y,
                                             recv_token, recv_slot, topk_w, out_reduce,
                                             ws_at<uint32_t>(ws, L.status),
                                             ws_at<uint32_t>(ws, L.ffn_ctr), stream,
                                             current_num_sms());
    if (err == cudaErrorNotSupported)
        return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled unavailable or rejected a tensor map");
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_grouped_swiglu_ffn_fp8");
}

moe_status moe_quantize_fp8_blocks(int64_t rows, int32_t cols, int32_t in_dtype, const void *in,
                                   uint8_t *codes, uint8_t *scales, cudaStream_t stream) {
    if (rows < 0 || cols < 1) return fail(MOE_ERR_INVALID_ARG, "rows < 0 or cols < 1");
    if (in_dtype != MOE_BF16 && in_dtype != MOE_F32)
        return fail(MOE_ERR_INVALID_ARG, "in_dtype must be MOE_BF16 or MOE_F32");
    if (cols % 32 != 0) return fail(MOE_ERR_UNSUPPORTED, "cols %% 32 != 0 (cols=%d)", cols);
    if (rows == 0) return MOE_OK;
    if (!in || !codes || !scales) return fail(MOE_ERR_INVALID_ARG, "NULL pointer argument");
    const bool bf16 = in_dtype == MOE_BF16;
    if (!aligned(in, 16) || !aligned(codes, bf16 ? 8 : 4))
        return fail(MOE_ERR_INVALID_ARG, "in not 16-byte or codes not %d-byte aligned", bf16 ? 8 : 4);
    cudaError_t err = launch_quant_blocks(rows, cols, bf16, in, codes, scales, stream, current_num_sms());
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_quantize_fp8_blocks");
}

moe_status moe_permute_quantize_fp8_blocks(const moe_config *cfg, const void *x, const int32_t *pos,
                                           int32_t tok_begin, int32_t tok_count, uint8_t *xr_q,
                                           uint8_t *xr_sf, cudaStream_t stream) {
    moe_status st = moe_config_check(cfg);
    if (st != MOE_OK) return st;
    const moe_config &c = *cfg;
    if (c.ffn_fp8 != 2) return fail(MOE_ERR_INVALID_ARG, "cfg->ffn_fp8 must be 2 (K-blocked scales)");
    if (!fused_permute_quant(c)) return fail(MOE_ERR_UNSUPPORTED, "H=%d > 8192", c.H);
    if ((st = check_range(c, tok_begin, tok_count, false)) != MOE_OK) return st;
    if (tok_count > 0 && (!x || !pos || !xr_q || !xr_sf))
        return fail(MOE_ERR_INVALID_ARG, "NULL pointer argument");
    if (!aligned(x, 16) || !aligned(xr_q, 16)) return fail(MOE_ERR_INVALID_ARG, "x / xr_q not 16-byte aligned");
    cudaError_t err = launch_permute_quant_blocks(c, x, pos, tok_begin, tok_count, xr_q, xr_sf, stream);
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_permute_quantize_fp8_blocks");
}

moe_status moe_grouped_swiglu_ffn_mxfp8(const moe_config *cfg, int64_t n_rows, const uint8_t *xr_q,
                                        const uint8_t *xr_sf, const int32_t *expert_offsets,
                                        const uint8_t *w13_q, const uint8_t *w13_sf, const uint8_t *w2_q,
                                        const uint8_t *w2_sf, uint8_t *h_q, uint8_t *h_sf, void *y,
                                        const int32_t *recv_token, const int32_t *recv_slot,
                                        const float *topk_w, float *out_reduce, void *ws,
                                        cudaStream_t stream) {
    moe_status st = moe_config_check(cfg);
    if (st != MOE_OK) return st;
    if ((st = check_ws(ws)) != MOE_OK) return st;
    const moe_config &c = *cfg;
    if (c.ffn_fp8 != 2) return fail(MOE_ERR_INVALID_ARG, "cfg->ffn_fp8 must be 2 (K-blocked scales)");
    if (n_rows < 0) return fail(MOE_ERR_INVALID_ARG, "n_rows < 0");
    if (n_rows == 0) return MOE_OK;
    if (!xr_q || !xr_sf || !expert_offsets || !w13_q || !w13_sf || !w2_q || !w2_sf || !h_q || !h_sf)
        return fail(MOE_ERR_INVALID_ARG, "NULL pointer argument");
    if (c.reduce_dense) {
        if (!recv_token || !recv_slot || !topk_w || !out_reduce)
            return fail(MOE_ERR_INVALID_ARG, "decode form needs recv_token, recv_slot, topk_w, out_reduce");
    } else if (!y) {
        return fail(MOE_ERR_INVALID_ARG, "y is NULL");
    }
    const void *a16[5] = {xr_q, w13_q, w2_q, h_q, y};
    for (const void *p : a16)
        if (p && !aligned(p, 16)) return fail(MOE_ERR_INVALID_ARG, "operand not 16-byte aligned");
    const void *a4[4] = {xr_sf, w13_sf, w2_sf, h_sf};
    for (const void *p : a4)
        if (!aligned(p, 4)) return fail(MOE_ERR_INVALID_ARG, "scale array not 4-byte aligned");
    int dev = 0, major = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (major != 10)
        return fail(MOE_ERR_UNSUPPORTED, "the MX FP8 FFN uses tcgen05 and needs sm_100 (got major %d)", major);
    const ScratchLayout L = scratch_layout(c);
    cudaError_t err = launch_ffn_mx(c, n_rows, xr_q, xr_sf, expert_offsets, w13_q, w13_sf, w2_q, w2_sf, h_q,
                                    h_sf, y, recv_token, recv_slot, topk_w, out_reduce,
                                    ws_at<uint32_t>(ws, L.status), ws_at<uint32_t>(ws, L.ffn_ctr), stream,
                                    current_num_sms());
    if (err == cudaErrorNotSupported)
        return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled unavailable or rejected a tensor map");
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_grouped_swiglu_ffn_mxfp8");
}

// The shared expert over rows [tb, tb + tc) of x: the step-5 kernel as one
// expert whose offsets {0, tc} live in the workspace, with its own counters.
static cudaError_t launch_shared_ffn(const moe_config &c, int tb, int tc, const void *x,
                                     const void *w13s, const void *w2s, void *hs, void *ys,
                                     void *ws, cudaStream_t s, int nsm) {
    if (tc == 0) return cudaSuccess;
    const ScratchLayout L = scratch_layout(c);
    int32_t *off = ws_at<int32_t>(ws, L.shared_off);
    cudaError_t err = launch_shared_offsets(off, tc, s);
    if (err != cudaSuccess) return err;
    moe_config cs = c;
    cs.E = 1;
    cs.I = c.shared_I;
    cs.reduce_dense = 0;
    cs.capacity = -1;
    const size_t eb = c.dtype == MOE_F32 ? 4 : 2;
    const void *xs = static_cast<const unsigned char *>(x) + eb * (size_t)tb * c.H;
    uint32_t *status = ws_at<uint32_t>(ws, L.status);
    if (c.dtype == MOE_BF16)
        return launch_ffn_tcgen05(cs, tc, xs, off, w13s, w2s, hs, ys, nullptr, nullptr, nullptr,
                                  nullptr, status, ws_at<uint32_t>(ws, L.shared_ctr), s, nsm);
    return launch_ffn_simt(cs, tc, xs, off, w13s, w2s, hs, ys, nullptr, nullptr, nullptr, nullptr, s);
}

moe_status moe_shared_expert_ffn(const moe_config *cfg, int32_t tok_begin, int32_t tok_count,
                                 const void *x, const void *w13_shared, const void *w2_shared,
                                 void *h_shared, void *y_shared, void *ws, cudaStream_t stream) {
    moe_status st = moe_config_check(cfg);
    if (st != MOE_OK) return st;
    if ((st = check_ws(ws)) != MOE_OK) return st;
    const moe_config &c = *cfg;
    if (c.shared_I <= 0) return fail(MOE_ERR_INVALID_ARG, "cfg has no shared expert (shared_I = 0)");
    if ((st = check_range(c, tok_begin, tok_count, false)) != MOE_OK) return st;
    if (tok_count == 0) return MOE_OK;
    if (!x || !w13_shared || !w2_shared || !h_shared || !y_shared)
        return fail(MOE_ERR_INVALID_ARG, "NULL pointer argument");
    const void *ptrs[5] = {x, w13_shared, w2_shared, h_shared, y_shared};
    for (const void *p : ptrs)
        if (!aligned(p, 16)) return fail(MOE_ERR_INVALID_ARG, "operand not 16-byte aligned");
    if (c.dtype == MOE_BF16) {
        int dev = 0, major = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        if (major != 10)
            return fail(MOE_ERR_UNSUPPORTED, "the bf16 FFN uses tcgen05 and needs sm_100 (got major %d)", major);
    }
    cudaError_t err = launch_shared_ffn(c, tok_begin, tok_count, x, w13_shared, w2_shared, h_shared,
                                        y_shared, ws, stream, current_num_sms());
    if (err == cudaErrorNotSupported)
        return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled unavailable or rejected a tensor map");
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_shared_expert_ffn");
}

moe_status moe_combine(const moe_config *cfg, const void *y, const int32_t *pos,
                       const float *topk_w, int32_t tok_begin, int32_t tok_count,
                       const void *y_shared, void *out, cudaStream_t stream) {
    moe_status st = moe_config_check(cfg);
    if (st != MOE_OK) return st;
    const moe_config &c = *cfg;
    if ((st = check_range(c, tok_begin, tok_count, false)) != MOE_OK) return st;
    if (tok_count > 0 && (!y || !pos || !topk_w || !out))
        return fail(MOE_ERR_INVALID_ARG, "NULL pointer argument");
    if (!aligned(y, 16) || !aligned(out, 16) || !aligned(y_shared, 16))
        return fail(MOE_ERR_INVALID_ARG, "y / y_shared / out not 16-byte aligned");
    cudaError_t err = launch_combine(c, y, pos, topk_w, tok_begin, tok_count, y_shared, out, stream);
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_combine");
}

moe_status moe_combine_backward(const moe_config *cfg, const void *dout, const void *y,
                                const int32_t *pos, const float *topk_w, int32_t tok_begin,
                                int32_t tok_count, void *dy, float *dw, cudaStream_t stream) {
    moe_status st = moe_config_check(cfg);
    if (st != MOE_OK) return st;
    const moe_config &c = *cfg;
    if (c.reduce_dense)
        return fail(MOE_ERR_UNSUPPORTED, "decode form: the expert rows y are not stored");
    if ((st = check_range(c, tok_begin, tok_count, false)) != MOE_OK) return st;
    if (tok_count > 0 && (!dout || !y || !pos || !topk_w || !dy || !dw))
        return fail(MOE_ERR_INVALID_ARG, "NULL pointer argument");
    if (!aligned(dout, 16) || !aligned(y, 16) || !aligned(dy, 16))
        return fail(MOE_ERR_INVALID_ARG, "dout / y / dy not 16-byte aligned");
    cudaError_t err = launch_combine_bwd(c, dout, y, pos, topk_w, tok_begin, tok_count, dy, dw, stream);
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_combine_backward");
}

moe_status moe_route_backward(const moe_config *cfg, const int32_t *topk_idx, const float *topk_w,
                              const float *dw, float *dlogits, float *dbias, void *ws,
                              cudaStream_t stream) {
    moe_status st = moe_config_check(cfg);
    if (st != MOE_OK) return st;
    if ((st = check_ws(ws)) != MOE_OK) return st;
    const moe_config &c = *cfg;
    if (c.T > 0 && (!topk_idx || !topk_w || !dw || !dlogits))
        return fail(MOE_ERR_INVALID_ARG, "NULL pointer argument");
    const ScratchLayout L = scratch_layout(c);
    cudaError_t err = launch_route_bwd(c, topk_idx, topk_w, dw, dlogits, dbias,
                                       ws_at<uint32_t>(ws, L.status), stream);
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_route_backward");
}

moe_status moe_permute_backward(const moe_config *cfg, const void *dxr, const int32_t *pos,
                                int32_t tok_begin, int32_t tok_count, void *dx, cudaStream_t stream) {
    moe_status st = moe_config_check(cfg);
    if (st != MOE_OK) return st;
    const moe_config &c = *cfg;
    if ((st = check_range(c, tok_begin, tok_count, false)) != MOE_OK) return st;
    if (tok_count > 0 && (!dxr || !pos || !dx)) return fail(MOE_ERR_INVALID_ARG, "NULL pointer argument");
    if (!aligned(dxr, 16) || !aligned(dx, 16)) return fail(MOE_ERR_INVALID_ARG, "dxr / dx not 16-byte aligned");
    // the combine with unit weights: dx[t] = sum of the token's kept receive rows
    cudaError_t err = launch_combine(c, dxr, pos, nullptr, tok_begin, tok_count, nullptr, dx, stream);
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_permute_backward");
}

moe_status moe_reduce_finalize(const moe_config *cfg, const float *out_reduce,
                               int32_t tok_begin, int32_t tok_count, const void *y_shared,
                               void *out, cudaStream_t stream) {
    moe_status st = moe_config_check(cfg);
    if (st != MOE_OK) return st;
    const moe_config &c = *cfg;
    if ((st = check_range(c, tok_begin, tok_count, false)) != MOE_OK) return st;
    if (tok_count > 0 && (!out_reduce || !out)) return fail(MOE_ERR_INVALID_ARG, "NULL pointer argument");
    if (!aligned(out_reduce, 16) || !aligned(out, 16) || !aligned(y_shared, 16))
        return fail(MOE_ERR_INVALID_ARG, "out_reduce / y_shared / out not 16-byte aligned");
    cudaError_t err = launch_reduce_finalize(c, out_reduce, tok_begin, tok_count, y_shared, out,
                                             stream, current_num_sms());
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_reduce_finalize");
}

// Host side of moe_forward_host: pinned activations in, the layer's output out.
struct HostIO {
    const float *logits, *bias;
    const void *x;
    void *out;
};

// The two-stream chunked layer.  With io set, logits, bias, x and out are the
// workspace's staging buffers: the copies in are enqueued first (logits and
// bias on s_dispatch ahead of routing, each chunk's x on s_compute so that it
// overlaps routing), and chunk c's output goes back on s_dispatch behind chunk
// c+1's dispatch, overlapping chunk c+1's FFN.
static moe_status forward_run(const moe_config &c, const ForwardLayout &F, const float *logits,
                              const float *bias, const void *x, const void *w13, const void *w2,
                              const void *w13_shared, const void *w2_shared,
                              const uint8_t *w13_scale, const uint8_t *w2_scale, void *out,
                              int32_t *topk_idx, float *topk_w, uint8_t *keep,
                              int32_t *splits_host, void *ws, cudaStream_t s_dispatch,
                              cudaStream_t s_compute, const HostIO *io, void *xr_save = nullptr,
                              void *y_save = nullptr) {
    const ScratchLayout L = scratch_layout(c);
    uint32_t *status = ws_at<uint32_t>(ws, L.status);
    int32_t *counts = ws_at<int32_t>(ws, F.counts);
    int32_t *kept_counts = ws_at<int32_t>(ws, F.kept_counts);
    float *out_reduce = c.reduce_dense ? ws_at<float>(ws, F.out_reduce) : nullptr;
    const int nsm = current_num_sms();
    const int nch = c.n_chunks;
    const int tc = F.tc;
    const size_t eb = c.dtype == MOE_F32 ? 4 : 2;
    const size_t chunk_bytes = eb * (size_t)tc * c.H;

    const bool shared = c.shared_I > 0;
    cudaEvent_t *ev = nullptr;
    cudaError_t err = get_events(4 * nch + 3, &ev);
    if (err != cudaSuccess) return cuda_fail(err, "event pool");
    cudaEvent_t ev_start = ev[0], ev_end = ev[1], ev_tail = ev[2];
    cudaEvent_t *ev_disp = ev + 3, *ev_done = ev + 3 + nch, *ev_shared = ev + 3 + 2 * nch;
    cudaEvent_t *ev_x = ev + 3 + 3 * nch;

#define MOE_TRY(expr, where)                                   \
    do {                                                       \
        cudaError_t e_ = (expr);                               \
        if (e_ != cudaSuccess) return cuda_fail(e_, where);    \
    } while (0)

    // the compute stream's earlier work on this workspace precedes the new dispatch
    MOE_TRY(cudaEventRecord(ev_start, s_compute), "record start");
    MOE_TRY(cudaStreamWaitEvent(s_dispatch, ev_start, 0), "wait start");
    if (io) {
        MOE_TRY(cudaMemcpyAsync((void *)logits, io->logits, sizeof(float) * (size_t)c.T * c.E,
                                cudaMemcpyHostToDevice, s_dispatch), "copy logits in");
        if (bias)
            MOE_TRY(cudaMemcpyAsync((void *)bias, io->bias, sizeof(float) * (size_t)c.E,
                                    cudaMemcpyHostToDevice, s_dispatch), "copy bias in");
        for (int ch = 0; ch < nch; ++ch) {
            MOE_TRY(cudaMemcpyAsync((char *)x + (size_t)ch * chunk_bytes,
                                    (const char *)io->x + (size_t)ch * chunk_bytes, chunk_bytes,
                                    cudaMemcpyHostToDevice, s_compute), "copy x in");
            MOE_TRY(cudaEventRecord(ev_x[ch], s_compute), "record x");
        }
    }
    MOE_TRY(launch_route_topk(c, logits, bias, topk_idx, topk_w, counts, status, s_dispatch, nsm),
            "route_topk");
    MOE_TRY(launch_capacity_clip(c, topk_idx, topk_w, counts, keep, kept_counts,
                                 ws_at<uint64_t>(ws, L.clip_thr), ws_at<int32_t>(ws, L.clip_seg),
                                 ws_at<uint64_t>(ws, L.clip_keys), status, s_dispatch, nsm),
            "capacity_clip");
    if (c.reduce_dense)
        MOE_TRY(cudaMemsetAsync(out_reduce, 0, sizeof(float) * (size_t)c.T * c.H, s_dispatch),
                "clear reduce buffer");

    // chunk ch's output back to the host, on s_dispatch once its combine is done
    auto copy_out = [&](int ch) -> cudaError_t {
        cudaError_t e = cudaStreamWaitEvent(s_dispatch, ev_done[ch], 0);
        if (e != cudaSuccess) return e;
        return cudaMemcpyAsync((char *)io->out + (size_t)ch * chunk_bytes,
                               (const char *)out + (size_t)ch * chunk_bytes, chunk_bytes,
                               cudaMemcpyDeviceToHost, s_dispatch);
    };
    const int split_stride = c.E + 1 + c.ep * c.ep;
    for (int ch = 0; ch < nch; ++ch) {
        const Slot &S = F.slot[ch & 1];
        const int tb = ch * tc;
        if (ch >= 2) MOE_TRY(cudaStreamWaitEvent(s_dispatch, ev_done[ch - 2], 0), "wait slot");
        int32_t *eoff = ws_at<int32_t>(ws, S.eoff);
        int32_t *recv_token = ws_at<int32_t>(ws, S.recv_token);
        int32_t *recv_slot = ws_at<int32_t>(ws, S.recv_slot);
        int32_t *pos = ws_at<int32_t>(ws, S.pos);
        // the saved dispatch outputs ([AX] expert_parallel_save_dispatch): chunk
        // ch's receive rows and expert outputs in the caller's buffers
        const size_t save_off = (size_t)ch * F.nmax * c.H * eb;
        void *xr = xr_save ? static_cast<char *>(xr_save) + save_off : ws_at<void>(ws, S.xr);
        void *h = ws_at<void>(ws, S.h);
        void *y = c.reduce_dense ? nullptr
                  : y_save ? static_cast<char *>(y_save) + save_off : ws_at<void>(ws, S.y);
        MOE_TRY(launch_dispatch_layout(c, tb, tc, topk_idx, keep, eoff, ws_at<int32_t>(ws, S.roff),
                                       recv_token, recv_slot, pos, ws_at<int32_t>(ws, S.splits),
                                       splits_host ? splits_host + (size_t)ch * split_stride : nullptr,
                                       ws, F.nmax, s_dispatch, nsm),
                "dispatch_layout");
        if (io) MOE_TRY(cudaStreamWaitEvent(s_dispatch, ev_x[ch], 0), "wait x");
        if (c.ffn_fp8 == 2) {
            // codes of the kept rows and their 32-value block scales, per receive row
            MOE_TRY(launch_permute_quant_blocks(c, x, pos, tb, tc, static_cast<uint8_t *>(xr),
                                                ws_at<uint8_t>(ws, S.xsf), s_dispatch), "permute + quantize x");
        } else if (c.ffn_fp8 && fused_permute_quant(c)) {
            // each kept token row quantised once and its codes written to its receive rows
            MOE_TRY(launch_permute_quant(c, x, pos, tb, tc, static_cast<uint8_t *>(xr),
                                         ws_at<uint8_t>(ws, F.xsc), s_dispatch), "permute + quantize x");
        } else if (c.ffn_fp8) {
            // rows too long for the fused kernel: quantise the chunk's rows, then permute the codes
            uint8_t *xq = ws_at<uint8_t>(ws, F.xq);
            MOE_TRY(launch_quant_rows(tc, c.H, true, static_cast<const char *>(x) + eb * (size_t)tb * c.H,
                                      xq + (size_t)tb * c.H, ws_at<uint8_t>(ws, F.xsc) + tb, nullptr,
                                      s_dispatch, nsm), "quantize x");
            MOE_TRY(launch_permute(c, xq, pos, tb, tc, xr, s_dispatch), "permute");
        } else {
            MOE_TRY(launch_permute(c, x, pos, tb, tc, xr, s_dispatch), "permute");
        }
        MOE_TRY(cudaEventRecord(ev_disp[ch], s_dispatch), "record dispatch");
        void *ys = shared ? ws_at<void>(ws, S.ys) : nullptr;
        if (shared) {
            // the shared expert of the chunk beside its routed FFN; the combine waits for it
            err = launch_shared_ffn(c, tb, tc, x, w13_shared, w2_shared, ws_at<void>(ws, S.hs), ys,
                                    ws, s_dispatch, nsm);
            if (err == cudaErrorNotSupported)
                return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled unavailable or rejected a tensor map");
            MOE_TRY(err, "shared_expert_ffn");
            MOE_TRY(cudaEventRecord(ev_shared[ch], s_dispatch), "record shared");
        }
        if (io && ch >= 1) MOE_TRY(copy_out(ch - 1), "copy out");
        MOE_TRY(cudaStreamWaitEvent(s_compute, ev_disp[ch], 0), "wait dispatch");
        if (F.nmax > 0) {
            if (c.ffn_fp8 == 2) {
                err = launch_ffn_mx(c, F.nmax, static_cast<const uint8_t *>(xr), ws_at<uint8_t>(ws, S.xsf), eoff,
                                    static_cast<const uint8_t *>(w13), w13_scale, static_cast<const uint8_t *>(w2),
                                    w2_scale, ws_at<uint8_t>(ws, S.hq), ws_at<uint8_t>(ws, S.hsc), y, recv_token,
                                    recv_slot, topk_w, out_reduce, status, ws_at<uint32_t>(ws, L.ffn_ctr),
                                    s_compute, nsm);
                if (err == cudaErrorNotSupported)
                    return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled unavailable or rejected a tensor map");
            } else if (c.ffn_fp8) {
                err = launch_ffn_tcgen05_fp8(c, F.nmax, static_cast<const uint8_t *>(xr),
                                             ws_at<uint8_t>(ws, F.xsc), eoff,
                                             static_cast<const uint8_t *>(w13), w13_scale,
                                             static_cast<const uint8_t *>(w2), w2_scale, h,
                                             ws_at<uint8_t>(ws, S.hq), ws_at<uint8_t>(ws, S.hsc), y,
                                             recv_token, recv_slot, topk_w, out_reduce, status,
                                             ws_at<uint32_t>(ws, L.ffn_ctr), s_compute, nsm);
                if (err == cudaErrorNotSupported)
                    return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled unavailable or rejected a tensor map");
            } else if (c.dtype == MOE_BF16) {
                err = launch_ffn_tcgen05(c, F.nmax, xr, eoff, w13, w2, h, y, recv_token, recv_slot,
                                         topk_w, out_reduce, status, ws_at<uint32_t>(ws, L.ffn_ctr),
                                         s_compute, nsm);
                if (err == cudaErrorNotSupported)
                    return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled unavailable or rejected a tensor map");
            } else {
                err = launch_ffn_simt(c, F.nmax, xr, eoff, w13, w2, h, y, recv_token, recv_slot,
                                      topk_w, out_reduce, s_compute);
            }
            MOE_TRY(err, "grouped_swiglu_ffn");
        }
        if (shared) MOE_TRY(cudaStreamWaitEvent(s_compute, ev_shared[ch], 0), "wait shared");
        if (c.reduce_dense)
            MOE_TRY(launch_reduce_finalize(c, out_reduce, tb, tc, ys, out, s_compute, nsm), "reduce_finalize");
        else
            MOE_TRY(launch_combine(c, y, pos, topk_w, tb, tc, ys, out, s_compute), "combine");
        MOE_TRY(cudaEventRecord(ev_done[ch], s_compute), "record done");
    }
    MOE_TRY(cudaEventRecord(ev_end, s_compute), "record end");
    MOE_TRY(cudaStreamWaitEvent(s_dispatch, ev_end, 0), "wait end");
    if (io) {
        MOE_TRY(copy_out(nch - 1), "copy out");
        MOE_TRY(cudaEventRecord(ev_tail, s_dispatch), "record tail");
        MOE_TRY(cudaStreamWaitEvent(s_compute, ev_tail, 0), "wait tail");
    }
#undef MOE_TRY
    return MOE_OK;
}

moe_status moe_forward_chunked(const moe_config *cfg, const float *logits, const float *bias,
                               const void *x, const void *w13, const void *w2,
                               const void *w13_shared, const void *w2_shared,
                               const uint8_t *w13_scale, const uint8_t *w2_scale, void *out,
                               int32_t *topk_idx, float *topk_w, uint8_t *keep,
                               int32_t *splits_host, void *ws, cudaStream_t s_dispatch,
                               cudaStream_t s_compute) {
    moe_status st = moe_config_check(cfg);
    if (st != MOE_OK) return st;
    if ((st = check_ws(ws)) != MOE_OK) return st;
    const moe_config &c = *cfg;
    if (c.T > 0 && (!logits || !x || !w13 || !w2 || !out || !topk_idx || !topk_w || !keep))
        return fail(MOE_ERR_INVALID_ARG, "NULL pointer argument");
    if (c.T > 0 && c.shared_I > 0 && (!w13_shared || !w2_shared))
        return fail(MOE_ERR_INVALID_ARG, "shared_I > 0 needs w13_shared and w2_shared");
    if (c.T > 0 && c.ffn_fp8 && (!w13_scale || !w2_scale))
        return fail(MOE_ERR_INVALID_ARG, "ffn_fp8 needs w13_scale and w2_scale");
    if (c.T == 0) return MOE_OK;
    return forward_run(c, forward_layout(c), logits, bias, x, w13, w2, w13_shared, w2_shared,
                       w13_scale, w2_scale, out, topk_idx, topk_w, keep, splits_host, ws,
                       s_dispatch, s_compute, nullptr);
}

moe_status moe_forward_chunked_save(const moe_config *cfg, const float *logits, const float *bias,
                                    const void *x, const void *w13, const void *w2,
                                    const void *w13_shared, const void *w2_shared, void *out,
                                    int32_t *topk_idx, float *topk_w, uint8_t *keep,
                                    int32_t *splits_host, void *xr_save, void *y_save, void *ws,
                                    cudaStream_t s_dispatch, cudaStream_t s_compute) {
    moe_status st = moe_config_check(cfg);
    if (st != MOE_OK) return st;
    if ((st = check_ws(ws)) != MOE_OK) return st;
    const moe_config &c = *cfg;
    if (c.ffn_fp8 || c.reduce_dense)
        return fail(MOE_ERR_UNSUPPORTED, "saving the dispatch outputs needs ffn_fp8 = 0 and reduce_dense = 0");
    if (c.T > 0 && (!logits || !x || !w13 || !w2 || !out || !topk_idx || !topk_w || !keep || !xr_save ||
                    !y_save))
        return fail(MOE_ERR_INVALID_ARG, "NULL pointer argument");
    if (c.T > 0 && c.shared_I > 0 && (!w13_shared || !w2_shared))
        return fail(MOE_ERR_INVALID_ARG, "shared_I > 0 needs w13_shared and w2_shared");
    if (!aligned(xr_save, 16) || !aligned(y_save, 16))
        return fail(MOE_ERR_INVALID_ARG, "xr_save / y_save not 16-byte aligned");
    if (c.T == 0) return MOE_OK;
    return forward_run(c, forward_layout(c), logits, bias, x, w13, w2, w13_shared, w2_shared, nullptr,
                       nullptr, out, topk_idx, topk_w, keep, splits_host, ws, s_dispatch, s_compute,
                       nullptr, xr_save, y_save);
}

size_t moe_backward_workspace_bytes(const moe_config *cfg) {
    if (moe_config_check(cfg) != MOE_OK) return 0;
    return backward_layout(*cfg).total;
}

moe_status moe_layer_backward(const moe_config *cfg, const void *x, const void *dout,
                              const void *w13, const void *w2, const void *w13_shared,
                              const void *w2_shared, const int32_t *topk_idx, const float *topk_w,
                              const uint8_t *keep, const void *xr_saved, const void *y_saved,
                              void *dx, float *dlogits, float *dbias, float *dw13, float *dw2,
                              float *dw13_shared, float *dw2_shared, int32_t accumulate, void *ws,
                              cudaStream_t stream) {
    moe_status st = moe_config_check(cfg);
    if (st != MOE_OK) return st;
    if ((st = check_ws(ws)) != MOE_OK) return st;
    const moe_config &c = *cfg;
    if (c.ffn_fp8 || c.reduce_dense)
        return fail(MOE_ERR_UNSUPPORTED, "the layer backward needs ffn_fp8 = 0 and reduce_dense = 0");
    if (accumulate != 0 && accumulate != 1) return fail(MOE_ERR_INVALID_ARG, "accumulate must be 0 or 1");
    if ((xr_saved == nullptr) != (y_saved == nullptr))
        return fail(MOE_ERR_INVALID_ARG, "xr_saved and y_saved are both given (saved) or both NULL (recompute)");
    if (!w13 || !w2 || !dw13 || !dw2 || (c.T > 0 && (!x || !dout || !topk_idx || !topk_w || !keep || !dx ||
                                                     !dlogits)))
        return fail(MOE_ERR_INVALID_ARG, "NULL pointer argument");
    const bool shared = c.shared_I > 0;
    if (shared && (!w13_shared || !w2_shared || !dw13_shared || !dw2_shared))
        return fail(MOE_ERR_INVALID_ARG, "shared_I > 0 needs the shared expert's weights and gradients");
    const void *al[6] = {x, dout, xr_saved, y_saved, dx, w13};
    for (const void *p : al)
        if (p && !aligned(p, 16)) return fail(MOE_ERR_INVALID_ARG, "operand not 16-byte aligned");
    if (c.dtype == MOE_BF16) {
        int dev = 0, major = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        if (major != 10)
            return fail(MOE_ERR_UNSUPPORTED, "the bf16 backward uses tcgen05 and needs sm_100 (got major %d)", major);
    }
    if (c.T == 0) return MOE_OK;
    const ScratchLayout L = scratch_layout(c);
    const BackwardLayout B = backward_layout(c);
    uint32_t *status = ws_at<uint32_t>(ws, L.status);
    uint32_t *ctr = ws_at<uint32_t>(ws, L.ffn_ctr);
    const int nsm = current_num_sms();
    const size_t eb = c.dtype == MOE_F32 ? 4 : 2;
    const bool bf16 = c.dtype == MOE_BF16;
    const int tc = B.tc;
    const int64_t nrow = B.nmax > 0 ? B.nmax : 1;   // the row distance between chunks' rows
    int32_t *pos = ws_at<int32_t>(ws, B.pos);
    float *dw = ws_at<float>(ws, B.dw);
    char *xr_all = xr_saved ? static_cast<char *>(const_cast<void *>(xr_saved)) : ws_at<char>(ws, B.xr);
    char *h_all = ws_at<char>(ws, B.h), *dy_all = ws_at<char>(ws, B.dy), *dgu_all = ws_at<char>(ws, B.dgu);
    moe_config cs = c;   // the shared expert: one expert of intermediate size shared_I
    cs.E = 1;
    cs.I = c.shared_I;
    cs.capacity = -1;
    int32_t *soff = ws_at<int32_t>(ws, L.shared_off);
#define MOE_TRY(expr, where)                                   \
    do {                                                       \
        cudaError_t e_ = (expr);                               \
        if (e_ == cudaErrorNotSupported)                       \
            return fail(MOE_ERR_CUDA, "%s: cuTensorMapEncodeTiled unavailable or rejected a tensor map", where); \
        if (e_ != cudaSuccess) return cuda_fail(e_, where);    \
    } while (0)
    for (int ch = 0; ch < c.n_chunks; ++ch) {
        const int tb = ch * tc;
        int32_t *eoff = ws_at<int32_t>(ws, B.eoff) + (size_t)ch * (c.E + 1);
        // the layout again, from the saved routing and keep mask (index work only)
        MOE_TRY(launch_dispatch_layout(c, tb, tc, topk_idx, keep, eoff, ws_at<int32_t>(ws, B.roff),
                                       ws_at<int32_t>(ws, B.recv_token), ws_at<int32_t>(ws, B.recv_slot), pos,
                                       ws_at<int32_t>(ws, B.splits), nullptr, ws, B.nmax, stream, nsm),
                "dispatch_layout");
        const size_t row0 = (size_t)ch * nrow;
        void *xr = xr_all + row0 * c.H * eb;
        void *h = h_all + row0 * c.I * eb, *dy = dy_all + row0 * c.H * eb, *dgu = dgu_all + row0 * 2 * c.I * eb;
        const void *y;
        if (y_saved) {
            y = static_cast<const char *>(y_saved) + row0 * c.H * eb;
        } else {
            // recompute: dispatch the rows again and run the expert FFN forward
            void *yw = ws_at<void>(ws, B.y);
            MOE_TRY(launch_permute(c, x, pos, tb, tc, xr, stream), "permute");
            if (B.nmax > 0) {
                if (bf16)
                    MOE_TRY(launch_ffn_tcgen05(c, B.nmax, xr, eoff, w13, w2, h, yw, nullptr, nullptr, nullptr,
                                               nullptr, status, ctr, stream, nsm),
                            "grouped_swiglu_ffn");
                else
                    MOE_TRY(launch_ffn_simt(c, B.nmax, xr, eoff, w13, w2, h, yw, nullptr, nullptr, nullptr,
                                            nullptr, stream),
                            "grouped_swiglu_ffn");
            }
            y = yw;
        }
        void *dxr = ws_at<void>(ws, B.dxr);
        MOE_TRY(launch_combine_bwd(c, dout, y, pos, topk_w, tb, tc, dy, dw, stream), "combine_backward");
        if (B.nmax > 0) {
            if (bf16)
                MOE_TRY(launch_ffn_tcgen05_dgrad(c, B.nmax, xr, dy, eoff, w13, w2, ws_at<void>(ws, B.gu), h, dgu,
                                                 dxr, status, ctr, stream, nsm),
                        "grouped_swiglu_ffn_backward");
            else
                MOE_TRY(launch_ffn_simt_dgrad(c, B.nmax, xr, dy, eoff, w13, w2, h, dgu, dxr, stream),
                        "grouped_swiglu_ffn_backward");
        }
        void *dxs = nullptr;
        if (shared) {
            // the shared expert saw every row of the chunk with weight 1: its dy is dout
            MOE_TRY(launch_shared_offsets(soff, tc, stream), "shared offsets");
            const void *xs = static_cast<const char *>(x) + eb * (size_t)tb * c.H;
            const void *ds = static_cast<const char *>(dout) + eb * (size_t)tb * c.H;
            void *hs = ws_at<char>(ws, B.hs) + eb * (size_t)tb * c.shared_I;
            void *dgus = ws_at<char>(ws, B.dgus) + eb * (size_t)tb * 2 * c.shared_I;
            dxs = ws_at<void>(ws, B.dxs);
            if (bf16)
                MOE_TRY(launch_ffn_tcgen05_dgrad(cs, tc, xs, ds, soff, w13_shared, w2_shared, ws_at<void>(ws, B.gus),
                                                 hs, dgus, dxs, status, ws_at<uint32_t>(ws, L.shared_ctr), stream,
                                                 nsm),
                        "shared expert backward");
            else
                MOE_TRY(launch_ffn_simt_dgrad(cs, tc, xs, ds, soff, w13_shared, w2_shared, hs, dgus, dxs, stream),
                        "shared expert backward");
        }
        // dx[t] = the sum of the token's kept receive-row gradients (+ its shared-expert row)
        MOE_TRY(launch_combine(c, dxr, pos, nullptr, tb, tc, dxs, dx, stream), "permute_backward");
    }
    // the weight gradients once, over every chunk's rows
    const int32_t *eoffs = ws_at<int32_t>(ws, B.eoff);
    if (bf16)
        MOE_TRY(launch_ffn_tcgen05_wgrad(c, c.n_chunks, nrow, eoffs, xr_all, dy_all, h_all, dgu_all, dw13, dw2,
                                         accumulate, status, stream, nsm),
                "weight gradients");
    else
        MOE_TRY(launch_ffn_simt_wgrad(c, c.n_chunks, nrow, eoffs, xr_all, dy_all, h_all, dgu_all, dw13, dw2,
                                      accumulate, stream),
                "weight gradients");
    if (shared) {
        MOE_TRY(launch_shared_offsets(soff, c.T, stream), "shared offsets");
        if (bf16)
            MOE_TRY(launch_ffn_tcgen05_wgrad(cs, 1, c.T, soff, x, dout, ws_at<void>(ws, B.hs),
                                             ws_at<void>(ws, B.dgus), dw13_shared, dw2_shared, accumulate, status,
                                             stream, nsm),
                    "shared weight gradients");
        else
            MOE_TRY(launch_ffn_simt_wgrad(cs, 1, c.T, soff, x, dout, ws_at<void>(ws, B.hs), ws_at<void>(ws, B.dgus),
                                          dw13_shared, dw2_shared, accumulate, stream),
                    "shared weight gradients");
    }
    MOE_TRY(launch_route_bwd(c, topk_idx, topk_w, dw, dlogits, dbias, status, stream), "route_backward");
#undef MOE_TRY
    return MOE_OK;
}

size_t moe_forward_host_workspace_bytes(const moe_config *cfg) {
    if (moe_config_check(cfg) != MOE_OK) return 0;
    return forward_layout(*cfg, true).total;
}

moe_status moe_forward_host(const moe_config *cfg, const float *logits_host,
                            const float *bias_host, const void *x_host, const void *w13,
                            const void *w2, const void *w13_shared, const void *w2_shared,
                            const uint8_t *w13_scale, const uint8_t *w2_scale,
                            void *out_host, int32_t *topk_idx, float *topk_w, uint8_t *keep,
                            int32_t *splits_host, void *ws, cudaStream_t s_dispatch,
                            cudaStream_t s_compute) {
    moe_status st = moe_config_check(cfg);
    if (st != MOE_OK) return st;
    if ((st = check_ws(ws)) != MOE_OK) return st;
    const moe_config &c = *cfg;
    if (c.T > 0 && (!logits_host || !x_host || !w13 || !w2 || !out_host || !topk_idx || !topk_w ||
                    !keep))
        return fail(MOE_ERR_INVALID_ARG, "NULL pointer argument");
    if (c.T > 0 && c.shared_I > 0 && (!w13_shared || !w2_shared))
        return fail(MOE_ERR_INVALID_ARG, "shared_I > 0 needs w13_shared and w2_shared");
    if (c.T > 0 && c.ffn_fp8 && (!w13_scale || !w2_scale))
        return fail(MOE_ERR_INVALID_ARG, "ffn_fp8 needs w13_scale and w2_scale");
    if (c.T == 0) return MOE_OK;
    const ForwardLayout F = forward_layout(c, true);
    const HostIO io{logits_host, bias_host, x_host, out_host};
    return forward_run(c, F, ws_at<float>(ws, F.stage_logits),
                       bias_host ? ws_at<float>(ws, F.stage_bias) : nullptr,
                       ws_at<void>(ws, F.stage_x), w13, w2, w13_shared, w2_shared, w13_scale,
                       w2_scale, ws_at<void>(ws, F.stage_out), topk_idx, topk_w, keep, splits_host, ws,
                       s_dispatch, s_compute, &io);
}

// One thread waits on something that never completes, through the same bounded
// helpers the kernels use, and reports the timeout like they do.
__global__ void watchdog_selftest_kernel(int which, uint64_t limit_ns, uint32_t *status) {
    __shared__ uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    fence_mbar_init();
    volatile int never = 0;
    // phase 0 never completes
    const bool ok = which == 0 ? mbar_wait_cluster_bounded(&bar, 0, &never, limit_ns)
                               : mbar_wait_bounded(&bar, 0, &never, limit_ns);
    if (!ok) raise_status(status, MOE_DEV_WAIT_TIMEOUT);
}

moe_status moe_watchdog_selftest(const moe_config *cfg, int32_t which, int32_t limit_us,
                                 void *ws, cudaStream_t stream) {
    moe_status st = moe_config_check(cfg);
    if (st != MOE_OK) return st;
    if ((st = check_ws(ws)) != MOE_OK) return st;
    if (which != 0 && which != 1) return fail(MOE_ERR_INVALID_ARG, "which must be 0 or 1");
    if (limit_us < 1 || limit_us > 2000000) return fail(MOE_ERR_INVALID_ARG, "limit_us outside [1, 2e6]");
    const ScratchLayout L = scratch_layout(*cfg);
    watchdog_selftest_kernel<<<1, 32, 0, stream>>>(which, (uint64_t)limit_us * 1000ull,
                                                   ws_at<uint32_t>(ws, L.status));
    cudaError_t err = cudaGetLastError();
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_watchdog_selftest");
}

moe_status moe_ep_regroup(const moe_config *cfg, const int32_t *counts, const void *in, void *out,
                          int64_t rows, int32_t inverse, int32_t *expert_offsets, void *ws,
                          cudaStream_t stream) {
    moe_status st = moe_config_check(cfg);
    if (st != MOE_OK) return st;
    if ((st = check_ws(ws)) != MOE_OK) return st;
    const moe_config &c = *cfg;
    if (c.ffn_fp8) return fail(MOE_ERR_UNSUPPORTED, "the EP regroup moves bf16 / fp32 rows (ffn_fp8 = 0)");
    if (rows < 0) return fail(MOE_ERR_INVALID_ARG, "rows < 0");
    if (inverse != 0 && inverse != 1) return fail(MOE_ERR_INVALID_ARG, "inverse must be 0 or 1");
    if (rows == 0) {
        if (expert_offsets) {
            cudaError_t err = cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (size_t)(c.E / c.ep + 1), stream);
            if (err != cudaSuccess) return cuda_fail(err, "moe_ep_regroup");
        }
        return MOE_OK;
    }
    if (!counts || !in || !out) return fail(MOE_ERR_INVALID_ARG, "NULL pointer argument");
    if (in == out) return fail(MOE_ERR_INVALID_ARG, "in and out must not be the same buffer");
    const int row_bytes = c.H * (c.dtype == MOE_F32 ? 4 : 2);
    if (row_bytes % 16 != 0) return fail(MOE_ERR_UNSUPPORTED, "rows of %d bytes: a multiple of 16 is needed", row_bytes);
    if (!aligned(in, 16) || !aligned(out, 16)) return fail(MOE_ERR_INVALID_ARG, "in / out not 16-byte aligned");
    if (!aligned(counts, 4)) return fail(MOE_ERR_INVALID_ARG, "counts not 4-byte aligned");
    const ScratchLayout L = scratch_layout(c);
    cudaError_t err = launch_ep_regroup(c.ep, c.E / c.ep, counts, in, out, rows, row_bytes, inverse,
                                        expert_offsets, ws_at<uint32_t>(ws, L.status), stream, current_num_sms());
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_ep_regroup");
}

moe_status moe_device_status(void *ws, uint32_t *flags, cudaStream_t stream) {
    if (!ws || !flags) return fail(MOE_ERR_INVALID_ARG, "NULL pointer argument");
    uint32_t v = 0;
    cudaError_t err = cudaMemcpyAsync(&v, ws, sizeof v, cudaMemcpyDeviceToHost, stream);
    if (err == cudaSuccess) err = cudaStreamSynchronize(stream);
    if (err == cudaSuccess) err = cudaMemsetAsync(ws, 0, sizeof v, stream);
    if (err == cudaSuccess) err = cudaStreamSynchronize(stream);
    if (err != cudaSuccess) return cuda_fail(err, "moe_device_status");
    *flags = v;
    if (v) return fail(MOE_ERR_DEVICE, "device status bits 0x%x", v);
    return MOE_OK;
}

const char *moe_status_string(moe_status s) {
    switch (s) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
        case MOE_ERR_WORKSPACE: return "bad workspace";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_DEVICE: return "device-detected error";
    }
    return "unknown status";
}

const char *moe_last_error_detail(void) { return g_detail; }

}  // extern "C"
