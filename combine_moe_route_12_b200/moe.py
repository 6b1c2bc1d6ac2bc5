"""ctypes binding over libmoe_b200.so (include/moe_b200.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  Tensors are torch CUDA tensors (device pointers are taken with
``data_ptr()``); ``stream`` defaults to torch's current stream.  Importing
this module raises if the library has not been built.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

from .build import LIB, ROOT

if not os.path.exists(LIB):
    raise ImportError(f"{LIB} is missing: build it with `python -m combine_moe_route_12_b200.build`")

_lib = ctypes.CDLL(LIB)

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_DEVICE = range(6)
MOE_F32, MOE_BF16 = 0, 1
MOE_DEV_NONFINITE_LOGIT = 0x1
MOE_DEV_WAIT_TIMEOUT = 0x2
MOE_DEV_BAD_INDEX = 0x4


class MoEConfig(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("T", "H", "E", "k", "I", "ep", "capacity", "dtype", "n_chunks", "reduce_dense",
                 "n_group", "topk_group", "group_score", "bias_select_only", "shared_I",
                 "ffn_fp8")]

    def __repr__(self):
        return "MoEConfig(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


class MoEError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"{status_string(status)} ({status}): {detail}")
        self.status = status


_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_CFG = ctypes.POINTER(MoEConfig)


def _decl(name, restype, *argtypes):
    f = getattr(_lib, name)
    f.restype = restype
    f.argtypes = list(argtypes)
    return f


_decl("moe_config_check", _I32, _CFG)
_decl("moe_workspace_bytes", ctypes.c_size_t, _CFG)
_decl("moe_forward_workspace_bytes", ctypes.c_size_t, _CFG)
_decl("moe_max_recv_rows", ctypes.c_int64, _CFG, _I32)
_decl("moe_route_topk", _I32, _CFG, _P, _P, _P, _P, _P, _P, _P)
_decl("moe_capacity_clip", _I32, _CFG, _P, _P, _P, _P, _P, _P, _P)
_decl("moe_dispatch_layout", _I32, _CFG, _I32, _I32, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P)
_decl("moe_dispatch_layout_noalloc", _I32, _CFG, _I32, _I32, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P)
_decl("moe_permute", _I32, _CFG, _P, _P, _I32, _I32, _P, _P)
_decl("moe_grouped_swiglu_ffn", _I32, _CFG, ctypes.c_int64, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P)
_decl("moe_combine", _I32, _CFG, _P, _P, _P, _I32, _I32, _P, _P, _P)
_decl("moe_reduce_finalize", _I32, _CFG, _P, _I32, _I32, _P, _P, _P)
_decl("moe_shared_expert_ffn", _I32, _CFG, _I32, _I32, _P, _P, _P, _P, _P, _P, _P)
_decl("moe_forward_chunked", _I32, _CFG, *([_P] * 17))
_decl("moe_forward_chunked_save", _I32, _CFG, *([_P] * 17))
_decl("moe_backward_workspace_bytes", ctypes.c_size_t, _CFG)
_decl("moe_layer_backward", _I32, _CFG, *([_P] * 18), _I32, _P, _P)
_decl("moe_forward_host_workspace_bytes", ctypes.c_size_t, _CFG)
_decl("moe_forward_host", _I32, _CFG, *([_P] * 17))
_decl("moe_quantize_fp8_rows", _I32, ctypes.c_int64, _I32, _I32, _P, _P, _P, _P)
_decl("moe_grouped_swiglu_ffn_fp8", _I32, _CFG, ctypes.c_int64, *([_P] * 17))
_decl("moe_permute_quantize_fp8", _I32, _CFG, _P, _P, _I32, _I32, _P, _P, _P)
_decl("moe_quantize_fp8_blocks", _I32, ctypes.c_int64, _I32, _I32, _P, _P, _P, _P)
_decl("moe_permute_quantize_fp8_blocks", _I32, _CFG, _P, _P, _I32, _I32, _P, _P, _P)
_decl("moe_grouped_swiglu_ffn_mxfp8", _I32, _CFG, ctypes.c_int64, *([_P] * 14), _P, _P)
_decl("moe_grouped_swiglu_ffn_backward", _I32, _CFG, ctypes.c_int64, *([_P] * 11), _I32, _P, _P)
_decl("moe_combine_backward", _I32, _CFG, _P, _P, _P, _P, _I32, _I32, _P, _P, _P)
_decl("moe_route_backward", _I32, _CFG, _P, _P, _P, _P, _P, _P, _P)
_decl("moe_permute_backward", _I32, _CFG, _P, _P, _I32, _I32, _P, _P)
_decl("moe_watchdog_selftest", _I32, _CFG, _I32, _I32, _P, _P)
_decl("moe_ep_regroup", _I32, _CFG, _P, _P, _P, ctypes.c_int64, ctypes.c_int32, _P, _P, _P)
_decl("moe_device_status", _I32, _P, ctypes.POINTER(ctypes.c_uint32), _P)
_decl("moe_status_string", ctypes.c_char_p, _I32)
_decl("moe_last_error_detail", ctypes.c_char_p)


def header_symbols() -> list[str]:
    """Entry points declared in include/moe_b200.h."""
    text = open(os.path.join(ROOT, "include", "moe_b200.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text)))


def status_string(status: int) -> str:
    return _lib.moe_status_string(status).decode()


def last_error_detail() -> str:
    return _lib.moe_last_error_detail().decode()


def _check(status: int) -> None:
    if status != MOE_OK:
        raise MoEError(status, last_error_detail())


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return ctypes.c_void_p(t)
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def make_config(T, H, E, k, I, ep, capacity=-1, dtype=MOE_BF16, n_chunks=1,
                reduce_dense=False, n_group=0, topk_group=0, group_score=0,
                bias_select_only=False, shared_I=0, ffn_fp8=False) -> MoEConfig:
    if isinstance(dtype, str):
        dtype = MOE_F32 if dtype == "f32" else MOE_BF16
    return MoEConfig(T, H, E, k, I, ep, -1 if capacity is None else capacity, dtype, n_chunks,
                     int(bool(reduce_dense)), n_group, topk_group, group_score,
                     int(bool(bias_select_only)), shared_I, int(ffn_fp8))


def config_from_workload(wl) -> MoEConfig:
    return make_config(wl.T, wl.H, wl.E, wl.k, wl.I, wl.ep, wl.capacity, wl.dtype, wl.n_chunks,
                       wl.reduce_dense, wl.n_group, wl.topk_group, wl.group_score,
                       wl.bias_select_only, wl.shared_I, wl.ffn_fp8)


# ------------------------------------------------------------------ sizes

def config_check(cfg: MoEConfig) -> None:
    _check(_lib.moe_config_check(ctypes.byref(cfg)))


def workspace_bytes(cfg: MoEConfig) -> int:
    return int(_lib.moe_workspace_bytes(ctypes.byref(cfg)))


def forward_workspace_bytes(cfg: MoEConfig) -> int:
    return int(_lib.moe_forward_workspace_bytes(ctypes.byref(cfg)))


def forward_host_workspace_bytes(cfg: MoEConfig) -> int:
    return int(_lib.moe_forward_host_workspace_bytes(ctypes.byref(cfg)))


def max_recv_rows(cfg: MoEConfig, tok_count: int) -> int:
    return int(_lib.moe_max_recv_rows(ctypes.byref(cfg), tok_count))


def alloc_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """Zero-filled workspace (torch allocations are 256-byte aligned)."""
    return torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=device)


# ------------------------------------------------------------------ the six steps

def moe_route_topk(cfg, logits, bias, topk_idx, topk_w, counts, ws, stream=None):
    _check(_lib.moe_route_topk(ctypes.byref(cfg), _ptr(logits), _ptr(bias), _ptr(topk_idx),
                               _ptr(topk_w), _ptr(counts), _ptr(ws), _stream(stream)))


def moe_capacity_clip(cfg, topk_idx, topk_w, counts, keep, kept_counts, ws, stream=None):
    _check(_lib.moe_capacity_clip(ctypes.byref(cfg), _ptr(topk_idx), _ptr(topk_w), _ptr(counts),
                                  _ptr(keep), _ptr(kept_counts), _ptr(ws), _stream(stream)))


def moe_dispatch_layout(cfg, tok_begin, tok_count, topk_idx, keep, expert_offsets, rank_offsets,
                        recv_token, recv_slot, pos, send_splits, splits_host, ws, stream=None):
    _check(_lib.moe_dispatch_layout(ctypes.byref(cfg), tok_begin, tok_count, _ptr(topk_idx),
                                    _ptr(keep), _ptr(expert_offsets), _ptr(rank_offsets),
                                    _ptr(recv_token), _ptr(recv_slot), _ptr(pos),
                                    _ptr(send_splits), _ptr(splits_host), _ptr(ws),
                                    _stream(stream)))


def moe_dispatch_layout_noalloc(cfg, tok_begin, tok_count, topk_idx, keep, expert_offsets,
                                rank_offsets, recv_token, recv_slot, pos, send_splits, splits_host,
                                status=None, stream=None):
    """moe_dispatch_layout without a workspace: for callers that cannot
    allocate device memory (see include/moe_b200.h).  Its scratch is one
    library-owned device array shared by every call, so calls must not overlap."""
    _check(_lib.moe_dispatch_layout_noalloc(ctypes.byref(cfg), tok_begin, tok_count, _ptr(topk_idx),
                                            _ptr(keep), _ptr(expert_offsets), _ptr(rank_offsets),
                                            _ptr(recv_token), _ptr(recv_slot), _ptr(pos),
                                            _ptr(send_splits), _ptr(splits_host), _ptr(status),
                                            _stream(stream)))


def moe_permute(cfg, x, pos, tok_begin, tok_count, xr, stream=None):
    _check(_lib.moe_permute(ctypes.byref(cfg), _ptr(x), _ptr(pos), tok_begin, tok_count, _ptr(xr),
                            _stream(stream)))


def moe_grouped_swiglu_ffn(cfg, n_rows, xr, expert_offsets, w13, w2, h, y, recv_token,
                           recv_slot, topk_w, out_reduce, ws, stream=None):
    _check(_lib.moe_grouped_swiglu_ffn(ctypes.byref(cfg), n_rows, _ptr(xr), _ptr(expert_offsets),
                                       _ptr(w13), _ptr(w2), _ptr(h), _ptr(y), _ptr(recv_token),
                                       _ptr(recv_slot), _ptr(topk_w), _ptr(out_reduce), _ptr(ws),
                                       _stream(stream)))


def moe_quantize_fp8_rows(inp, codes, scales, stream=None):
    """Row-wise E4M3 codes and UE8M0 scale bytes of a bf16 or fp32 [rows, cols] tensor."""
    rows, cols = inp.shape
    in_dtype = MOE_BF16 if inp.dtype == torch.bfloat16 else MOE_F32
    assert codes.dtype == torch.uint8 and scales.dtype == torch.uint8
    assert tuple(codes.shape) == (rows, cols) and scales.numel() >= rows
    _check(_lib.moe_quantize_fp8_rows(rows, cols, in_dtype, _ptr(inp), _ptr(codes), _ptr(scales),
                                      _stream(stream)))


def quantize_fp8(inp, stream=None):
    """(codes, scales) of moe_quantize_fp8_rows over the last dimension of inp."""
    flat = inp.reshape(-1, inp.shape[-1])
    codes = torch.empty(flat.shape, dtype=torch.uint8, device=inp.device)
    scales = torch.empty(flat.shape[0], dtype=torch.uint8, device=inp.device)
    moe_quantize_fp8_rows(flat, codes, scales, stream)
    return codes.view(inp.shape), scales.view(inp.shape[:-1])


def moe_quantize_fp8_blocks(inp, codes, scales, stream=None):
    """E4M3 codes and one UE8M0 scale byte per 32 values of each row of a bf16 or
    fp32 [rows, cols] tensor (scales [rows, cols / 32])."""
    rows, cols = inp.shape
    in_dtype = MOE_BF16 if inp.dtype == torch.bfloat16 else MOE_F32
    assert codes.dtype == torch.uint8 and scales.dtype == torch.uint8
    assert tuple(codes.shape) == (rows, cols) and scales.numel() >= rows * (cols // 32)
    _check(_lib.moe_quantize_fp8_blocks(rows, cols, in_dtype, _ptr(inp), _ptr(codes), _ptr(scales),
                                        _stream(stream)))


def quantize_fp8_blocks(inp, stream=None):
    """(codes, scales [..., cols / 32]) of moe_quantize_fp8_blocks over the last dimension."""
    flat = inp.reshape(-1, inp.shape[-1])
    codes = torch.empty(flat.shape, dtype=torch.uint8, device=inp.device)
    scales = torch.empty(flat.shape[0], flat.shape[1] // 32, dtype=torch.uint8, device=inp.device)
    moe_quantize_fp8_blocks(flat, codes, scales, stream)
    return codes.view(inp.shape), scales.view(*inp.shape[:-1], inp.shape[-1] // 32)


def moe_permute_quantize_fp8_blocks(cfg, x, pos, tok_begin, tok_count, xr_q, xr_sf, stream=None):
    """Kept token rows of x quantised by 32-value blocks; codes and scales to their receive rows."""
    _check(_lib.moe_permute_quantize_fp8_blocks(ctypes.byref(cfg), _ptr(x), _ptr(pos), tok_begin,
                                                tok_count, _ptr(xr_q), _ptr(xr_sf), _stream(stream)))


def moe_grouped_swiglu_ffn_mxfp8(cfg, n_rows, xr_q, xr_sf, expert_offsets, w13_q, w13_sf, w2_q, w2_sf,
                                 h_q, h_sf, y, recv_token, recv_slot, topk_w, out_reduce, ws, stream=None):
    _check(_lib.moe_grouped_swiglu_ffn_mxfp8(
        ctypes.byref(cfg), n_rows, _ptr(xr_q), _ptr(xr_sf), _ptr(expert_offsets), _ptr(w13_q),
        _ptr(w13_sf), _ptr(w2_q), _ptr(w2_sf), _ptr(h_q), _ptr(h_sf), _ptr(y), _ptr(recv_token),
        _ptr(recv_slot), _ptr(topk_w), _ptr(out_reduce), _ptr(ws), _stream(stream)))


def moe_permute_quantize_fp8(cfg, x, pos, tok_begin, tok_count, xr_q, x_scale, stream=None):
    """Kept token rows of x quantised to E4M3 codes and written to their receive rows."""
    _check(_lib.moe_permute_quantize_fp8(ctypes.byref(cfg), _ptr(x), _ptr(pos), tok_begin,
                                         tok_count, _ptr(xr_q), _ptr(x_scale), _stream(stream)))


def moe_grouped_swiglu_ffn_backward(cfg, n_rows, xr, dy, expert_offsets, w13, w2, gu, h, dgu, dxr,
                                    dw13, dw2, accumulate, ws, stream=None):
    """The expert FFN's backward over one receive buffer: dxr, the recomputed h,
    [dg | du], and the fp32 weight gradients (written, or added to with accumulate)."""
    _check(_lib.moe_grouped_swiglu_ffn_backward(
        ctypes.byref(cfg), n_rows, _ptr(xr), _ptr(dy), _ptr(expert_offsets), _ptr(w13), _ptr(w2),
        _ptr(gu), _ptr(h), _ptr(dgu), _ptr(dxr), _ptr(dw13), _ptr(dw2), int(accumulate), _ptr(ws),
        _stream(stream)))


def moe_combine_backward(cfg, dout, y, pos, topk_w, tok_begin, tok_count, dy, dw, stream=None):
    """dy[pos] = w * dout and dw = <dout, y[pos]> for the chunk's kept slots."""
    _check(_lib.moe_combine_backward(ctypes.byref(cfg), _ptr(dout), _ptr(y), _ptr(pos),
                                     _ptr(topk_w), tok_begin, tok_count, _ptr(dy), _ptr(dw),
                                     _stream(stream)))


def moe_route_backward(cfg, topk_idx, topk_w, dw, dlogits, dbias, ws, stream=None):
    """dlogits through the softmax over the selected logits; dbias its column sums."""
    _check(_lib.moe_route_backward(ctypes.byref(cfg), _ptr(topk_idx), _ptr(topk_w), _ptr(dw),
                                   _ptr(dlogits), _ptr(dbias), _ptr(ws), _stream(stream)))


def moe_permute_backward(cfg, dxr, pos, tok_begin, tok_count, dx, stream=None):
    """dx[t] = the sum of the token's kept receive rows of dxr."""
    _check(_lib.moe_permute_backward(ctypes.byref(cfg), _ptr(dxr), _ptr(pos), tok_begin,
                                     tok_count, _ptr(dx), _stream(stream)))


def moe_grouped_swiglu_ffn_fp8(cfg, n_rows, xr_q, x_scale, expert_offsets, w13_q, w13_scale, w2_q,
                               w2_scale, h, h_q, h_scale, y, recv_token, recv_slot, topk_w,
                               out_reduce, ws, stream=None):
    _check(_lib.moe_grouped_swiglu_ffn_fp8(
        ctypes.byref(cfg), n_rows, _ptr(xr_q), _ptr(x_scale), _ptr(expert_offsets), _ptr(w13_q),
        _ptr(w13_scale), _ptr(w2_q), _ptr(w2_scale), _ptr(h), _ptr(h_q), _ptr(h_scale), _ptr(y),
        _ptr(recv_token), _ptr(recv_slot), _ptr(topk_w), _ptr(out_reduce), _ptr(ws),
        _stream(stream)))


def moe_combine(cfg, y, pos, topk_w, tok_begin, tok_count, out, stream=None, y_shared=None):
    _check(_lib.moe_combine(ctypes.byref(cfg), _ptr(y), _ptr(pos), _ptr(topk_w), tok_begin,
                            tok_count, _ptr(y_shared), _ptr(out), _stream(stream)))


def moe_reduce_finalize(cfg, out_reduce, tok_begin, tok_count, out, stream=None, y_shared=None):
    _check(_lib.moe_reduce_finalize(ctypes.byref(cfg), _ptr(out_reduce), tok_begin, tok_count,
                                    _ptr(y_shared), _ptr(out), _stream(stream)))


def moe_shared_expert_ffn(cfg, tok_begin, tok_count, x, w13_shared, w2_shared, h_shared, y_shared,
                          ws, stream=None):
    _check(_lib.moe_shared_expert_ffn(ctypes.byref(cfg), tok_begin, tok_count, _ptr(x),
                                      _ptr(w13_shared), _ptr(w2_shared), _ptr(h_shared),
                                      _ptr(y_shared), _ptr(ws), _stream(stream)))


def moe_forward_chunked(cfg, logits, bias, x, w13, w2, out, topk_idx, topk_w, keep, splits_host,
                        ws, s_dispatch=None, s_compute=None, w13_shared=None, w2_shared=None,
                        w13_scale=None, w2_scale=None):
    _check(_lib.moe_forward_chunked(ctypes.byref(cfg), _ptr(logits), _ptr(bias), _ptr(x),
                                    _ptr(w13), _ptr(w2), _ptr(w13_shared), _ptr(w2_shared),
                                    _ptr(w13_scale), _ptr(w2_scale),
                                    _ptr(out), _ptr(topk_idx), _ptr(topk_w),
                                    _ptr(keep), _ptr(splits_host), _ptr(ws),
                                    _stream(s_dispatch), _stream(s_compute)))


def moe_forward_chunked_save(cfg, logits, bias, x, w13, w2, out, topk_idx, topk_w, keep, splits_host,
                             xr_save, y_save, ws, s_dispatch=None, s_compute=None, w13_shared=None,
                             w2_shared=None):
    """moe_forward_chunked that also writes every chunk's receive rows and expert
    outputs to xr_save / y_save ([n_chunks, N_max, H])."""
    _check(_lib.moe_forward_chunked_save(ctypes.byref(cfg), _ptr(logits), _ptr(bias), _ptr(x), _ptr(w13),
                                         _ptr(w2), _ptr(w13_shared), _ptr(w2_shared), _ptr(out),
                                         _ptr(topk_idx), _ptr(topk_w), _ptr(keep), _ptr(splits_host),
                                         _ptr(xr_save), _ptr(y_save), _ptr(ws), _stream(s_dispatch),
                                         _stream(s_compute)))


def backward_workspace_bytes(cfg: MoEConfig) -> int:
    return int(_lib.moe_backward_workspace_bytes(ctypes.byref(cfg)))


def moe_layer_backward(cfg, x, dout, w13, w2, topk_idx, topk_w, keep, dx, dlogits, dbias, dw13, dw2,
                       ws, xr_saved=None, y_saved=None, w13_shared=None, w2_shared=None,
                       dw13_shared=None, dw2_shared=None, accumulate=False, stream=None):
    """The layer's backward: with xr_saved / y_saved (from moe_forward_chunked_save)
    the dispatch outputs are read, without them recomputed."""
    _check(_lib.moe_layer_backward(ctypes.byref(cfg), _ptr(x), _ptr(dout), _ptr(w13), _ptr(w2),
                                   _ptr(w13_shared), _ptr(w2_shared), _ptr(topk_idx), _ptr(topk_w),
                                   _ptr(keep), _ptr(xr_saved), _ptr(y_saved), _ptr(dx), _ptr(dlogits),
                                   _ptr(dbias), _ptr(dw13), _ptr(dw2), _ptr(dw13_shared),
                                   _ptr(dw2_shared), int(bool(accumulate)), _ptr(ws), _stream(stream)))


def moe_forward_host(cfg, logits_host, bias_host, x_host, w13, w2, out_host, topk_idx, topk_w,
                     keep, splits_host, ws, s_dispatch=None, s_compute=None, w13_shared=None,
                     w2_shared=None, w13_scale=None, w2_scale=None):
    """The chunked layer with logits, bias, x and out in (pinned) host memory."""
    for t in (logits_host, bias_host, x_host, out_host):
        if t is not None and t.is_cuda:
            raise ValueError("moe_forward_host takes host tensors for logits, bias, x and out")
    _check(_lib.moe_forward_host(ctypes.byref(cfg), _ptr(logits_host), _ptr(bias_host),
                                 _ptr(x_host), _ptr(w13), _ptr(w2), _ptr(w13_shared),
                                 _ptr(w2_shared), _ptr(w13_scale), _ptr(w2_scale), _ptr(out_host), _ptr(topk_idx), _ptr(topk_w),
                                 _ptr(keep), _ptr(splits_host), _ptr(ws), _stream(s_dispatch),
                                 _stream(s_compute)))


def moe_watchdog_selftest(cfg, which: int, limit_us: int, ws, stream=None):
    """Runs one of the library's bounded waits on something that never completes
    (0: a cluster-scope mbarrier wait, 1: a CTA-scope mbarrier wait); it sets
    MOE_DEV_WAIT_TIMEOUT."""
    _check(_lib.moe_watchdog_selftest(ctypes.byref(cfg), which, limit_us, _ptr(ws), _stream(stream)))


def moe_ep_regroup(cfg, counts, inp, out, rows, inverse, ws, expert_offsets=None, stream=None):
    """Source-major receive rows -> expert-major (inverse = 0), or back (1); see
    include/moe_b200.h.  counts: device int32 [ep, E // ep]; expert_offsets: the
    expert-major buffer's local expert offsets [E // ep + 1] (written when given)."""
    _check(_lib.moe_ep_regroup(ctypes.byref(cfg), _ptr(counts), _ptr(inp), _ptr(out), ctypes.c_int64(rows),
                               ctypes.c_int32(int(inverse)), _ptr(expert_offsets), _ptr(ws), _stream(stream)))


def moe_device_status(ws, stream=None) -> int:
    """Synchronises the stream; returns and clears the device status bits."""
    flags = ctypes.c_uint32(0)
    st = _lib.moe_device_status(_ptr(ws), ctypes.byref(flags), _stream(stream))
    if st not in (MOE_OK, MOE_ERR_DEVICE):
        _check(st)
    return int(flags.value)


# ------------------------------------------------------------------ convenience

class MoELayer:
    """Owns the buffers of one layer shape and runs ``moe_forward_chunked``.

    Weights are the caller's ([E, 2I, H] and [E, H, I] in the layer dtype).
    Allocation goes through torch; the library allocates nothing.
    """

    def __init__(self, cfg: MoEConfig, device="cuda", host_splits: bool = True,
                 host_io: bool = False):
        config_check(cfg)
        self.cfg = cfg
        dev = torch.device(device)
        T, k = cfg.T, cfg.k
        # host_io: room to stage host activations, for forward_host
        nbytes = forward_host_workspace_bytes(cfg) if host_io else forward_workspace_bytes(cfg)
        self.host_io = host_io
        self.ws = alloc_workspace(nbytes, dev)
        self.topk_idx = torch.empty(T, k, dtype=torch.int32, device=dev)
        self.topk_w = torch.empty(T, k, dtype=torch.float32, device=dev)
        self.keep = torch.empty(T, k, dtype=torch.uint8, device=dev)
        n = cfg.n_chunks * (cfg.E + 1 + cfg.ep * cfg.ep)
        self.splits_host = torch.zeros(n, dtype=torch.int32, pin_memory=True) if host_splits else None
        self.s_dispatch = torch.cuda.Stream(device=dev)

    def forward(self, logits, bias, x, w13, w2, out, s_compute=None, w13_shared=None,
                w2_shared=None, w13_scale=None, w2_scale=None):
        """w13_scale, w2_scale: with cfg.ffn_fp8, w13 and w2 are E4M3 codes and
        these their UE8M0 row scales (quantize_fp8)."""
        s_compute = s_compute or torch.cuda.current_stream()
        moe_forward_chunked(self.cfg, logits, bias, x, w13, w2, out, self.topk_idx, self.topk_w,
                            self.keep, self.splits_host, self.ws, self.s_dispatch, s_compute,
                            w13_shared, w2_shared, w13_scale, w2_scale)
        return out

    def forward_host(self, logits_host, bias_host, x_host, w13, w2, out_host, s_compute=None,
                     w13_shared=None, w2_shared=None, w13_scale=None, w2_scale=None):
        """forward() with logits, bias, x and out in pinned host memory; out_host
        is valid once s_compute (or the dispatch stream) has been synchronised."""
        if not self.host_io:
            raise ValueError("MoELayer(host_io=True) is needed for forward_host")
        s_compute = s_compute or torch.cuda.current_stream()
        moe_forward_host(self.cfg, logits_host, bias_host, x_host, w13, w2, out_host,
                         self.topk_idx, self.topk_w, self.keep, self.splits_host, self.ws,
                         self.s_dispatch, s_compute, w13_shared, w2_shared, w13_scale, w2_scale)
        return out_host

    def splits(self, chunk: int):
        """Host copy of chunk `chunk`'s (expert_offsets, send_splits); valid after a sync."""
        c = self.cfg
        stride = c.E + 1 + c.ep * c.ep
        v = self.splits_host[chunk * stride:(chunk + 1) * stride]
        return v[:c.E + 1], v[c.E + 1:].view(c.ep, c.ep)
