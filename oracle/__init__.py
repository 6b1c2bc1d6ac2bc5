"""CPU oracle for the expert-parallel MoE layer hot path (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
and reference legs may import this package.  The product path never does.

The arithmetic lives in ``moe_oracle.c`` (plain single-threaded C, fp64 for the
FFN and combine, IEEE fp32 with explicit fma for the routing weights).  This
module only compiles it with gcc and marshals numpy arrays through ctypes.
bf16 tensors travel as uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import tempfile

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liborc.so")
CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]

ORC_OK, ORC_ERR_ARG, ORC_ERR_NONFINITE = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/_build/liborc.so`` (atomic rename)."""
    os.makedirs(_BUILD, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    fd, tmp = tempfile.mkstemp(suffix=".so", dir=_BUILD)
    os.close(fd)
    subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i = ctypes.c_int
        L.orc_exp_det.argtypes = [ctypes.c_float]
        L.orc_exp_det.restype = ctypes.c_float
        L.orc_route_topk.argtypes = [i, i, i, P, P, P, P, P]
        L.orc_route_topk.restype = i
        L.orc_route_topk_ex.argtypes = [i, i, i, P, P, i, i, i, i, P, P, P]
        L.orc_route_topk_ex.restype = i
        L.orc_capacity_clip.argtypes = [i, i, i, i, P, P, P, P]
        L.orc_capacity_clip.restype = i
        L.orc_dispatch_layout.argtypes = [i, i, i, i, i, i, P, P, P, P, P, P, P, P]
        L.orc_dispatch_layout.restype = i
        L.orc_permute.argtypes = [i, i, i, P, P, P]
        L.orc_permute.restype = None
        L.orc_ffn_row.argtypes = [i, i, i, P, P, P, i, P, P, P]
        L.orc_ffn_row.restype = None
        L.orc_combine.argtypes = [i, i, i, i, i, P, P, P, P, P]
        L.orc_combine.restype = None
        L.orc_combine_exact.argtypes = [i, i, i, i, i, P, P, P, P, P]
        L.orc_combine_exact.restype = None
        L.orc_bf16_from_double.argtypes = [ctypes.c_double]
        L.orc_bf16_from_double.restype = ctypes.c_uint16
        L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_decode.restype = ctypes.c_double
        L.orc_e4m3_encode.argtypes = [ctypes.c_double]
        L.orc_e4m3_encode.restype = ctypes.c_uint8
        L.orc_ue8m0_scale.argtypes = [ctypes.c_double]
        L.orc_ue8m0_scale.restype = ctypes.c_uint8
        L.orc_quantize_rows.argtypes = [ctypes.c_int64, i, i, P, P, P]
        L.orc_quantize_rows.restype = None
        L.orc_ffn_row_fp8.argtypes = [i, i, P, ctypes.c_uint8, P, P, P, P, P, P, P, P, P]
        L.orc_ffn_row_fp8.restype = None
        L.orc_ffn_row_bwd.argtypes = [i, i, i, P, P, P, P, P, P, P, P]
        L.orc_ffn_row_bwd.restype = None
        L.orc_layer_bwd.argtypes = [i, i, i, i, i, i, P, P, P, P, P, P, P, P, P, P, P, P]
        L.orc_layer_bwd.restype = None
        L.orc_quantize_blocks.argtypes = [ctypes.c_int64, i, i, i, P, P, P]
        L.orc_quantize_blocks.restype = None
        L.orc_dot_blocked.argtypes = [i, i, P, P, P, P]
        L.orc_dot_blocked.restype = ctypes.c_double
        L.orc_ffn_row_fp8_blocked.argtypes = [i, i, i, P, P, P, P, P, P, P, P, P, P, P]
        L.orc_ffn_row_fp8_blocked.restype = None
        L.orc_combine_bwd.argtypes = [i, i, i, i, i, P, P, P, P, P, P]
        L.orc_combine_bwd.restype = None
        L.orc_route_bwd.argtypes = [i, i, i, P, P, P, P]
        L.orc_route_bwd.restype = None
        _lib = L
    return _lib


def _p(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return 0
    if a.dtype == np.uint16:
        return 1
    if a.dtype == np.float64:
        return 2          # no rounding anywhere: the backward's finite-difference checks
    raise TypeError(f"storage arrays are float32, uint16 (bf16 bits) or float64, got {a.dtype}")


# --------------------------------------------------------------------------- steps

def exp_det(r: float) -> float:
    return float(lib().orc_exp_det(ctypes.c_float(float(r))))


def route_topk(logits: np.ndarray, bias: np.ndarray | None, k: int, n_group: int = 0,
               topk_group: int = 0, group_score: int = 0, bias_select_only: bool = False):
    """Returns (topk_idx int32 [T,k], topk_w float32 [T,k], counts int32 [E], status).

    n_group > 1 selects grouped top-k (topk_group groups kept per token by the
    best biased logit of a group, group_score 0, or the sum of its two best, 1);
    bias_select_only makes the bias steer the selection only."""
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = logits.shape
    if bias is not None:
        bias = np.ascontiguousarray(bias, dtype=np.float32)
    idx = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float32)
    counts = np.zeros(E, np.int32)
    st = lib().orc_route_topk_ex(T, E, k, _p(logits), _p(bias), int(n_group), int(topk_group),
                                 int(group_score), int(bool(bias_select_only)),
                                 _p(idx), _p(w), _p(counts))
    return idx, w, counts, st


def capacity_clip(topk_idx: np.ndarray, topk_w: np.ndarray, E: int, capacity: int):
    """Returns (keep uint8 [T,k], kept_counts int32 [E]).  capacity < 0: no cap."""
    topk_idx = np.ascontiguousarray(topk_idx, dtype=np.int32)
    topk_w = np.ascontiguousarray(topk_w, dtype=np.float32)
    T, k = topk_idx.shape
    keep = np.zeros((T, k), np.uint8)
    kept = np.zeros(E, np.int32)
    st = lib().orc_capacity_clip(T, E, k, int(capacity), _p(topk_idx), _p(topk_w), _p(keep), _p(kept))
    if st != ORC_OK:
        raise ValueError(f"orc_capacity_clip status {st}")
    return keep, kept


def dispatch_layout(topk_idx: np.ndarray, keep: np.ndarray, E: int, ep: int,
                    tok_begin: int = 0, tok_count: int | None = None) -> dict:
    topk_idx = np.ascontiguousarray(topk_idx, dtype=np.int32)
    keep = np.ascontiguousarray(keep, dtype=np.uint8)
    T, k = topk_idx.shape
    if tok_count is None:
        tok_count = T - tok_begin
    nmax = tok_count * k
    out = dict(
        expert_offsets=np.zeros(E + 1, np.int32),
        rank_offsets=np.zeros(ep + 1, np.int32),
        recv_token=np.full(max(nmax, 1), -1, np.int32),
        recv_slot=np.full(max(nmax, 1), -1, np.int32),
        pos=np.zeros((tok_count, k), np.int32),
        send_splits=np.zeros((ep, ep), np.int32),
    )
    n = lib().orc_dispatch_layout(T, E, k, ep, tok_begin, tok_count, _p(topk_idx), _p(keep),
                                  _p(out["expert_offsets"]), _p(out["rank_offsets"]),
                                  _p(out["recv_token"]), _p(out["recv_slot"]), _p(out["pos"]),
                                  _p(out["send_splits"]))
    if n < 0:
        raise ValueError("orc_dispatch_layout rejected its arguments")
    out["N"] = n
    out["recv_token"] = out["recv_token"][:n].copy()
    out["recv_slot"] = out["recv_slot"][:n].copy()
    return out


def permute(x: np.ndarray, recv_token: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x)
    recv_token = np.ascontiguousarray(recv_token, dtype=np.int32)
    T, H = x.shape
    N = recv_token.shape[0]
    xr = np.zeros((N, H), x.dtype)
    lib().orc_permute(H, x.dtype.itemsize, N, _p(x), _p(recv_token), _p(xr))
    return xr


def ffn_row(x_row: np.ndarray, w13_e: np.ndarray, w2_e: np.ndarray, round_h: bool = True):
    """One expert's SwiGLU FFN on one row.  Returns (h_store, y_store, y_exact)."""
    x_row = np.ascontiguousarray(x_row)
    w13_e = np.ascontiguousarray(w13_e)
    w2_e = np.ascontiguousarray(w2_e)
    dt = _dtype_code(x_row)
    assert _dtype_code(w13_e) == dt and _dtype_code(w2_e) == dt
    H = x_row.shape[0]
    I = w13_e.shape[0] // 2
    assert w13_e.shape == (2 * I, H) and w2_e.shape == (H, I)
    h = np.zeros(I, x_row.dtype)
    y = np.zeros(H, x_row.dtype)
    ye = np.zeros(H, np.float64)
    lib().orc_ffn_row(H, I, dt, _p(x_row), _p(w13_e), _p(w2_e), int(bool(round_h)), _p(h), _p(y), _p(ye))
    return h, y, ye


def ffn(xr: np.ndarray, expert_offsets: np.ndarray, w13: np.ndarray, w2: np.ndarray,
        round_h: bool = True):
    """FFN over a whole expert-contiguous buffer.  Returns (h, y, y_exact)."""
    N, H = xr.shape
    E = w13.shape[0]
    I = w13.shape[1] // 2
    h = np.zeros((N, I), xr.dtype)
    y = np.zeros((N, H), xr.dtype)
    ye = np.zeros((N, H), np.float64)
    for e in range(E):
        for p in range(int(expert_offsets[e]), int(expert_offsets[e + 1])):
            h[p], y[p], ye[p] = ffn_row(xr[p], w13[e], w2[e], round_h)
    return h, y, ye


def combine(y: np.ndarray, pos: np.ndarray, topk_w: np.ndarray, T: int,
            tok_begin: int = 0, out: np.ndarray | None = None,
            y_shared: np.ndarray | None = None) -> np.ndarray:
    """y_shared: the chunk's [tok_count, H] rows of the shared expert's output
    (same dtype as y), added into the sum before its rounding, or None."""
    y = np.ascontiguousarray(y)
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    topk_w = np.ascontiguousarray(topk_w, dtype=np.float32)
    dt = _dtype_code(y)
    H = y.shape[1]
    tok_count, k = pos.shape
    if out is None:
        out = np.zeros((T, H), y.dtype)
    if y_shared is not None:
        y_shared = np.ascontiguousarray(y_shared, dtype=y.dtype)
    lib().orc_combine(H, k, dt, tok_begin, tok_count, _p(y), _p(pos), _p(topk_w), _p(y_shared), _p(out))
    return out


def combine_exact(y_exact: np.ndarray, pos: np.ndarray, topk_w: np.ndarray, T: int,
                  out_dtype, tok_begin: int = 0, out: np.ndarray | None = None,
                  y_shared: np.ndarray | None = None) -> np.ndarray:
    y_exact = np.ascontiguousarray(y_exact, dtype=np.float64)
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    topk_w = np.ascontiguousarray(topk_w, dtype=np.float32)
    H = y_exact.shape[1]
    tok_count, k = pos.shape
    if out is None:
        out = np.zeros((T, H), out_dtype)
    dt = _dtype_code(out)
    if y_shared is not None:
        y_shared = np.ascontiguousarray(y_shared, dtype=out.dtype)
    lib().orc_combine_exact(H, k, dt, tok_begin, tok_count, _p(y_exact), _p(pos), _p(topk_w),
                            _p(y_shared), _p(out))
    return out


def bf16_bits_from_double(v: float) -> int:
    return int(lib().orc_bf16_from_double(float(v)))


# --------------------------------------------------------------------------- FP8 FFN

def e4m3_decode(codes) -> np.ndarray:
    """E4M3 codes (uint8) -> their values (float64; NaN for the NaN codes)."""
    c = np.asarray(codes, np.uint8)
    f = lib().orc_e4m3_decode
    return np.array([f(int(v)) for v in c.ravel()], np.float64).reshape(c.shape)


def e4m3_encode(values) -> np.ndarray:
    """Nearest E4M3 code, ties to even, saturating at +-448."""
    v = np.asarray(values, np.float64)
    f = lib().orc_e4m3_encode
    return np.array([f(float(a)) for a in v.ravel()], np.uint8).reshape(v.shape)


def ue8m0_scale(amax: float) -> int:
    """Biased exponent byte of the smallest 2^e with amax <= 448 * 2^e."""
    return int(lib().orc_ue8m0_scale(float(amax)))


def quantize_rows(a: np.ndarray):
    """Row-wise FP8 quantisation of a float32 or bf16-bits [rows, cols] array.
    Returns (codes uint8 [rows, cols], scales uint8 [rows])."""
    a = np.ascontiguousarray(a)
    dt = _dtype_code(a)
    rows, cols = a.shape
    codes = np.zeros((rows, cols), np.uint8)
    scales = np.zeros(rows, np.uint8)
    lib().orc_quantize_rows(rows, cols, dt, _p(a), _p(codes), _p(scales))
    return codes, scales


def quantize_blocks(a: np.ndarray, block: int = 128):
    """FP8 quantisation with one UE8M0 scale per row and per block of `block`
    columns.  Returns (codes uint8 [rows, cols], scales uint8 [rows, ceil(cols/block)])."""
    a = np.ascontiguousarray(a)
    dt = _dtype_code(a)
    rows, cols = a.shape
    nb = (cols + block - 1) // block
    codes = np.zeros((rows, cols), np.uint8)
    scales = np.zeros((rows, nb), np.uint8)
    lib().orc_quantize_blocks(rows, cols, block, dt, _p(a), _p(codes), _p(scales))
    return codes, scales


def dot_blocked(a_codes, a_scales, b_codes, b_scales, block: int = 128) -> float:
    """<dequant(a), dequant(b)> for two K-blocked FP8 rows, block by block."""
    a_codes = np.ascontiguousarray(a_codes, np.uint8)
    b_codes = np.ascontiguousarray(b_codes, np.uint8)
    a_scales = np.ascontiguousarray(a_scales, np.uint8)
    b_scales = np.ascontiguousarray(b_scales, np.uint8)
    return float(lib().orc_dot_blocked(a_codes.shape[0], block, _p(a_codes), _p(a_scales),
                                       _p(b_codes), _p(b_scales)))


def dequantize_rows(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    return e4m3_decode(codes) * np.ldexp(1.0, scales.astype(np.int32) - 127)[:, None]


def ffn_row_fp8(x_codes, x_scale, w13_codes, w13_scales, w2_codes, w2_scales):
    """One expert's FP8 SwiGLU FFN on one row.  Returns
    (h bf16 bits [I], hq codes [I], h scale byte, y bf16 bits [H], y_exact [H])."""
    x_codes = np.ascontiguousarray(x_codes, np.uint8)
    w13_codes = np.ascontiguousarray(w13_codes, np.uint8)
    w13_scales = np.ascontiguousarray(w13_scales, np.uint8)
    w2_codes = np.ascontiguousarray(w2_codes, np.uint8)
    w2_scales = np.ascontiguousarray(w2_scales, np.uint8)
    H = x_codes.shape[0]
    I = w13_codes.shape[0] // 2
    assert w13_codes.shape == (2 * I, H) and w2_codes.shape == (H, I)
    assert w13_scales.shape == (2 * I,) and w2_scales.shape == (H,)
    h = np.zeros(I, np.uint16)
    hq = np.zeros(I, np.uint8)
    sh = ctypes.c_uint8(0)
    y = np.zeros(H, np.uint16)
    ye = np.zeros(H, np.float64)
    lib().orc_ffn_row_fp8(H, I, _p(x_codes), int(x_scale), _p(w13_codes), _p(w13_scales),
                          _p(w2_codes), _p(w2_scales), _p(h), _p(hq), ctypes.byref(sh), _p(y), _p(ye))
    return h, hq, int(sh.value), y, ye


def ffn_row_fp8_blocked(x_codes, x_scales, w13_codes, w13_scales, w2_codes, w2_scales, block=32):
    """One expert's FP8 SwiGLU FFN on one row with K-blocked scales (one UE8M0
    scale per row and per `block` K values; h quantised by blocks of I).  Returns
    (h bf16 bits [I], hq codes [I], h scales [I/block], y bf16 bits [H], y_exact [H])."""
    x_codes = np.ascontiguousarray(x_codes, np.uint8)
    x_scales = np.ascontiguousarray(x_scales, np.uint8)
    w13_codes = np.ascontiguousarray(w13_codes, np.uint8)
    w13_scales = np.ascontiguousarray(w13_scales, np.uint8)
    w2_codes = np.ascontiguousarray(w2_codes, np.uint8)
    w2_scales = np.ascontiguousarray(w2_scales, np.uint8)
    H = x_codes.shape[0]
    I = w13_codes.shape[0] // 2
    nbh, nbi = -(-H // block), -(-I // block)
    assert w13_codes.shape == (2 * I, H) and w2_codes.shape == (H, I)
    assert x_scales.shape == (nbh,) and w13_scales.shape == (2 * I, nbh) and w2_scales.shape == (H, nbi)
    h = np.zeros(I, np.uint16)
    hq = np.zeros(I, np.uint8)
    hs = np.zeros(nbi, np.uint8)
    y = np.zeros(H, np.uint16)
    ye = np.zeros(H, np.float64)
    lib().orc_ffn_row_fp8_blocked(H, I, block, _p(x_codes), _p(x_scales), _p(w13_codes), _p(w13_scales),
                                  _p(w2_codes), _p(w2_scales), _p(h), _p(hq), _p(hs), _p(y), _p(ye))
    return h, hq, hs, y, ye


# --------------------------------------------------------------------------- backward

def ffn_row_backward(x_row, w13_e, w2_e, dy):
    """One expert's SwiGLU FFN backward on one row.  Returns (dx [H], dW13 [2I, H],
    dW2 [H, I], y [H]) in float64."""
    x_row = np.ascontiguousarray(x_row)
    w13_e = np.ascontiguousarray(w13_e)
    w2_e = np.ascontiguousarray(w2_e)
    dt = _dtype_code(x_row)
    H = x_row.shape[0]
    I = w13_e.shape[0] // 2
    dy = np.ascontiguousarray(dy, np.float64)
    dx = np.zeros(H, np.float64)
    dW13 = np.zeros((2 * I, H), np.float64)
    dW2 = np.zeros((H, I), np.float64)
    y = np.zeros(H, np.float64)
    lib().orc_ffn_row_bwd(H, I, dt, _p(x_row), _p(w13_e), _p(w2_e), _p(dy), _p(dx), _p(dW13),
                          _p(dW2), _p(y))
    return dx, dW13, dW2, y


def ffn_backward(xr, expert_offsets, w13, w2, dy):
    """The grouped SwiGLU FFN's backward over an expert-contiguous receive buffer:
    for every row p of expert e, the row backward of orc_ffn_row_bwd with dy[p].
    Returns float64 (dxr [N, H], dW13 [E, 2I, H], dW2 [E, H, I])."""
    xr = np.ascontiguousarray(xr)
    dy = np.ascontiguousarray(dy, np.float64)
    N, H = xr.shape
    E = w13.shape[0]
    I = w13.shape[1] // 2
    dxr = np.zeros((N, H), np.float64)
    dW13 = np.zeros((E, 2 * I, H), np.float64)
    dW2 = np.zeros((E, H, I), np.float64)
    for e in range(E):
        for p in range(int(expert_offsets[e]), int(expert_offsets[e + 1])):
            dx, a, b, _ = ffn_row_backward(xr[p], w13[e], w2[e], dy[p])
            dxr[p] = dx
            dW13[e] += a
            dW2[e] += b
    return dxr, dW13, dW2


def combine_backward(dout, y, pos, topk_w, tok_begin: int = 0):
    """Backward of the combine for the chunk's tokens: (dy [N, H] in y's storage
    type, zero on rows no slot points to; dw [T, k] float64, zero outside the chunk
    and for dropped slots)."""
    dout = np.ascontiguousarray(dout)
    y = np.ascontiguousarray(y)
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    topk_w = np.ascontiguousarray(topk_w, dtype=np.float32)
    dt = _dtype_code(y)
    assert _dtype_code(dout) == dt
    tok_count, k = pos.shape
    H = y.shape[1]
    dy = np.zeros_like(y)
    dw = np.zeros(topk_w.shape, np.float64)
    lib().orc_combine_bwd(H, k, dt, tok_begin, tok_count, _p(dout), _p(y), _p(pos), _p(topk_w),
                          _p(dy), _p(dw))
    return dy, dw


def route_backward(topk_idx, topk_w, dw, E: int):
    """dlogits [T, E] (float64) from dw [T, k] through the softmax over the selected."""
    topk_idx = np.ascontiguousarray(topk_idx, dtype=np.int32)
    topk_w = np.ascontiguousarray(topk_w, dtype=np.float32)
    dw = np.ascontiguousarray(dw, dtype=np.float64)
    T, k = topk_idx.shape
    dl = np.zeros((T, E), np.float64)
    lib().orc_route_bwd(T, E, k, _p(topk_idx), _p(topk_w), _p(dw), _p(dl))
    return dl


def moe_layer_backward(logits, bias, x, w13, w2, k: int, ep: int, dout, capacity: int = -1,
                       n_chunks: int = 1, n_group: int = 0, topk_group: int = 0,
                       group_score: int = 0, bias_select_only: bool = False,
                       w13_shared=None, w2_shared=None, save_dispatch: bool = False) -> dict:
    """Gradient of L = <dout, out> for the layer of moe_layer (axolotl
    expert_parallel_save_dispatch): the routing top-k, keep mask and layouts are
    what the forward saved; with save_dispatch the expert rows are read from the
    forward's receive buffers (the saved dispatch outputs), otherwise they are
    recomputed from x (the same values).  Returns float64 dx [T, H], dlogits
    [T, E], dbias [E] (zero when the bias steers the selection only), dW13,
    dW2 and, with a shared expert, dW13_shared, dW2_shared; and the saved
    routing."""
    T, E = logits.shape
    H = x.shape[1]
    I = w13.shape[1] // 2
    dt = _dtype_code(x)
    idx, w, _, st = route_topk(logits, bias, k, n_group, topk_group, group_score, bias_select_only)
    if st != ORC_OK:
        raise ValueError(f"route_topk status {st}")
    keep, _ = capacity_clip(idx, w, E, capacity)
    if save_dispatch:
        # the forward's receive rows, chunk after chunk, and each slot's row in them
        tc = T // n_chunks
        rows, row_of, base = [], np.zeros((T, k), np.int32), 0
        for c in range(n_chunks):
            lay = dispatch_layout(idx, keep, E, ep, c * tc, tc)
            rows.append(permute(x, lay["recv_token"]))
            pos = lay["pos"]
            row_of[c * tc:(c + 1) * tc] = np.where(pos >= 0, pos + base, 0)
            base += lay["N"]
        x_rows = np.ascontiguousarray(np.concatenate(rows) if base > 0 else x[:1])
    else:
        x_rows = x
        row_of = np.repeat(np.arange(T, dtype=np.int32)[:, None], k, axis=1)
    dout = np.ascontiguousarray(dout, np.float64)
    dx = np.zeros((T, H), np.float64)
    dz = np.zeros((T, k), np.float64)
    dW13 = np.zeros((E, 2 * I, H), np.float64)
    dW2 = np.zeros((E, H, I), np.float64)
    lib().orc_layer_bwd(T, H, E, k, I, dt, _p(idx), _p(w), _p(keep), _p(x_rows),
                        _p(np.ascontiguousarray(row_of)), _p(np.ascontiguousarray(w13)),
                        _p(np.ascontiguousarray(w2)), _p(dout), _p(dx), _p(dz), _p(dW13), _p(dW2))
    dlogits = np.zeros((T, E), np.float64)
    np.add.at(dlogits, (np.repeat(np.arange(T), k), idx.ravel()), dz.ravel())
    dbias = np.zeros(E, np.float64) if bias is None or bias_select_only else dlogits.sum(axis=0)
    res = dict(dx=dx, dlogits=dlogits, dbias=dbias, dW13=dW13, dW2=dW2, topk_idx=idx, topk_w=w,
               keep=keep)
    if w13_shared is not None:
        # the shared expert: every token, weight 1 (one expert, one slot)
        Is = w13_shared.shape[0] // 2
        dW13s = np.zeros((1, 2 * Is, H), np.float64)
        dW2s = np.zeros((1, H, Is), np.float64)
        ones = np.ones((T, 1), np.float32)
        lib().orc_layer_bwd(T, H, 1, 1, Is, dt, _p(np.zeros((T, 1), np.int32)), _p(ones),
                            _p(np.ones((T, 1), np.uint8)), _p(np.ascontiguousarray(x)),
                            _p(np.arange(T, dtype=np.int32)[:, None].copy()),
                            _p(np.ascontiguousarray(w13_shared)), _p(np.ascontiguousarray(w2_shared)),
                            _p(dout), _p(dx), _p(np.zeros((T, 1), np.float64)), _p(dW13s), _p(dW2s))
        res.update(dW13_shared=dW13s[0], dW2_shared=dW2s[0])
    return res


# --------------------------------------------------------------------------- whole layer

def shared_expert(x: np.ndarray, w13s: np.ndarray, w2s: np.ndarray):
    """The shared expert over the rows of x: one expert's FFN (w13s [2I_s, H],
    w2s [H, I_s]) applied to every row.  Returns (h, y, y_exact) like ffn()."""
    T = x.shape[0]
    return ffn(x, np.array([0, T], np.int32), w13s[None], w2s[None])


def moe_layer(logits, bias, x, w13, w2, k: int, ep: int, capacity: int = -1,
              n_chunks: int = 1, reduce_dense: bool = False, n_group: int = 0,
              topk_group: int = 0, group_score: int = 0, bias_select_only: bool = False,
              w13_shared=None, w2_shared=None) -> dict:
    """All six steps in the order the pages give them, chunk by chunk.

    Route and clip run once over all T tokens (the capacity is per forward);
    layout, permute, FFN and combine run per contiguous token chunk (axolotl
    expert_parallel_dispatch_chunks).  Returns every intermediate.
    """
    T, E = logits.shape
    idx, w, counts, st = route_topk(logits, bias, k, n_group, topk_group, group_score, bias_select_only)
    if st != ORC_OK:
        raise ValueError(f"route_topk status {st}")
    keep, kept = capacity_clip(idx, w, E, capacity)
    out = np.zeros((T, x.shape[1]), x.dtype)
    chunks = []
    tc = T // n_chunks
    for c in range(n_chunks):
        tb = c * tc
        lay = dispatch_layout(idx, keep, E, ep, tb, tc)
        xr = permute(x, lay["recv_token"])
        h, y, ye = ffn(xr, lay["expert_offsets"], w13, w2)
        ys = None
        if w13_shared is not None:
            _, ys, _ = shared_expert(x[tb:tb + tc], w13_shared, w2_shared)
        if reduce_dense:
            combine_exact(ye, lay["pos"], w, T, x.dtype, tb, out, y_shared=ys)
        else:
            combine(y, lay["pos"], w, T, tb, out, y_shared=ys)
        chunks.append(dict(layout=lay, xr=xr, h=h, y=y, y_exact=ye, y_shared=ys))
    return dict(topk_idx=idx, topk_w=w, counts=counts, keep=keep, kept_counts=kept,
                chunks=chunks, out=out)
