"""Host-only checks of the C ABI: the library loads without a GPU, exports every
entry point the header declares, and its argument / topology checks
(axolotl ExpertParallelArgs, validate_expert_parallel_topology) reject what
they should.  No call here touches a device."""
import ctypes

import pytest

from combine_moe_route_12_b200 import build

build.build()
from combine_moe_route_12_b200 import moe  # noqa: E402
from combine_moe_route_12_b200.workload import WORKLOADS  # noqa: E402


def test_library_exports_every_header_symbol():
    lib = ctypes.CDLL(build.LIB)
    names = moe.header_symbols()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
    for required in ("moe_route_topk", "moe_capacity_clip", "moe_dispatch_layout",
                     "moe_permute", "moe_grouped_swiglu_ffn", "moe_combine",
                     "moe_forward_chunked"):
        assert required in names


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_workloads_pass_topology_checks(name):
    cfg = moe.config_from_workload(WORKLOADS[name])
    moe.config_check(cfg)
    assert moe.workspace_bytes(cfg) > 0
    assert moe.forward_workspace_bytes(cfg) >= moe.workspace_bytes(cfg)


def test_max_recv_rows_is_padded_worst_case():
    c = moe.make_config(256, 7168, 256, 8, 2048, 64, capacity=1024)
    assert moe.max_recv_rows(c, 256) == 256 * 8           # cap never binds
    c = moe.make_config(16384, 2048, 128, 8, 768, 4, capacity=1024)
    assert moe.max_recv_rows(c, 16384) == 128 * 1024      # cap binds
    c = moe.make_config(64, 128, 8, 2, 128, 2, capacity=0)
    assert moe.max_recv_rows(c, 64) == 0


@pytest.mark.parametrize("kw,status", [
    (dict(E=10, ep=4), moe.MOE_ERR_INVALID_ARG),           # E % ep
    (dict(T=100, ep=8), moe.MOE_ERR_INVALID_ARG),          # tokens per source rank
    (dict(T=96, n_chunks=5), moe.MOE_ERR_INVALID_ARG),     # T % n_chunks
    (dict(k=9, E=8, ep=1), moe.MOE_ERR_INVALID_ARG),       # k > E
    (dict(k=33, E=64), moe.MOE_ERR_UNSUPPORTED),
    (dict(E=2048, ep=2), moe.MOE_ERR_UNSUPPORTED),
    (dict(H=96), moe.MOE_ERR_UNSUPPORTED),                 # bf16 tiles need H % 64
    (dict(I=100), moe.MOE_ERR_UNSUPPORTED),
    (dict(dtype=7), moe.MOE_ERR_INVALID_ARG),
    (dict(n_chunks=0), moe.MOE_ERR_INVALID_ARG),
    (dict(ffn_fp8=True, dtype=moe.MOE_F32), moe.MOE_ERR_UNSUPPORTED),   # FP8 FFN needs bf16
    (dict(ffn_fp8=True, H=192), moe.MOE_ERR_UNSUPPORTED),               # and H, I % 128
    (dict(ffn_fp8=True, I=192), moe.MOE_ERR_UNSUPPORTED),
    (dict(ffn_fp8=True, shared_I=128), moe.MOE_ERR_UNSUPPORTED),        # no FP8 shared expert
])
def test_config_rejections(kw, status):
    base = dict(T=64, H=128, E=8, k=2, I=128, ep=2, capacity=-1, dtype=moe.MOE_BF16,
                n_chunks=1, reduce_dense=False)
    base.update(kw)
    cfg = moe.make_config(**base)
    with pytest.raises(moe.MoEError) as ei:
        moe.config_check(cfg)
    assert ei.value.status == status
    assert moe.last_error_detail()
    assert moe.workspace_bytes(cfg) == 0


def test_null_workspace_rejected_before_any_launch():
    cfg = moe.make_config(64, 128, 8, 2, 128, 2)
    st = moe._lib.moe_route_topk(ctypes.byref(cfg), None, None, None, None, None, None, None)
    assert st == moe.MOE_ERR_WORKSPACE
    st = moe._lib.moe_dispatch_layout(ctypes.byref(cfg), 0, 60, None, None, None, None, None,
                                      None, None, None, None, ctypes.c_void_p(256), None)
    assert st == moe.MOE_ERR_INVALID_ARG and "NULL" in moe.last_error_detail()
    st = moe._lib.moe_dispatch_layout(ctypes.byref(cfg), 0, 63, None, None, None, None, None,
                                      None, None, None, None, ctypes.c_void_p(256), None)
    assert st == moe.MOE_ERR_INVALID_ARG and "divisible" in moe.last_error_detail()


def test_status_strings():
    for s in range(6):
        assert moe.status_string(s)


def test_fp8_entry_points_reject_bad_arguments_before_any_launch():
    ws = ctypes.c_void_p(256)            # aligned, never dereferenced on these paths
    # the row quantisation: bf16 rows must be a whole number of 8-value vectors
    st = moe._lib.moe_quantize_fp8_rows(4, 12, moe.MOE_BF16, None, None, None, None)
    assert st == moe.MOE_ERR_UNSUPPORTED
    st = moe._lib.moe_quantize_fp8_rows(4, 16, moe.MOE_BF16, None, None, None, None)
    assert st == moe.MOE_ERR_INVALID_ARG and "NULL" in moe.last_error_detail()
    st = moe._lib.moe_quantize_fp8_rows(0, 16, moe.MOE_BF16, None, None, None, None)
    assert st == moe.MOE_OK                                  # nothing to do
    st = moe._lib.moe_quantize_fp8_rows(4, 16, 5, None, None, None, None)
    assert st == moe.MOE_ERR_INVALID_ARG
    bf = moe.make_config(64, 128, 8, 2, 128, 2)
    f8 = moe.make_config(64, 128, 8, 2, 128, 2, ffn_fp8=True)
    # the FFN entry points refuse the other form's config
    st = moe._lib.moe_grouped_swiglu_ffn(ctypes.byref(f8), 16, *([None] * 10), ws, None)
    assert st == moe.MOE_ERR_INVALID_ARG and "fp8" in moe.last_error_detail()
    st = moe._lib.moe_grouped_swiglu_ffn_fp8(ctypes.byref(bf), 16, *([None] * 15), ws, None)
    assert st == moe.MOE_ERR_INVALID_ARG and "fp8" in moe.last_error_detail()
    st = moe._lib.moe_grouped_swiglu_ffn_fp8(ctypes.byref(f8), 16, *([None] * 15), ws, None)
    assert st == moe.MOE_ERR_INVALID_ARG and "NULL" in moe.last_error_detail()
    # the fused quantise-and-permute: FP8 configs with H <= 8192 only
    st = moe._lib.moe_permute_quantize_fp8(ctypes.byref(bf), None, None, 0, 64, None, None, None)
    assert st == moe.MOE_ERR_INVALID_ARG
    big = moe.make_config(64, 8320, 8, 2, 128, 2, ffn_fp8=True)
    st = moe._lib.moe_permute_quantize_fp8(ctypes.byref(big), None, None, 0, 64, None, None, None)
    assert st == moe.MOE_ERR_UNSUPPORTED
    # the forward entries need the weights' scales in FP8
    for fn in (moe._lib.moe_forward_chunked, moe._lib.moe_forward_host):
        p = ctypes.c_void_p(512)
        st = fn(ctypes.byref(f8), p, None, p, p, p, None, None, None, None, p, p, p, p, None, ws,
                None, None)
        assert st == moe.MOE_ERR_INVALID_ARG and "scale" in moe.last_error_detail()


def test_forward_workspace_sizes():
    bf = moe.make_config(4096, 2048, 128, 8, 768, 2)
    f8 = moe.make_config(4096, 2048, 128, 8, 768, 2, ffn_fp8=True)
    # FP8 receive rows take one byte per value instead of two; h's codes and scales are added
    assert moe.forward_workspace_bytes(f8) < moe.forward_workspace_bytes(bf)
    # the host-buffer form adds staging for logits, bias, x and out
    extra = moe.forward_host_workspace_bytes(bf) - moe.forward_workspace_bytes(bf)
    assert extra >= 4 * 4096 * 128 + 4 * 128 + 2 * 2 * 4096 * 2048
    assert extra < 4 * 4096 * 128 + 4 * 128 + 2 * 2 * 4096 * 2048 + 4 * 256


def test_backward_entry_points_reject_bad_arguments_before_any_launch():
    ws = ctypes.c_void_p(256)            # aligned, never dereferenced on these paths
    p = ctypes.c_void_p(512)
    bf = moe.make_config(64, 128, 8, 2, 128, 2)
    f8 = moe.make_config(64, 128, 8, 2, 128, 2, ffn_fp8=True)
    dec = moe.make_config(64, 128, 8, 2, 128, 2, reduce_dense=True)
    ffn_bwd = moe._lib.moe_grouped_swiglu_ffn_backward
    st = ffn_bwd(ctypes.byref(bf), 16, *([p] * 11), 2, ws, None)
    assert st == moe.MOE_ERR_INVALID_ARG and "accumulate" in moe.last_error_detail()
    st = ffn_bwd(ctypes.byref(f8), 16, *([p] * 11), 0, ws, None)
    assert st == moe.MOE_ERR_UNSUPPORTED
    st = ffn_bwd(ctypes.byref(bf), 16, None, *([p] * 10), 0, ws, None)
    assert st == moe.MOE_ERR_INVALID_ARG and "NULL" in moe.last_error_detail()
    st = ffn_bwd(ctypes.byref(bf), -1, *([p] * 11), 0, ws, None)
    assert st == moe.MOE_ERR_INVALID_ARG
    bwd = moe._lib.moe_layer_backward
    # save mode needs both saved buffers: one alone is an error
    args = [p] * 9 + [p, None] + [p] * 7
    st = bwd(ctypes.byref(bf), *args, 0, ws, None)
    assert st == moe.MOE_ERR_INVALID_ARG and "saved" in moe.last_error_detail()
    args = [p] * 9 + [None, None] + [p] * 7
    for cfg in (f8, dec):
        st = bwd(ctypes.byref(cfg), *args, 0, ws, None)
        assert st == moe.MOE_ERR_UNSUPPORTED
    st = bwd(ctypes.byref(bf), *([None] * 18), 0, ws, None)
    assert st == moe.MOE_ERR_INVALID_ARG and "NULL" in moe.last_error_detail()
    sv = moe._lib.moe_forward_chunked_save
    st = sv(ctypes.byref(dec), *([p] * 14), ws, None, None)
    assert st == moe.MOE_ERR_UNSUPPORTED
    st = sv(ctypes.byref(bf), *([p] * 12), None, p, ws, None, None)
    assert st == moe.MOE_ERR_INVALID_ARG and "NULL" in moe.last_error_detail()


def test_backward_workspace_holds_every_chunks_rows():
    one = moe.make_config(8192, 7168, 256, 8, 2048, 8, n_chunks=1)
    two = moe.make_config(8192, 7168, 256, 8, 2048, 8, n_chunks=2)
    # the rows the weight gradients read (receive rows, dy, h, dg | du) for all
    # chunks, plus one chunk's slot of the rest: the two-chunk layer needs less
    b1, b2 = moe.backward_workspace_bytes(one), moe.backward_workspace_bytes(two)
    rows_all = 65536 * (7168 + 7168 + 2048 + 2 * 2048) * 2
    assert rows_all < b1 and rows_all < b2 < b1
