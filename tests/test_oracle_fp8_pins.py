"""Pins of the oracle's FP8 expert FFN (E4M3 codes with UE8M0 row scales) to
things other than itself: PyTorch's float8_e4m3fn conversions (a library
implementation of the same format), closed forms of the scale rule, the
format's error bound, and the already-pinned bf16 FFN of the oracle on the
dequantised operands.

Sources: LightLLM PR 1687 review page (FP8 grouped GEMM with UE8M0 scales,
silu_and_mul followed by quantisation); the E4M3 format (1 sign, 4 exponent
bits with bias 7, 3 fraction bits, no infinities, largest finite 448).
"""
import numpy as np
import pytest
import torch

import oracle



def _torch_e4m3(values: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(values, np.float32)).to(torch.float8_e4m3fn) \
        .view(torch.uint8).numpy()


def _torch_decode(codes: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn) \
        .to(torch.float64).numpy()


def _finite_values():
    d = _torch_decode(np.arange(256, dtype=np.uint8))
    return np.unique(d[~np.isnan(d)])


def test_e4m3_decode_matches_library_for_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ours, ref = oracle.e4m3_decode(codes), _torch_decode(codes)
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(ours[ok], ref[ok])
    assert np.isnan(ours[0x7F]) and np.isnan(ours[0xFF])
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9 and ours[0x08] == 2.0 ** -6


def test_e4m3_encode_rounds_to_nearest_even_like_library():
    fin = _finite_values()
    mids = (fin[1:] + fin[:-1]) / 2                      # every tie between neighbours
    rng = np.random.default_rng(0)
    vals = np.concatenate([fin, mids, rng.uniform(-448, 448, 20000), rng.normal(0, 1e-2, 20000),
                           rng.normal(0, 1e-3, 5000)]).astype(np.float32)
    np.testing.assert_array_equal(oracle.e4m3_encode(vals.astype(np.float64)), _torch_e4m3(vals))
    # ties go to the even fraction: 1 + 1/16 lies between 1 (fraction 0) and 1.125 (fraction 1)
    assert oracle.e4m3_encode(1.0625) == 0x38
    assert oracle.e4m3_encode(1.1875) == 0x3A             # between 1.125 and 1.25: to 1.25


def test_e4m3_encode_saturates_and_round_trips():
    assert oracle.e4m3_encode(448.0) == 0x7E
    assert oracle.e4m3_encode(470.0) == 0x7E
    assert oracle.e4m3_encode(1e30) == 0x7E
    assert oracle.e4m3_encode(-np.inf) == 0xFE
    assert oracle.e4m3_encode(np.nan) == 0x7F
    assert oracle.e4m3_encode(-0.0) == 0x80
    assert oracle.e4m3_encode(2.0 ** -11) == 0x00        # below half the smallest subnormal
    codes = np.arange(256, dtype=np.uint8)
    vals = oracle.e4m3_decode(codes)
    ok = ~np.isnan(vals)
    np.testing.assert_array_equal(oracle.e4m3_encode(vals[ok]), codes[ok])


def test_ue8m0_scale_closed_forms():
    assert oracle.ue8m0_scale(448.0) == 127                  # 448 fits with scale 1
    assert oracle.ue8m0_scale(448.0 * (1 + 2.0 ** -40)) == 128
    assert oracle.ue8m0_scale(224.0) == 126                  # 224 <= 448 / 2
    assert oracle.ue8m0_scale(224.0 * (1 + 2.0 ** -40)) == 127
    assert oracle.ue8m0_scale(448.0 * 2.0 ** -8) == 119      # a scale of 2^-8
    assert oracle.ue8m0_scale(1.0) == 127 - 8                # 1 <= 448 / 2^8 = 1.75
    assert oracle.ue8m0_scale(0.0) == 127                    # a zero row keeps scale 1
    assert oracle.ue8m0_scale(1e-300) == 1                   # clamped at 2^-126
    assert oracle.ue8m0_scale(1e300) == 254                  # clamped at 2^127
    for e in range(-100, 100, 7):                            # a power of two times 448 is exact
        assert oracle.ue8m0_scale(448.0 * 2.0 ** e) == 127 + e


@pytest.mark.parametrize("scale", [1e-3, 1.0, 37.0])
def test_quantize_rows_error_bound_minimal_scale_and_library_codes(scale):
    rng = np.random.default_rng(1)
    a32 = (rng.normal(0, 1, (64, 200)) * scale).astype(np.float32)
    a32[3] = 0.0                                              # a zero row
    a32[5, :] = 0.0
    a32[5, 17] = -3.0                                         # a single nonzero
    bits = (a32.view(np.uint32) >> 16).astype(np.uint16)      # bf16 by truncation: exact inputs
    a = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    codes, scales = oracle.quantize_rows(bits)
    e = scales.astype(np.int32) - 127
    dq = oracle.dequantize_rows(codes, scales)
    for r in range(a.shape[0]):
        amax = np.abs(a[r]).max()
        if amax == 0:
            assert scales[r] == 127 and (codes[r] & 0x7F == 0).all()
            continue
        # minimal scale: the largest magnitude, scaled, lands in (224, 448]
        assert 224 < amax * 2.0 ** -e[r] <= 448, (r, amax, e[r])
        top = np.abs(oracle.e4m3_decode(codes[r])).max()
        assert 224 <= top <= 448, (r, top)
        # the codes are the library's conversion of the exactly scaled values
        np.testing.assert_array_equal(codes[r], _torch_e4m3(np.ldexp(a[r], -e[r]).astype(np.float32)))
        # half a quantum: 2^-4 relative in the normal range, 2^-10 * 2^e below it
        bound = np.maximum(np.abs(a[r]) * 2.0 ** -4, 2.0 ** (e[r] - 10))
        assert (np.abs(dq[r] - a[r]) <= bound).all()


def _random_fp8_operands(rng, H, I):
    """Codes of moderate magnitude and scale bytes near the weights' natural range."""
    def codes(shape):
        v = rng.normal(0, 64, shape)
        return oracle.e4m3_encode(v)
    x = codes(H)
    w13 = codes((2 * I, H))
    w2 = codes((H, I))
    sx = 127 - 6
    w13_s = (127 - 12 + rng.integers(-1, 2, 2 * I)).astype(np.uint8)
    w2_s = (127 - 11 + rng.integers(-1, 2, H)).astype(np.uint8)
    return x, sx, w13, w13_s, w2, w2_s


def _bf16_bits(v: np.ndarray) -> np.ndarray:
    b = np.asarray(v, np.float32).view(np.uint32)
    assert (b & 0xFFFF == 0).all(), "value not exactly representable in bf16"
    return (b >> 16).astype(np.uint16)


def test_ffn_row_fp8_h_equals_bf16_oracle_on_dequantised_operands():
    rng = np.random.default_rng(2)
    H, I = 96, 40
    x, sx, w13, w13_s, w2, w2_s = _random_fp8_operands(rng, H, I)
    h, hq, sh, y, ye = oracle.ffn_row_fp8(x, sx, w13, w13_s, w2, w2_s)
    # E4M3 values times powers of two are exact bf16 values
    xb = _bf16_bits(_torch_decode(x) * 2.0 ** (sx - 127))
    w13b = _bf16_bits(_torch_decode(w13) * np.ldexp(1.0, w13_s.astype(np.int32) - 127)[:, None])
    w2b = _bf16_bits(_torch_decode(w2) * np.ldexp(1.0, w2_s.astype(np.int32) - 127)[:, None])
    h_ref, _, _ = oracle.ffn_row(xb, w13b, w2b)
    np.testing.assert_array_equal(h, h_ref)
    assert (h != 0).sum() > I // 2


def test_ffn_row_fp8_second_gemm_by_library_matmul():
    rng = np.random.default_rng(3)
    H, I = 64, 48
    x, sx, w13, w13_s, w2, w2_s = _random_fp8_operands(rng, H, I)
    h, hq, sh, y, ye = oracle.ffn_row_fp8(x, sx, w13, w13_s, w2, w2_s)
    # h is quantised as one row
    hq_ref, sh_ref = oracle.quantize_rows(h[None])
    np.testing.assert_array_equal(hq, hq_ref[0])
    assert sh == sh_ref[0]
    w2_dq = _torch_decode(w2) * np.ldexp(1.0, w2_s.astype(np.int32) - 127)[:, None]
    h_dq = _torch_decode(hq) * 2.0 ** (sh - 127)
    ref = w2_dq @ h_dq
    np.testing.assert_allclose(ye, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    np.testing.assert_array_equal(y, [oracle.bf16_bits_from_double(v) for v in ye])


def test_ffn_row_fp8_weight_row_scale_is_a_power_of_two_per_row():
    rng = np.random.default_rng(4)
    H, I = 32, 32
    x, sx, w13, w13_s, w2, w2_s = _random_fp8_operands(rng, H, I)
    _, _, _, _, ye = oracle.ffn_row_fp8(x, sx, w13, w13_s, w2, w2_s)
    w2_s2 = w2_s.copy()
    w2_s2[5] += 3                                             # output channel 5 times 8
    _, _, _, _, ye2 = oracle.ffn_row_fp8(x, sx, w13, w13_s, w2, w2_s2)
    assert ye2[5] == 8 * ye[5]
    np.testing.assert_array_equal(np.delete(ye2, 5), np.delete(ye, 5))


def test_quantize_blocks_reduces_to_rows_and_is_exact_per_block():
    rng = np.random.default_rng(9)
    a = (rng.normal(0, 1, (16, 384)) * np.ldexp(1.0, rng.integers(-20, 20, (16, 1)))).astype(np.float32)
    a[:, 128:256] *= 1e-3                       # a quiet middle block takes its own scale
    # one block spanning the row is the row quantisation
    c_row, s_row = oracle.quantize_rows(a)
    c1, s1 = oracle.quantize_blocks(a, 384)
    np.testing.assert_array_equal(c1, c_row)
    np.testing.assert_array_equal(s1[:, 0], s_row)
    # each 128-column block is the row quantisation of that block alone
    c, s = oracle.quantize_blocks(a, 128)
    for b in range(3):
        cb, sb = oracle.quantize_rows(np.ascontiguousarray(a[:, 128 * b:128 * (b + 1)]))
        np.testing.assert_array_equal(c[:, 128 * b:128 * (b + 1)], cb)
        np.testing.assert_array_equal(s[:, b], sb)
    assert (s[:, 1] < s[:, 0]).all()            # the quiet block's scale is smaller
    # a ragged last block
    c, s = oracle.quantize_blocks(a[:, :300].copy(), 128)
    assert s.shape == (16, 3)
    cb, sb = oracle.quantize_rows(np.ascontiguousarray(a[:, 256:300]))
    np.testing.assert_array_equal(c[:, 256:300], cb)
    np.testing.assert_array_equal(s[:, 2], sb)


def test_dot_blocked_equals_library_dequantised_dot():
    rng = np.random.default_rng(10)
    K = 512
    a = rng.normal(0, 1, (4, K)).astype(np.float32)
    b = (rng.normal(0, 1, (4, K)) * 50).astype(np.float32)
    ca, sa = oracle.quantize_blocks(a, 128)
    cb, sb = oracle.quantize_blocks(b, 128)
    for r in range(4):
        deq = lambda c, s: _torch_decode(c) * np.repeat(np.ldexp(1.0, s.astype(np.int32) - 127), 128)
        ref = float(np.dot(deq(ca[r], sa[r]), deq(cb[r], sb[r])))
        got = oracle.dot_blocked(ca[r], sa[r], cb[r], sb[r], 128)
        assert abs(got - ref) <= 1e-12 * max(1.0, abs(ref))


# ----------------------------------------------------------------- K-blocked FP8 expert row

def _blocked_operands(rng, H, I, block, uniform_rows=False):
    """x [H], W13 [2I, H], W2 [H, I] as bf16-representable floats quantised by
    rows and `block`-column blocks.  uniform_rows: every block of a row holds the
    row's largest magnitude (its first element), so each block's scale is the row's."""
    def mat(rows, cols, scale):
        a = (rng.normal(0, 1, (rows, cols)) * scale).astype(np.float32)
        a *= np.ldexp(1.0, rng.integers(-3, 4, (rows, 1)))
        if uniform_rows:
            m = np.abs(a).max(axis=1, keepdims=True) * 1.5
            a[:, ::block] = m * np.sign(a[:, ::block] + 0.5)
        return a
    x = mat(1, H, 1.0)
    w13 = mat(2 * I, H, 1.0 / np.sqrt(H))
    w2 = mat(H, I, 1.0 / np.sqrt(H))
    q = lambda a: oracle.quantize_blocks(a, block)
    return q(x), q(w13), q(w2), (x, w13, w2)


def test_ffn_row_fp8_blocked_equals_row_form_when_every_block_holds_the_row_max():
    """When each block's largest magnitude is its row's, every block scale equals
    the row scale and the codes are those of the row quantisation: g, u and so h
    must be the row form's bit for bit (block partial sums and the whole sum are
    both exact in double for E4M3 products)."""
    rng = np.random.default_rng(21)
    H, I, block = 128, 64, 32
    (xq, xs), (wq, ws), (w2q, w2s), raw = _blocked_operands(rng, H, I, block, uniform_rows=True)
    for a, (c, s) in zip(raw, ((xq, xs), (wq, ws), (w2q, w2s))):
        cr, sr = oracle.quantize_rows(a)
        np.testing.assert_array_equal(c, cr)
        assert (s == sr[:, None]).all()
    h_b, _, _, _, _ = oracle.ffn_row_fp8_blocked(xq[0], xs[0], wq, ws, w2q, w2s, block)
    h_r, _, _, _, _ = oracle.ffn_row_fp8(xq[0], xs[0, 0], wq, ws[:, 0], w2q, w2s[:, 0])
    np.testing.assert_array_equal(h_b, h_r)
    assert (h_b != 0).sum() > I // 2


@pytest.mark.parametrize("block", [32, 128])
def test_ffn_row_fp8_blocked_against_library_dequantised_matmuls(block):
    """Every step of the blocked row against library-decoded operands (torch's
    float8_e4m3fn, each block times its power of two) and numpy matmuls in fp64:
    g and u, h rounded to bf16 once, h's block quantisation, and y."""
    rng = np.random.default_rng(22 + block)
    H, I = 256, 128
    (xq, xs), (wq, ws), (w2q, w2s), _ = _blocked_operands(rng, H, I, block)
    h, hq, hs, y, ye = oracle.ffn_row_fp8_blocked(xq[0], xs[0], wq, ws, w2q, w2s, block)
    deq = lambda c, s: _torch_decode(c) * np.repeat(np.ldexp(1.0, s.astype(np.int32) - 127), block, axis=-1)
    x = deq(xq[0], xs[0])
    g = deq(wq[:I], ws[:I]) @ x
    u = deq(wq[I:], ws[I:]) @ x
    hv = g / (1.0 + np.exp(-g)) * u
    h_ref = np.array([oracle.bf16_bits_from_double(v) for v in hv], np.uint16)
    # the fp64 sums run in another order: h may differ where a value sits on a bf16 boundary
    assert (h == h_ref).mean() >= 0.99
    hq_ref, hs_ref = oracle.quantize_blocks(h[None], block)
    np.testing.assert_array_equal(hq, hq_ref[0])
    np.testing.assert_array_equal(hs, hs_ref[0])
    ref = deq(w2q, w2s) @ deq(hq, hs)
    np.testing.assert_allclose(ye, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    np.testing.assert_array_equal(y, [oracle.bf16_bits_from_double(v) for v in ye])
    assert len(set(hs.tolist())) > 1 or I == block     # blocks take their own scales


def test_ffn_row_fp8_blocked_block_scale_multiplies_its_block_only():
    """Raising one W2 block scale by 3 multiplies that block's contribution to its
    output by 8 and changes nothing else."""
    rng = np.random.default_rng(25)
    H, I, block = 64, 64, 32
    (xq, xs), (wq, ws), (w2q, w2s), _ = _blocked_operands(rng, H, I, block)
    h, hq, hs, _, ye = oracle.ffn_row_fp8_blocked(xq[0], xs[0], wq, ws, w2q, w2s, block)
    w2s2 = w2s.copy()
    w2s2[7, 1] += 3
    _, _, _, _, ye2 = oracle.ffn_row_fp8_blocked(xq[0], xs[0], wq, ws, w2q, w2s2, block)
    part = lambda s: oracle.dot_blocked(w2q[7, 32:], s[7, 1:], hq[32:], hs[1:], block)
    assert abs((ye2[7] - ye[7]) - 7 * part(w2s)) <= 1e-12 * max(1.0, abs(ye[7]))
    np.testing.assert_array_equal(np.delete(ye2, 7), np.delete(ye, 7))
