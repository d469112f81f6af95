"""Pins of the FP8 quantization oracle (``oracle/fp8.py``) to things other than itself.

- The E4M3 code table and its round-to-nearest-even conversion against torch's
  own float8_e4m3fn type (a library routine).
- The power-of-two scale rule by brute force over exponents.
- Exactness on inputs that are representable, and the half-step error bound
  on those that are not.
- The group geometry (1 x 128 rows, 128 x 128 blocks) by perturbing one element.
- The FP8 layer on weights chosen so that each quantization in it is either
  lossless or pinned above: permutation and identity matrices, unit vectors.
"""
import numpy as np
import pytest
import torch

import oracle.fp8 as F
import oracle.moe_oracle as M


def _torch_codes(v32: np.ndarray) -> np.ndarray:
    return torch.from_numpy(v32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_code_table_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = F.e4m3_decode(codes)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(lib))
    ok = ~np.isnan(lib)
    assert np.array_equal(ours[ok], lib[ok])
    assert np.isnan(ours).sum() == 2 and F.e4m3_decode(0x7E) == 448.0


def test_rounding_matches_torch_conversion():
    pos = F.e4m3_decode(np.arange(0x7F))
    mids = (pos[:-1] + pos[1:]) / 2                     # every tie
    quarter = pos[:-1] + (pos[1:] - pos[:-1]) / 4       # off-tie points
    rng = np.random.default_rng(5)
    rand = np.exp2(rng.uniform(-13, np.log2(448), 200_000))
    v = np.concatenate([pos, mids, quarter, rand, [0.0]]).astype(np.float32)
    v = np.concatenate([v, -v])
    assert np.all(np.abs(v) <= 448)
    assert np.array_equal(F.e4m3_encode(v), _torch_codes(v))


def _bf16(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).float().numpy()


def test_scale_exponent_is_the_smallest_fitting_power_of_two():
    rng = np.random.default_rng(6)
    amax = np.concatenate([
        _bf16(np.exp2(rng.uniform(-130, 127, 3000))),
        448.0 * np.exp2(np.arange(-60, 60)),                                  # exact boundaries
        _bf16(448.0 * np.exp2(np.arange(-60, 60)) * (1 + 2.0 ** -7)),        # next bf16 above
        _bf16(224.0 * np.exp2(np.arange(-60, 60)) * (1 + 2.0 ** -7)),
        [0.0, 2.0 ** -133, 2.0 ** -120],
    ])
    got = F.scale_exponent(amax)
    for a, e in zip(amax, got):
        brute = next(k for k in range(-127, 128) if a <= 448.0 * 2.0 ** k)
        assert e == brute, (a, e, brute)
    assert F.scale_exponent(448.0) == 0 and F.scale_exponent(449.0) == 1
    assert F.scale_exponent(224.0) == -1 and F.scale_exponent(0.0) == -127


def test_representable_group_round_trips_exactly():
    rng = np.random.default_rng(7)
    for k in (-20, -3, 0, 5):
        codes = rng.integers(0, 0x7F, size=(3, 256)).astype(np.uint8)
        codes[:, 0] = 0x7E                          # 448 in every group ...
        codes[:, 128] = 0x7E
        codes |= (rng.integers(0, 2, size=codes.shape) * 0x80).astype(np.uint8)
        x = F.e4m3_decode(codes) * 2.0 ** k         # ... so each group's scale is 2^k
        q, e = F.quantize_rows(x)
        assert np.all(e == k)
        assert np.array_equal(F.e4m3_decode(q), F.e4m3_decode(codes))
        assert np.array_equal(F.dequantize_groups(q, e, 1, F.GROUP), x)


def test_error_is_within_half_a_step():
    rng = np.random.default_rng(8)
    x = rng.standard_normal((16, 512))
    x[3] *= 1e-3
    x[5, :128] *= 1e4
    x[9, 256:] = 0.0
    x = _bf16(x).astype(np.float64)
    q, e = F.quantize_rows(x)
    s = np.repeat(np.exp2(e.astype(np.float64)), F.GROUP, axis=1)
    err = np.abs(F.dequantize_groups(q, e, 1, F.GROUP) - x)
    normal = np.abs(x) / s >= 2.0 ** -6
    assert np.all(err[normal] <= 2.0 ** -4 * np.abs(x[normal]))
    assert np.all(err[~normal] <= 2.0 ** -10 * s[~normal])
    top = (np.abs(x) / s).reshape(16, 4, F.GROUP).max(axis=2)
    nonzero = top > 0
    assert np.all((top[nonzero] > 224) & (top[nonzero] <= 448))
    assert np.all(e[9, 2:] == -127)


def test_row_groups_run_along_the_columns():
    rng = np.random.default_rng(9)
    x = _bf16(rng.standard_normal((4, 384))).astype(np.float64)
    q0, e0 = F.quantize_rows(x)
    assert e0.shape == (4, 3)
    x2 = x.copy()
    x2[2, 130] = 1000.0
    q1, e1 = F.quantize_rows(x2)
    changed = np.argwhere(e0 != e1)
    assert changed.tolist() == [[2, 1]]
    diff = np.argwhere(q0 != q1)
    assert set(map(tuple, diff)) <= {(2, c) for c in range(128, 256)}
    assert np.array_equal(F.qdq_rows(x2), F.dequantize_groups(q1, e1, 1, 128))


def test_weight_blocks_are_128_by_128():
    rng = np.random.default_rng(10)
    w = _bf16(rng.standard_normal((256, 384)) * 0.02).astype(np.float64)
    q0, e0 = F.quantize_blocks(w)
    assert e0.shape == (2, 3)
    w2 = w.copy()
    w2[200, 300] = 3.0
    q1, e1 = F.quantize_blocks(w2)
    assert np.argwhere(e0 != e1).tolist() == [[1, 2]]
    diff = np.argwhere(q0 != q1)
    assert all(128 <= r < 256 and 256 <= c < 384 for r, c in diff) and len(diff) > 100
    # a stack quantizes each matrix on its own
    qs, es = F.quantize_blocks(np.stack([w, w2]))
    assert np.array_equal(qs[0], q0) and np.array_equal(es[1], e1)
    assert np.array_equal(F.qdq_blocks(w2), F.dequantize_groups(q1, e1, 128, 128))


def test_backward_groups_are_128_tokens_of_one_channel():
    rng = np.random.default_rng(15)
    x = _bf16(rng.standard_normal((300, 40)) * np.exp2(rng.integers(-5, 5, size=(1, 40)))).astype(np.float64)
    q, e = F.quantize_cols(x)
    assert e.shape == (3, 40)                       # 128 + 128 + 44 rows
    qt, et = F.quantize_rows(x.T)                   # the same groups, seen transposed
    assert np.array_equal(q, qt.T) and np.array_equal(e, et.T)
    x2 = x.copy()
    x2[200, 7] = 1e4
    q2, e2 = F.quantize_cols(x2)
    assert np.argwhere(e != e2).tolist() == [[1, 7]]
    assert all(c == 7 and 128 <= r < 256 for r, c in np.argwhere(q != q2))


def test_ragged_last_group_has_its_own_scale():
    x = np.zeros((1, 144))
    x[0, :128] = 448.0
    x[0, 128:] = 0.75
    q, e = F.quantize_rows(x)
    assert e.tolist() == [[0, -9]]                  # 0.75 <= 448 * 2^-9 = 0.875
    assert np.all(F.e4m3_decode(q[0, 128:]) * 2.0 ** -9 == 0.75)


def _perm(n, seed):
    p = np.random.default_rng(seed).permutation(n)
    m = np.zeros((n, n))
    m[np.arange(n), p] = 1.0
    return m


def test_fp8_ffn_quantizes_the_input_rows_and_h():
    """W_gate = W_up = P, W_down = P^T (lossless) -> FFN = qdq(SiLU(u~) * u~), u~ = qdq(u)."""
    rng = np.random.default_rng(11)
    u = _bf16(rng.standard_normal((6, 128)) * np.array([[1], [1e-2], [10], [1], [3], [0.1]])).astype(np.float64)
    P = _perm(128, 1)
    got = F.swiglu_ffn_fp8(u, P, P, P.T)
    ut = F.qdq_rows(u)
    want = F.qdq_rows(M.silu(ut) * ut)
    assert np.array_equal(got, want)
    assert not np.array_equal(got, M.swiglu_ffn(u, P, P, P.T))


def test_fp8_ffn_quantizes_h_in_row_groups_of_128():
    """Representable u and gate/up weights, W_down = I: the output is qdq_rows of the plain H."""
    rng = np.random.default_rng(12)
    d, I = 128, 256
    u = F.e4m3_decode(rng.integers(0, 0x7F, size=(5, d))) * 2.0 ** -8
    u[:, 0] = 448.0 * 2.0 ** -8
    wg = F.e4m3_decode(rng.integers(0, 0x50, size=(I, d))) * 2.0 ** -12
    wu = F.e4m3_decode(rng.integers(0, 0x50, size=(I, d)) | 0x80) * 2.0 ** -12
    wg[:128, 0] = wg[128:, 1] = wu[:128, 2] = wu[128:, 3] = 448.0 * 2.0 ** -12
    assert np.array_equal(F.qdq_rows(u), u)
    assert np.array_equal(F.qdq_blocks(wg), wg) and np.array_equal(F.qdq_blocks(wu), wu)
    got = F.swiglu_ffn_fp8(u, wg, wu, np.eye(I))      # W_down = I: the output is H itself
    h = M.silu(u @ wg.T) * (u @ wu.T)
    assert np.array_equal(got, F.qdq_rows(h))
    assert not np.array_equal(got, h)


def test_fp8_ffn_quantizes_weights_in_blocks():
    """u = unit vectors (lossless): the gate/up inputs are columns of the block-quantized weights."""
    rng = np.random.default_rng(13)
    d = I = 256
    wg = _bf16(rng.standard_normal((I, d)) * np.exp2(rng.integers(-4, 4, size=(I, 1)))).astype(np.float64)
    wu = _bf16(rng.standard_normal((I, d)) * 0.1).astype(np.float64)
    j = np.array([3, 130, 255])
    u = np.zeros((3, d))
    u[np.arange(3), j] = 1.0
    got = F.swiglu_ffn_fp8(u, wg, wu, np.eye(d))
    gq, uq = F.qdq_blocks(wg), F.qdq_blocks(wu)
    want = F.qdq_rows(M.silu(gq[:, j].T) * uq[:, j].T)
    assert np.array_equal(got, want)
    # row-wise weight groups would give another result here (rows differ in scale by up to 2^7)
    gr = F.dequantize_groups(*F.quantize_groups(wg, 1, 128), 1, 128)
    assert not np.array_equal(want, F.qdq_rows(M.silu(gr[:, j].T) * uq[:, j].T))


def _tiny_layer(seed, d=256, I=128, N=8, Ks=1):
    rng = np.random.default_rng(seed)
    b = lambda *s, sd=0.05: _bf16(rng.standard_normal(s) * sd).astype(np.float64)
    x = b(24, d, sd=1.0)
    return x, b(N, d), (b(N, I, d), b(N, I, d), b(N, d, I)), (b(Ks, I, d), b(Ks, I, d), b(Ks, d, I))


def test_fp8_layer_routes_in_high_precision_and_keeps_the_residual():
    x, e, ex, sh = _tiny_layer(14)
    h8, r8 = F.moe_forward_fp8(x, e, 3, ex, sh)
    h, r = M.moe_forward(x, e, 3, ex, sh)
    assert np.array_equal(r8.idx, r.idx) and np.array_equal(r8.gate, r.gate)
    only_u, _ = F.moe_forward_fp8(x, e, 3, ex, sh, flags=M.FLAG_NO_SHARED | M.FLAG_NO_ROUTED)
    assert np.array_equal(only_u, x)
    # the FFN terms carry the FP8 error: a few per cent of their size, not zero
    rel = np.sqrt(np.mean((h8 - h) ** 2)) / np.sqrt(np.mean((h - x) ** 2))
    assert 2e-3 < rel < 8e-2, rel
