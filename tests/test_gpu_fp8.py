"""Parity of the FP8 quantization kernels (through the C ABI) with the oracle.

Codes and scale bytes are integers: they must be bit-exact, except that a
zero code may carry either sign (0x00 and 0x80 stand for the same value).
Both sides decide the rounding on the same exact quotient x * 2^-e, so no
tolerance is needed.  Inputs are seeded normals with rows and groups scaled by
powers of two, plus groups built to hit every corner: exact ties between E4M3
values, maxima exactly at 448 * 2^k and one bf16 step above, all-zero groups,
subnormal groups, and negative values that round to zero.
"""
import numpy as np
import pytest
import torch

import oracle.fp8 as F
import workloads as W
from fine_grained_shared_b200 import moe as B

pytestmark = pytest.mark.gpu


def _same_codes(got: np.ndarray, want: np.ndarray):
    zero = (want & 0x7F) == 0
    bad = np.argwhere((got != want) & ~zero)
    assert bad.size == 0, f"{len(bad)} codes differ, first at {bad[:5].tolist()}"
    assert np.all((got[zero] & 0x7F) == 0)


def _special_rows(rows: int, cols: int, seed: int) -> torch.Tensor:
    """bf16 [rows, cols]: normals scaled by 2^k per row and per group, and corner-case groups."""
    x = W.normal_bf16(seed, 40, 0, (rows, cols), 1.0).float().numpy()
    rng = np.random.default_rng(seed)
    x *= np.exp2(rng.integers(-60, 60, size=(rows, 1))).astype(np.float32)
    groups = -(-cols // 128)
    pos = F.e4m3_decode(np.arange(0x7F))
    ties = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)
    for r in range(rows):
        g = int(rng.integers(0, groups))
        lo, hi = g * 128, min(cols, g * 128 + 128)
        kind = r % 6
        k = float(rng.integers(-40, 40))
        if kind == 0:    # exact ties under a scale of 2^k
            x[r, lo:hi] = rng.choice(ties, hi - lo) * np.float32(2.0 ** k) * rng.choice([-1, 1], hi - lo)
            x[r, lo] = np.float32(448.0 * 2.0 ** k)
        elif kind == 1:  # maximum one bf16 step above 448 * 2^k
            x[r, lo] = np.float32(448.0 * 2.0 ** k * (1 + 2.0 ** -7))
        elif kind == 2:
            x[r, lo:hi] = 0.0
        elif kind == 3:  # subnormal group: the scale exponent takes its clamp
            x[r, lo:hi] = rng.integers(-64, 64, hi - lo).astype(np.float32) * np.float32(2.0 ** -133)
        elif kind == 4:  # tiny negatives next to a large maximum round to -0
            x[r, lo:hi] = np.float32(-(2.0 ** (k - 30)))
            x[r, lo] = np.float32(448.0 * 2.0 ** k)
    return W.to_bf16(x)


def _check_rows(x: torch.Tensor, q: torch.Tensor, sc: torch.Tensor, rows=None):
    xn = x.float().numpy().astype(np.float64)
    qn, sn = q.cpu().numpy(), sc.cpu().numpy().astype(np.int64)
    if rows is not None:
        xn, qn, sn = xn[rows], qn[rows], sn[rows]
    qo, eo = F.quantize_rows(xn)
    assert np.array_equal(sn - 127, eo)
    _same_codes(qn, qo)


@pytest.mark.parametrize("rows,cols", [(1, 16), (3, 144), (7, 272), (37, 2048), (513, 1408), (64, 7168),
                                       (2, 128), (300, 208)])
def test_rows_match_oracle(rows, cols):
    x = _special_rows(rows, cols, seed=rows * 7919 + cols)
    q, sc = B.quantize_fp8_rows(x.cuda())
    torch.cuda.synchronize()
    _check_rows(x, q, sc)


def test_rows_full_size_sampled():
    """The 16B prefill layer's permuted activations, [T * K, d] = [98304, 2048], in the
    launch configuration the benchmark times (grid-stride over more tasks than resident warps)."""
    rows, cols = 16384 * 6, 2048
    x = _special_rows(rows, cols, seed=5)
    q, sc = B.quantize_fp8_rows(x.cuda())
    torch.cuda.synchronize()
    sample = np.sort(np.random.default_rng(1).choice(rows, 160, replace=False))
    sample = np.concatenate([[0, 1, rows - 1], sample])
    _check_rows(x, q, sc, sample)
    # every group's largest element lands in (224, 448] (all-zero and clamped groups aside)
    xs = x.view(rows, cols // 128, 128).float().abs().amax(dim=2)
    e = sc.cpu().to(torch.int64) - 127
    top = xs / torch.exp2(e.double()).float()
    ok = (e == -127) | ((top > 224) & (top <= 448))
    assert bool(ok.all())


def test_rows_of_a_strided_subset_view_rejected_by_alignment():
    x = torch.zeros((4, 136), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(B.MoEError) as ei:
        B.quantize_fp8_rows(x)
    assert ei.value.status == B.MOE_ERR_ALIGNMENT


def _check_blocks(w: torch.Tensor, q: torch.Tensor, sc: torch.Tensor, mats=None):
    wn = w.float().numpy().astype(np.float64)
    qn, sn = q.cpu().numpy(), sc.cpu().numpy().astype(np.int64)
    for m in (range(wn.shape[0]) if mats is None else mats):
        qo, eo = F.quantize_groups(wn[m], 128, 128)
        assert np.array_equal(sn[m] - 127, eo), m
        _same_codes(qn[m], qo)


@pytest.mark.parametrize("batch,rows,cols", [(1, 128, 128), (3, 200, 144), (2, 1408, 2048), (1, 1, 16),
                                             (4, 257, 1104)])
def test_blocks_match_oracle(batch, rows, cols):
    w = W.normal_bf16(batch * 131 + rows, 41, cols, (batch, rows, cols), 0.02).float()
    w[:, :rows // 2] *= 64.0                  # blocks of different scale within a matrix
    w[-1, -1, -1] = 448.0 * 2.0 ** -3        # one block whose maximum sits on a boundary
    w = w.to(torch.bfloat16)
    q, sc = B.quantize_fp8_blocks(w.cuda())
    torch.cuda.synchronize()
    _check_blocks(w, q, sc)


def test_blocks_full_size_sampled():
    """All 64 W_gate matrices of the 16B layer, [64, 1408, 2048]; three compared in full."""
    w = W.normal_bf16(77, 42, 0, (64, 1408, 2048), 0.02)
    q, sc = B.quantize_fp8_blocks(w.cuda())
    torch.cuda.synchronize()
    _check_blocks(w, q, sc, mats=[0, 31, 63])


def test_block_quantize_of_one_matrix_equals_its_slice_of_a_stack():
    w = W.normal_bf16(3, 43, 0, (3, 256, 384), 0.1).cuda()
    q, sc = B.quantize_fp8_blocks(w)
    q1, sc1 = B.quantize_fp8_blocks(w[1].contiguous())
    assert torch.equal(q[1], q1) and torch.equal(sc[1], sc1)
