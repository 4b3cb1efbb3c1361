"""The NVFP4 quantiser's rounding ties, driven through the kernel.

Random inputs reach an exact tie only by chance, so these rows are built to hit
them (vLLM API page "prepare_trtllm_nvfp4", _quantize_nvfp4_global_scale: the
E2M1 thresholds 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0 with ties to the even
code, the sign bit iff the scaled value is negative, the E4M3 block scale of
gs * amax / 6, saturating at 448).

Construction.  Every row holds BF16 values that are multiples of 2^-5 (or
powers of two down to 2^-6 in the filler) whose squares sum to exactly H, so
the FP32 sum of squares is exact whatever the order, ss / H = 1, and with
eps = 2^-40 the inverse RMS is exactly 1; with norm weights 1 and gain centre
0 the normed value y equals x.  A "tie block" has amax = 6 (fl(6 * fl(1/6)) is
exactly 1), so its scale is e4m3(gs): with gs = 1 the output scale is 1 and the
quantised value q equals y, i.e. lands exactly on each threshold; gs a few
FP32 ulps above or below 1 moves q the same few ulps off the threshold; and
gs set to an E4M3 midpoint (or one ulp either side) puts the scale itself on
a tie.  Copies of the tie block scaled by 2^-1 .. 2^-3 reach the same q through
block scales 1/2 .. 1/8.

Each call's codes and scales must equal the oracle's bit for bit, and the
oracle must report near-threshold cases, which shows the ties were reached.
"""
import numpy as np
import pytest
import torch

import expert_combine_b200 as eb
import oracle
from expert_combine_b200 import synth

pytestmark = pytest.mark.gpu

THRESHOLDS = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)
TIE_A = np.array([6.0, *THRESHOLDS, *(-t for t in THRESHOLDS), -0.0], np.float64)
TIE_B = np.array([-6.0, 0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, 0.125, -0.125])
EPS = 2.0 ** -40


def _bf16_bits(v):
    """Exact BF16 values (float64 in) -> uint16 bit patterns, sign of zero kept."""
    f = np.asarray(v, np.float32)
    u = f.view(np.uint32)
    assert np.all((u & 0xFFFF) == 0), "value not exact in BF16"
    return (u >> 16).astype(np.uint16)


def _row(H, blocks, flip=False):
    """Tie blocks at the front (or back), filler after (before), sum of squares exactly H."""
    ties = np.concatenate(blocks)
    rest = H - ties.size
    need = H - float(np.sum(ties * ties))
    assert need >= 0
    fill = []
    n1 = int(need)
    fill += [1.0] * n1
    r = need - n1
    v = 0.5
    while r > 0:
        assert v >= 2.0 ** -6, "filler cannot reach the sum exactly"
        if r >= v * v:
            fill.append(v)
            r -= v * v
        else:
            v /= 2
    assert len(fill) <= rest, "row too short for its filler"
    fill += [0.0] * (rest - len(fill))
    fill = np.array(fill)
    fill[1::2] *= -1.0                                   # both signs among the filler
    row = np.concatenate([fill, ties]) if flip else np.concatenate([ties, fill])
    assert float(np.sum(row * row)) == H
    return row


def _rows(H):
    scaled = [TIE_A * 2.0 ** -s for s in (1, 2, 3)]
    return np.stack([
        _row(H, [TIE_A, TIE_B, *scaled]),
        _row(H, [-TIE_A, -TIE_B, *[-b for b in scaled]]),
        _row(H, [TIE_B, TIE_A, scaled[0]], flip=True),
        _row(H, [TIE_A[::-1], scaled[2], scaled[1]]),
    ])


def _run(rows, gs, dev):
    M, H = rows.shape
    x = torch.from_numpy(_bf16_bits(rows).view(np.int16)).view(torch.bfloat16).to(dev)
    w = torch.ones(H, dtype=torch.bfloat16, device=dev)
    g = torch.tensor([gs], dtype=torch.float32, device=dev)
    packed, sf = eb.norm_quant_nvfp4(x, M, w, 0.0, EPS, g)
    torch.cuda.synchronize()
    p_o, s_o, near = oracle.norm_quant(synth.host(x), M, H, 1, synth.host(w), 0.0, EPS, float(np.float32(gs)),
                                       return_near=True)
    assert np.array_equal(synth.host(packed), p_o), f"codes differ at gs={gs!r}"
    assert np.array_equal(synth.host(sf), s_o), f"scales differ at gs={gs!r}"
    assert eb.device_status() == 0
    return synth.host(packed), synth.host(sf), near


def _ulps_from(v, n):
    """The binary32 value n units in the last place from v (v > 0)."""
    u = int(np.array([v], np.float32).view(np.uint32)[0]) + n
    return float(np.array([u], np.uint32).view(np.float32)[0])


@pytest.mark.parametrize("H", [512, 2048])          # the pair-row and the wide-row kernels
def test_e2m1_thresholds_and_neighbours(cuda_dev, H, report_near):
    rows = _rows(H)
    total_near = 0
    for n in (-3, -2, -1, 0, 1, 2, 3):
        gs = _ulps_from(1.0, n)
        packed, sf, near = _run(rows, gs, cuda_dev)
        total_near += near[0]
        if n == 0:
            # q == y exactly: the tie block's codes follow the page's table
            # (ties to the even code: 0.25 -> 0, 0.75 -> 2 (1.0), 1.25 -> 2,
            # 1.75 -> 4 (2.0), 2.5 -> 4, 3.5 -> 6 (4.0), 5.0 -> 6; 6 -> 7;
            # negative values carry the sign bit, -0 does not)
            codes = np.stack([packed[0, :8] & 0xF, packed[0, :8] >> 4], axis=1).reshape(-1)
            assert sf[0, 0] == 0x38                                        # scale 1.0
            assert codes.tolist() == [7, 0, 2, 2, 4, 4, 6, 6, 8, 10, 10, 12, 12, 14, 14, 0]
            # the same block scaled by 2^-s, with block scale 2^-s: same codes
            for s, blk in ((1, 2), (2, 3), (3, 4)):
                assert sf[0, blk] == 0x38 - 8 * s
                c = np.stack([packed[0, 8 * blk:8 * blk + 8] & 0xF, packed[0, 8 * blk:8 * blk + 8] >> 4],
                             axis=1).reshape(-1)
                assert np.array_equal(c, codes)
            # grid points and the signed tiny values of the second block
            cb = np.stack([packed[0, 8:16] & 0xF, packed[0, 8:16] >> 4], axis=1).reshape(-1)
            assert cb.tolist() == [15, 0, 1, 2, 3, 4, 5, 6, 9, 10, 11, 12, 13, 14, 0, 8]
    report_near(f"E2M1 ties, H={H}", (total_near, 0), 7 * rows.size, 7 * rows.size // 16)
    assert total_near >= 7 * 4        # every threshold reached in every row at gs = 1 alone


# E4M3 midpoints (normal, subnormal, next to the top) and what round-to-nearest-
# even with saturation makes of them, from the format definition (bias 7, three
# fraction bits, 0x7F is NaN so 448 = 0x7E is the largest finite value).
E4M3_MIDPOINTS = [
    (1.0625, 0x38),            # between 1.0 (0x38) and 1.125 (0x39): even 0x38
    (1.1875, 0x3A),            # between 1.125 and 1.25: even 0x3A
    (1.9375, 0x40),            # between 1.875 (0x3F) and 2.0 (0x40)
    (0.296875, 0x2A),          # between 0.28125 (0x29) and 0.3125 (0x2A)
    (432.0, 0x7E),             # between 416 (0x7D) and 448 (0x7E)
    (464.0, 0x7E),             # above 448: saturates
    (2.0 ** -10, 0x00),        # between 0 and the smallest subnormal 2^-9
    (3 * 2.0 ** -10, 0x02),    # between 2^-9 (0x01) and 2^-8 (0x02)
    (15 * 2.0 ** -10, 0x08),   # between 7*2^-9 (0x07) and 2^-6 (0x08)
]


@pytest.mark.parametrize("H", [512, 2048])
def test_e4m3_scale_ties(cuda_dev, H, report_near):
    rows = _rows(H)
    total_near_sf = 0
    for v, code in E4M3_MIDPOINTS:
        for n in (-1, 0, 1):
            gs = _ulps_from(v, n)
            _, sf, near = _run(rows, gs, cuda_dev)
            total_near_sf += near[1]
            if n == 0:
                assert oracle.e4m3_rn_sat(v) == code
                assert sf[0, 0] == code, f"gs={v}: tie block scale {sf[0, 0]:#x}, want {code:#x}"
    report_near(f"E4M3 ties, H={H}", (0, total_near_sf), 0, 27 * rows.size // 16)
    assert total_near_sf >= 8 * 4     # the eight true midpoints, in every row's tie block


def test_negative_zero_and_zero_scale(cuda_dev):
    """A zero block scale (gs so small that e4m3 gives 0) turns every q into
    +-0: no sign bit, whatever the sign of y (the page's rule: sign iff q < 0)."""
    rows = _rows(512)
    packed, sf, _ = _run(rows, 2.0 ** -12, cuda_dev)
    assert sf[:, 0].tolist() == [0, 0, 0, 0]
    assert np.all(packed[:, :8] == 0)
