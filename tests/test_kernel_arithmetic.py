"""Host-side checks of the arithmetic the CUDA kernels hard-code.

The softmax kernels evaluate part of their exponentials as exp2_fma()
(wall_common.cuh): range reduction x = n + f with |f| <= 1/2 through the
1.5 * 2^23 rounding constant, a degree-3 polynomial for 2^f, and n added to
the exponent field.  These tests read the coefficients from the header and
replay the same fp32 steps in numpy, so a mistyped coefficient, a wrong
rounding constant or a wrong exponent shift fails here, without a GPU.
The integer-anchor factors 2^k are built directly as bf16 bit patterns; the
bit recipe is checked against exact powers of two.
"""
import pathlib
import re

import numpy as np

HEADER = pathlib.Path(__file__).resolve().parents[1] / "channel_decay_softmax_b200" / "csrc" / "wall_common.cuh"
BWD = pathlib.Path(__file__).resolve().parents[1] / "channel_decay_softmax_b200" / "csrc" / "wall_attn_bwd_sm100.cu"


def _exp2_fma_coefficients():
    src = HEADER.read_text()
    body = src[src.index("float exp2_fma(float x)"):]
    body = body[: body.index("\n}\n")]
    nums = [float(v) for v in re.findall(r"(-?\d+\.\d*)f", body)]
    # clamp, rounding constant (twice), then c3, c2, c1, c0 in Horner order
    assert nums[0] == -126.0 and nums[1] == nums[2] == 12582912.0, nums
    c3, c2, c1, c0 = nums[3:7]
    return np.float32(c0), np.float32(c1), np.float32(c2), np.float32(c3)


def _exp2_fma(x):
    c0, c1, c2, c3 = _exp2_fma_coefficients()
    x = np.maximum(np.float32(x), np.float32(-126.0)).astype(np.float32)
    y = (x + np.float32(12582912.0)).astype(np.float32)
    f = (x - (y - np.float32(12582912.0))).astype(np.float32)
    p = (((c3 * f + c2) * f + c1) * f + c0).astype(np.float32)
    bits = p.view(np.int32).astype(np.int64) + (y.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_exp2_fma_relative_error_bound():
    # the softmax range: logits minus the row's log-sum-exp, so x <= ~0
    x = np.concatenate([np.linspace(-125.0, 0.5, 400001), -np.arange(0, 126, dtype=np.float64),
                        np.array([-0.5, 0.5, -1.5, -2.5])]).astype(np.float32)
    got = _exp2_fma(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 1e-4, rel.max()  # fit: 7.6e-5; bf16 P needs 2^-9


def test_exp2_fma_integers_and_clamp():
    # integer arguments: f = 0, result c0 * 2^n, normal down to 2^-125
    x = -np.arange(0, 126, dtype=np.float32)
    got = _exp2_fma(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.all(np.abs(got - ref) / ref < 1e-4)
    # at and below the clamp the result is at most 2^-125 (a subnormal
    # encoding at -126), negligible next to any row's leading term
    tiny = _exp2_fma(np.array([-126.0, -126.4, -200.0, -1e6], dtype=np.float32))
    assert np.all((tiny >= 0) & (tiny <= 2.0 ** -125))


def test_pow2_bf16_bit_recipe():
    # pow2_bf16(k) = (k + 127) << 7 for k in [-126, 127]: the bf16 bits of 2^k
    src = BWD.read_text()
    assert "e < -126 ? 0u : e > 127 ? 0x7F80u : uint32_t(e + 127) << 7" in src
    for k in range(-126, 128):
        bits = (k + 127) << 7
        val = np.array([bits << 16], dtype=np.uint32).view(np.float32)[0]
        assert val == np.float32(2.0 ** k), k
    assert np.array([0x7F80 << 16], dtype=np.uint32).view(np.float32)[0] == np.inf
