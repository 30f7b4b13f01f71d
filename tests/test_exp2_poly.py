"""The FMA-pipe 2^x used by the flash-attention softmax: the committed cubic
and range reduction, evaluated step by step in float32 exactly as the device
does, stay within 1e-4 relative error of 2^x over the range softmax uses."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "llama_decoder_only_rmsnorm_b200", "csrc", "common.cuh")


def coefficients():
    text = open(HDR).read()
    return [np.float32(float(re.search(rf"#define L3_EXP2_C{k} ([-0-9.e]+)f", text).group(1))) for k in range(4)]


def device_exp2(x, c):
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    shift = np.float32(12582912.0)
    t = (x + shift).astype(np.float32)
    n = (t - shift).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = c[3]
    for k in (2, 1, 0):
        p = (p * f + c[k]).astype(np.float32)
    return (p.view(np.int32) + (t.view(np.int32) << 23)).view(np.float32)


def test_poly_exp2_relative_error_bound():
    c = coefficients()
    x = -np.concatenate([np.linspace(0, 1, 100001), np.linspace(1, 125, 400001)]).astype(np.float32)
    got = device_exp2(x, c).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(got - want) / want) < 1e-4
    # exact at integers (f = 0 gives c0 scaled by 2^n, c0 within 1e-4 of 1)
    assert abs(float(device_exp2(np.array([0.0], np.float32), c)[0]) - 1.0) < 1e-4


def test_poly_exp2_clamps_far_negative_inputs_to_tiny_values():
    c = coefficients()
    y = device_exp2(np.array([-200.0, -1e30], np.float32), c)
    assert np.all(y >= 0) and np.all(y < 1e-37)
