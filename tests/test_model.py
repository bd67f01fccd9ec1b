"""The work model and the fast-I2F identity against the numbers the MixLLM page prints."""
import json
import os

import numpy as np

from mixed_precision_quantized_mx_b200 import model

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "paper_numbers.json")))


def test_intensity_gains_printed_on_page():
    g = GOLD["intensity"]
    M, N, K = g["M"], g["N"], g["K"]
    base = model.intensity(M, N, K, 1.0, 1.0)
    w4 = model.intensity(M, N, K, 1.0, 0.5)
    a4 = model.intensity(M, N, K, 0.5, 1.0)
    assert round(w4 / base - 1, 2) == g["weight_8_to_4_gain"]
    assert round(a4 / base - 1, 4) == g["act_8_to_4_gain"]


def test_fast_i2f_identity_over_window():
    g = GOLD["fast_i2f"]
    bias = int(g["bias_bits"], 16)
    assert np.array([bias], np.uint32).view(np.float32)[0] == np.float32(g["bias_float"])
    half = g["window_values"] // 2
    v = np.concatenate([np.arange(-half, -half + 4096), np.arange(-4096, 4096),
                        np.arange(half - 4096, half)]).astype(np.int64)
    f = (v + bias).astype(np.uint32).view(np.float32) - np.float32(g["bias_float"])
    assert np.array_equal(f.astype(np.int64), v)
    # the group bound: |k-long int8 dot| <= 127^2 k < 2^22 for k <= 128
    assert 127 * 127 * g["max_group"] < half


def test_byte_model_small_case():
    # N=256, K=256, g=128, 32 8-bit rows, M=2 counted by hand
    w = 32 * 256 + 224 * 128 + 2 * 256 * 2 + 224 * 2 / 2 + 4 * 256
    assert model.weight_bytes(256, 256, 128, 32) == w
    assert model.gemm_bytes(2, 256, 256, 128, 32) == w + 2 * 256 + 4 + 2 * 2 * 256
    assert model.gemm_ops(2, 3, 4) == 48
