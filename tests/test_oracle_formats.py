"""Pins of the oracle's number-format conversions against numpy / torch."""
import numpy as np
import torch

import oracle
import workloads


def test_f16_rounding_matches_numpy():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.uniform(-9, 5, 20000),
        # exact ties between neighbouring fp16 values (normal and subnormal)
        (np.arange(1, 2048, dtype=np.float64) + 0.5) * 2.0 ** -24,
        (1024 + np.arange(0, 1024) + 0.5) * 2.0 ** -10,
        [65504.0, 65519.99, 65520.0, 1e9, 0.0, -0.0, 2.0 ** -25, 2.0 ** -25 * 1.0000001, 5.9604644775390625e-08],
    ])
    x = np.concatenate([x, -x])
    with np.errstate(over="ignore"):
        want = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(oracle.f64_to_f16(x), want)
    allh = np.arange(65536, dtype=np.uint16)
    fin = (allh & 0x7C00) != 0x7C00
    assert np.array_equal(oracle.f16_to_f64(allh[fin]), allh[fin].view(np.float16).astype(np.float64))


def test_bf16_rounding_matches_torch_on_f32_inputs():
    rng = np.random.default_rng(1)
    x32 = (rng.standard_normal(50000) * 10.0 ** rng.uniform(-30, 30, 50000)).astype(np.float32)
    # add exact ties at bf16 granularity
    ties = (np.arange(256, 512, dtype=np.uint32) << 16 | 0x8000).view(np.float32)
    x32 = np.concatenate([x32, ties, -ties])
    want = torch.from_numpy(x32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.f64_to_bf16(x32.astype(np.float64)), want)
    assert np.array_equal(workloads.f32_to_bf16_bits(x32), want)
    allb = np.arange(65536, dtype=np.uint16)
    with np.errstate(invalid="ignore"):  # the signalling-NaN patterns among all 65,536
        as64 = workloads.bf16_bits_to_f32(allb).astype(np.float64)
    assert np.array_equal(oracle.bf16_to_f64(allb)[~np.isnan(oracle.bf16_to_f64(allb))],
                          as64[~np.isnan(oracle.bf16_to_f64(allb))])
