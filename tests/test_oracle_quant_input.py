"""Pins of the oracle's activation quantiser (BF16 rows -> E4M3 codes + 1x128 power-of-two
scales), the step before dispatch for BF16 input to an E4M3 layer (youleyou, "DeepSeek 模型
更新解读 Tile Kernels 与 DeepEP V2 新特性", Tile Kernels feature list, quantisation item)."""
import numpy as np
import torch

import oracle


def _bf16_bits(v):
    return torch.tensor(v, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy() \
        .view(np.uint16)


def test_scale_boundaries_and_zero_block():
    # block 0: amax exactly 448 * 2^3 -> scale 2^3; block 1: the next BF16 above it -> 2^4;
    # block 2: all zero -> scale 1 and zero codes; block 3: tiny values -> negative exponent
    row = np.zeros(512, np.float32)
    row[5] = 448.0 * 8
    row[128 + 7] = -448.0 * 8 * (1 + 2.0 ** -7)
    row[128 + 8] = 1.0
    row[384:] = np.linspace(-3e-4, 3e-4, 128, dtype=np.float32)
    bits = _bf16_bits(row[None, :])
    codes, scales = oracle.quantize_activations(bits)
    assert scales[0, 0] == 8.0 and scales[0, 1] == 16.0 and scales[0, 2] == 1.0
    assert np.all(codes[0, 256:384] == 0)
    s3 = float(scales[0, 3])
    assert s3 < 1.0 and np.log2(s3) == round(np.log2(s3))
    # the largest magnitude lands on 448 exactly in block 0
    assert oracle.e4m3_decode(codes[0, 5:6])[0] == 448.0


def test_tiny_blocks_take_the_smallest_normal_scale():
    # amax = 1e-38 would need 2^-135; the scale stays a normal fp32 power of two, 2^-126,
    # and the codes are those of x * 2^126 (about 0.85 -> 0.875)
    row = np.full((1, 128), 1.0e-38, np.float32)
    bits = _bf16_bits(row)
    codes, scales = oracle.quantize_activations(bits)
    assert scales[0, 0] == np.float32(2.0 ** -126)
    xv = oracle.bf16_bits_to_f64(bits)[0, 0]
    ref = torch.tensor([xv * 2.0 ** 126], dtype=torch.float32).to(torch.float8_e4m3fn).double()
    assert oracle.e4m3_decode(codes[0, :1])[0] == float(ref[0]) == 0.875


def test_codes_are_the_float8_cast_of_the_scaled_bf16_values():
    rng = np.random.default_rng(11)
    x = (rng.standard_normal((6, 1024)) * np.array([1e-2, 1, 30])[:, None].repeat(2, 0))
    bits = _bf16_bits(x.astype(np.float32))
    codes, scales = oracle.quantize_activations(bits)
    xv = oracle.bf16_bits_to_f64(bits)
    blocks = np.abs(xv).reshape(6, 8, 128).max(2)
    assert np.all(blocks <= 448 * scales) and np.all(blocks > 224 * scales)
    ref = torch.from_numpy((xv.reshape(6, 8, 128) / scales[:, :, None]).reshape(6, 1024)
                           .astype(np.float32)).to(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(ref, oracle.e4m3_decode(codes))
    # dequantised values are within half an E4M3 step (relative 2^-4) of the input
    deq = oracle.dequant_x(codes, scales, "e4m3")
    big = np.abs(xv) > 2.0 ** -6 * np.repeat(scales, 128, 1)
    assert np.all(np.abs(deq - xv)[big] <= 2.0 ** -4 * np.abs(xv)[big])
