"""Kernel-level parity on the GPU through the C ABI: INT4 quantise / dequant and
BF16 rounding are integer/bit work, so they must match the oracle exactly."""
import numpy as np
import pytest

import synthetic as S
from oracle import quant as Q

pytestmark = pytest.mark.gpu


def _special_matrix():
    w = S.random_vectors((16, 256), seed=61, scale=0.02)
    w[0, :32] = 0.0                                               # all-zero group
    w[1, :8] = np.array([0.625, -0.625, 0.125, 0.375, 1.75, 0, 0, 0])  # exact ties at scale 0.25
    w[1, 8:32] = 0.0
    w[2, :32] = 1e-9 * S.random_vectors((32,), seed=62)          # subnormal fp16 scales
    w[3, :32] = 3.0e4 * S.random_vectors((32,), seed=63)         # large scales
    return w


@pytest.mark.parametrize("group", [32, 128])
def test_quantize_int4_bit_exact(group):
    from dynamic_depth_b200 import weights as Wt
    for w in (_special_matrix(), S.random_vectors((3 * 128, 512), seed=64, scale=0.02)):
        gp, gs = Wt.quantize_int4_device(w, group)
        op, os_ = Q.quantize_int4(w, group)
        assert np.array_equal(gp, op)
        assert np.array_equal(gs, os_.view(np.uint16))


def test_quantize_real_407m_matrix_bit_exact():
    from dynamic_depth_b200 import weights as Wt
    for name, w in S.master_weights(S.M407):
        if name == "pre0.wd":
            gp, gs = Wt.quantize_int4_device(w, 128)
            op, os_ = Q.quantize_int4(w, 128)
            assert np.array_equal(gp, op) and np.array_equal(gs, os_.view(np.uint16))
            break


def test_dequant_int4_bit_exact():
    import torch
    from dynamic_depth_b200 import lib, check
    rng = np.random.default_rng(65)
    N, K, g = 64, 512, 128
    packed = rng.integers(0, 256, (N, K // 2)).astype(np.uint8)   # every nibble value, including u = 0
    scales = (rng.standard_normal((N, K // g)) * 0.01).astype(np.float16)
    want = Q.dequantize_int4(packed, scales, g)
    dp = torch.from_numpy(packed).cuda()
    ds = torch.from_numpy(scales.view(np.int16)).cuda()
    out = torch.empty((N, K), dtype=torch.float32, device="cuda")
    check(lib().tl_dequant_int4(dp.data_ptr(), ds.data_ptr(), N, K, g, out.data_ptr(),
                                torch.cuda.current_stream().cuda_stream), "dequant")
    got = out.cpu().numpy().astype(np.float64)
    assert np.array_equal(got, want)


def test_round_bf16_bit_exact():
    from dynamic_depth_b200 import weights as Wt
    x = np.concatenate([
        S.random_vectors((100000,), seed=66, scale=0.02),
        np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -8 + 2 ** -40, -(1 + 2 ** -8 + 2 ** -40), 0.0, -0.0,
                  2.0 ** -133 * 0.75, 2.0 ** -130 * 1.5, 2.0 ** -127, 3.0e38, -1e-45]),
    ])
    got = Wt.round_bf16_device(x)
    assert np.array_equal(got, Q.bf16_bits(x))
