"""The test-side e4m3 codec against its definition and torch's conversion."""
import numpy as np
import torch

from tests import e4m3


def test_decode_known_codes():
    assert e4m3.decode(np.array([0x00, 0x01, 0x08, 0x38, 0x7E, 0xFE, 0x80]))[:6].tolist() == \
        [0.0, 2.0 ** -9, 2.0 ** -6, 1.0, 448.0, -448.0]
    assert np.isnan(e4m3.decode(np.array([0x7F, 0xFF]))).all()
    assert np.signbit(e4m3.decode(np.array([0x80])))[0]


def test_quantize_is_identity_on_codes():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    assert np.array_equal(e4m3.quantize(e4m3.decode(codes).astype(np.float32)), codes)


def test_quantize_matches_torch_in_range():
    rng = np.random.default_rng(0)
    y = np.concatenate([rng.standard_normal(20000) * 50, rng.standard_normal(2000) * 1e-2,
                        rng.uniform(-448, 448, 5000)]).astype(np.float32)
    ref = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(e4m3.quantize(y), ref)


def test_quantize_ties_and_saturation():
    # 1.0625 lies halfway between 1.0 (code 0x38) and 1.125 (0x39): even code wins.
    assert e4m3.quantize(np.float32([1.0625, 1.1875]))[:2].tolist() == [0x38, 0x3A]
    assert e4m3.quantize(np.float32([1e4, -1e4, 464.0])).tolist() == [0x7E, 0xFE, 0x7E]
    assert e4m3.quantize(np.float32([np.nan]))[0] == 0x7F
