"""Pins of the oracle's e4m3 decoder (oracle/fp8.py): hand-derived codes from the format
definition, and every one of the 256 codes against the library's float8_e4m3fn conversion."""
import numpy as np
import torch

from oracle import decode_e4m3


def test_hand_codes():
    # 0x38: exponent 7, mantissa 0 -> 1.0; 0x7E: exponent 15, mantissa 6 -> 1.75 * 2^8 = 448;
    # 0x01: subnormal 1/8 * 2^-6 = 2^-9; 0xC2: -(1 + 2/8) * 2^(8 - 7) = -2.5; 0x00 / 0x80: +-0
    codes = np.array([0x38, 0x7E, 0x01, 0xC2, 0x00, 0x80, 0x08, 0x07], np.uint8)
    want = [1.0, 448.0, 2.0 ** -9, -2.5, 0.0, -0.0, 2.0 ** -6, 7 / 8 * 2.0 ** -6]
    assert decode_e4m3(codes).tolist() == want
    assert np.isnan(decode_e4m3(np.array([0x7F, 0xFF], np.uint8))).all()


def test_all_codes_match_library():
    codes = np.arange(256, dtype=np.uint8)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = decode_e4m3(codes)
    both_nan = np.isnan(lib) & np.isnan(ours)
    assert np.array_equal(np.where(both_nan, 0, lib), np.where(both_nan, 0, ours))
    assert np.array_equal(np.isnan(lib), np.isnan(ours))
