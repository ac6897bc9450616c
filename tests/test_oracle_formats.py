"""Pins for the oracle's number formats (bf16 rounding, E4M3 encode/decode).

The oracle writes both formats from their definitions; here they are checked
against (a) hand-derived code points of the OCP E4M3 grid (tests/golden/
e4m3_grid.txt) and (b) PyTorch's CPU casts, a library routine that is run,
not read.  A wrong bias, a dropped subnormal branch, round-half-up instead of
ties-to-even or a lost sign each fail one of these.
"""
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _parse_float(tok):
    if tok in ("inf", "-inf"):
        return float(tok)
    if "0x" in tok:
        return float.fromhex(tok)
    return float(tok)


def _torch_e4m3_bytes(v: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(v, np.float32)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


def test_e4m3_golden_grid(oracle):
    vals, codes = [], []
    with open(os.path.join(GOLDEN, "e4m3_grid.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            vals.append(_parse_float(parts[0]))
            codes.append(int(parts[1], 16))
    got = oracle.e4m3_encode(np.array(vals, np.float32))
    for v, c, g in zip(vals, codes, got):
        assert g == c, "e4m3(%r) = %02x, expected %02x" % (v, g, c)


def test_e4m3_decode_all_codes_vs_torch(oracle):
    codes = np.arange(256, dtype=np.uint8)
    mine = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan)
    assert nan.sum() == 2  # 0x7f and 0xff
    assert np.array_equal(mine[~nan].view(np.uint32), ref[~nan].view(np.uint32))
    assert mine[0x7E] == 448.0 and mine[0x01] == 2.0 ** -9 and mine[0x08] == 2.0 ** -6


def test_e4m3_encode_vs_torch_every_bf16_times_scales(oracle):
    # Every bf16 bit pattern, divided by a handful of scales, lands all over
    # the E4M3 range (normal, subnormal, ties).  Inside |v| <= 464 PyTorch's
    # cast rounds to nearest-even like the oracle; beyond it PyTorch gives
    # NaN while the oracle saturates, so that range is checked separately.
    bits = np.arange(65536, dtype=np.uint32) << 16
    base = bits.view(np.float32)
    base = base[np.isfinite(base)]
    for s in (1.0, 3.0, 0.0067, 2.0 ** -7, 117.3, 1.0e-30, 5.5e3):
        with np.errstate(over="ignore"):
            v = (base / np.float32(s)).astype(np.float32)
        v = v[np.isfinite(v)]
        inr = np.abs(v) <= 464.0
        mine = oracle.e4m3_encode(v[inr])
        ref = _torch_e4m3_bytes(v[inr])
        bad = np.nonzero(mine != ref)[0]
        assert bad.size == 0, "scale %r: first mismatch v=%r mine=%02x torch=%02x" % (
            s, v[inr][bad[0]], mine[bad[0]], ref[bad[0]])
        out = v[~inr]
        sat = oracle.e4m3_encode(out)
        assert np.all(sat == np.where(out > 0, 0x7E, 0xFE))


def test_e4m3_encode_random_fp32_vs_torch(oracle):
    rng = np.random.default_rng(7)
    u = rng.integers(0, 2 ** 32, size=1 << 20, dtype=np.uint64).astype(np.uint32)
    v = u.view(np.float32)
    v = v[np.isfinite(v) & (np.abs(v) <= 464.0)]
    assert np.array_equal(oracle.e4m3_encode(v), _torch_e4m3_bytes(v))


def test_e4m3_roundtrip_is_identity_on_grid(oracle):
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    assert np.array_equal(oracle.e4m3_encode(oracle.e4m3_decode(codes)), codes)


def test_bf16_round_vs_torch(oracle):
    rng = np.random.default_rng(11)
    u = rng.integers(0, 2 ** 32, size=1 << 20, dtype=np.uint64).astype(np.uint32)
    # add exact ties and near-ties around the dropped half
    ties = (rng.integers(0, 2 ** 16, size=4096, dtype=np.uint64).astype(np.uint32) << 16) | 0x8000
    u = np.concatenate([u, ties, ties + 1, ties - 1])
    v = u.view(np.float32)
    mine = oracle.bf16_round(v)
    ref = torch.from_numpy(v.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    nan = np.isnan(v)
    # NaN must stay NaN (payload is not specified)
    m_exp = (mine[nan] >> 7) & 0xFF
    assert np.all((m_exp == 0xFF) & ((mine[nan] & 0x7F) != 0))
    assert np.array_equal(mine[~nan], ref[~nan])


def test_bf16_widen_is_exact(oracle):
    b = np.arange(65536, dtype=np.uint16)
    f = oracle.bf16_to_f32(b)
    fin = np.isfinite(f)
    assert np.array_equal(oracle.bf16_round(f[fin]), b[fin])
