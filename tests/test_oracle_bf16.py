"""Pins for the oracle's bf16 conversions: hand-worked IEEE cases, the
library's binary32 -> bf16 conversion on values that binary32 holds exactly,
and the nearest-value property on random doubles."""
import math

import numpy as np
import pytest
import torch

from conftest import closed_form, load_golden


def _bits_to_f64(bits):
    return torch.tensor(np.array(bits, dtype=np.uint16).view(np.int16)).view(torch.bfloat16).double().numpy()


def test_golden_rounding_table(orc):
    g = load_golden("bf16_rounding.json")
    for case in g["cases"]:
        v = closed_form(case["value"])
        got = orc.f64_to_bf16_scalar(v)
        assert got == int(case["bits"], 16), (case, hex(got))


def test_widen_all_patterns_match_library(orc):
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = orc.bf16_to_f64(allbits)
    lib = _bits_to_f64(allbits)
    nan = np.isnan(lib)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], lib[~nan])
    # signed zeros keep their sign
    assert np.array_equal(np.signbit(ours[~nan]), np.signbit(lib[~nan]))


def test_round_trip_every_pattern(orc):
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    v = orc.bf16_to_f64(allbits)
    back = orc.f64_to_bf16(v)
    ok = ~np.isnan(v)
    assert np.array_equal(back[ok], allbits[ok])


def test_binary32_values_match_library_conversion(orc):
    """For a value binary32 holds exactly, rounding it once from fp64 is the
    same as the library's binary32 -> bf16 round-to-nearest-even."""
    g = torch.Generator().manual_seed(0)
    words = torch.randint(0, 2**32, (200000,), generator=g, dtype=torch.int64)
    f = torch.from_numpy(words.numpy().astype(np.uint32).view(np.float32))
    f = f[~torch.isnan(f)]
    # add ties: binary32 words whose low 16 bits are exactly 0x8000
    ties = torch.from_numpy(((words[:20000].numpy().astype(np.uint32) & 0xFFFF0000) | 0x8000)
                            .view(np.float32))
    ties = ties[~torch.isnan(ties)]
    f = torch.cat([f, ties])
    lib = f.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    ours = orc.f64_to_bf16(f.double().numpy())
    assert np.array_equal(ours, lib)


def test_nearest_value_property(orc):
    """The result is a nearest bf16 to the exact double; on a tie the even one."""
    rng = np.random.default_rng(1)
    v = rng.standard_normal(50000) * np.exp2(rng.integers(-30, 30, 50000))
    h = orc.f64_to_bf16(v)
    hv = orc.bf16_to_f64(h)
    up = orc.bf16_to_f64((h.astype(np.int64) + 1).astype(np.uint16))
    dn = orc.bf16_to_f64((h.astype(np.int64) - 1).astype(np.uint16))
    err = np.abs(hv - v)
    assert np.all(err <= np.abs(up - v))
    assert np.all(err <= np.abs(dn - v))
    tie = (err == np.abs(up - v)) | (err == np.abs(dn - v))
    assert np.all(h[tie] % 2 == 0)


def test_monotone(orc):
    rng = np.random.default_rng(2)
    v = np.sort(rng.standard_normal(100000) * 3.0)
    hv = orc.bf16_to_f64(orc.f64_to_bf16(v))
    assert np.all(np.diff(hv) >= 0)
