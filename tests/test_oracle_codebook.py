"""Pins for the oracle's 1MAD codebook (QTIP blog, "The codebook is computed").

The pages fix: the LCG constants, the byte sum of the LCG output (Irwin-Hall
with n = 4), the centring by 510 = 4 * 127.5 and the scale 147.8 =
sqrt(4 (256^2 - 1) / 12), and that 1MAD at L = 16 takes exactly 908 distinct
values over the 65,536 states.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np

import oracle

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")))


def test_908_distinct_values_at_L16():
    # printed on the page; any slip in the LCG constants or the byte sum moves it
    assert len(np.unique(oracle.codebook_f64(16))) == GOLD["one_mad_distinct_values_L16"]["value"]


def test_irwin_hall_closed_form_of_the_constants():
    c = GOLD["one_mad_constants"]
    # the multiplier is odd, so x -> a x + b is a bijection of Z/2^32 and a
    # uniform 32-bit input gives a uniform output: its byte sum is Irwin-Hall(4)
    assert c["lcg_multiplier"] % 2 == 1
    mean = 4 * 127.5
    var = 4 * (256 ** 2 - 1) / 12
    assert mean == c["centre"]
    assert round(math.sqrt(var), 1) == c["scale"]


def test_special_states_follow_the_printed_constants():
    # Two states whose LCG output the printed constants fix without the
    # multiplication: at x = 0 the output is the increment itself, and at
    # x = 2^31 an odd multiplier gives a x = 2^31 (mod 2^32), so the output is
    # the increment with its top bit flipped.  The increment 76625530 =
    # 0x0491367A has bytes 4, 145, 54, 122 (sum 325); flipping its top bit
    # raises the top byte from 4 to 132 (sum 453).
    inc = GOLD["one_mad_constants"]["lcg_increment"]
    assert inc == 0x0491367A
    assert oracle.bytesum_1mad(0) == 4 + 145 + 54 + 122 == 325
    assert oracle.bytesum_1mad(2 ** 31) == 132 + 145 + 54 + 122 == 453
    # the table is indexed by the state itself: entry 0 is that value, centred
    # and scaled, at every L
    for L in (8, 12, 16):
        assert oracle.codebook_f64(L)[0] == (325.0 - 510.0) / 147.8


def test_bytesum_distribution_matches_irwin_hall():
    # sample uniform 32-bit inputs; by the bijection above the oracle's byte sum
    # must follow the n=4 discrete uniform-sum law (mean 510, var 21845).
    rng = np.random.default_rng(123)
    xs = rng.integers(0, 2 ** 32, 200_000, dtype=np.uint64)
    bs = np.array([oracle.bytesum_1mad(int(x)) for x in xs[:20000]], dtype=np.float64)
    n = bs.size
    assert abs(bs.mean() - 510.0) < 5 * math.sqrt(21845.0 / n)
    assert abs(bs.var() / 21845.0 - 1.0) < 0.05
    # exact law of the sum of 4 bytes: P(sum = 0) = P(sum = 1020) = 2^-32
    assert bs.min() >= 0 and bs.max() <= 1020


def test_codebook_moments_are_standard_normal_like():
    c = oracle.codebook_f64(16)
    assert abs(c.mean()) < 0.01
    assert abs(c.std() - 1.0) < 0.01


def test_fp32_codebook_is_correctly_rounded_page_value():
    # the fp32 table is the page's fp64 value rounded once; check against the
    # exact rational (bytesum - 510) / 147.8 for every reachable byte sum.
    b = Fraction(147.8)
    c32 = oracle.codebook_f32(16)
    c64 = oracle.codebook_f64(16)
    for j in range(0, 1 << 16, 97):
        ex = (Fraction(oracle.bytesum_1mad(j)) - 510) / b
        v = np.float32(c32[j])
        lo = np.nextafter(v, np.float32(-np.inf))
        hi = np.nextafter(v, np.float32(np.inf))
        err = abs(Fraction(float(v)) - ex)
        assert err <= abs(Fraction(float(lo)) - ex) and err <= abs(Fraction(float(hi)) - ex)
        assert float(c64[j]) == float(Fraction(oracle.bytesum_1mad(j) - 510) / b) or \
            abs(float(c64[j]) - float(ex)) <= 2 ** -52 * 4


def test_fp16_codebook_is_round_to_nearest_even():
    c16 = oracle.codebook_f16(12).astype(np.float64)
    c64 = oracle.codebook_f64(12)
    # |fp16 - exact| at most half an fp16 ulp
    ulp = np.spacing(np.abs(c16).astype(np.float16)).astype(np.float64)
    assert np.all(np.abs(c16 - c64) <= ulp / 2 + 1e-18)
