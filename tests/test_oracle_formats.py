"""Pins for the oracle's number formats and FP4 pack, no GPU.

Each check ties the oracle to something other than itself: the OCP format tables (golden fixtures),
torch's FP8 E4M3 cast (a library routine), brute-force nearest-value search, exact round trips and
the quantisation error bound."""
import os

import numpy as np
import pytest
import torch

from oracle import csa_oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _read_table(name):
    rows = []
    for line in open(os.path.join(GOLD, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        a, b = line.split()
        rows.append((int(a, 0), float(b)))
    return rows


def test_e4m3_golden_codes():
    for code, val in _read_table("e4m3_codes.txt"):
        got = O.e4m3_decode(code)
        assert got == val and np.signbit(got) == np.signbit(val), hex(code)


def test_e4m3_decode_all_codes_vs_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = O.e4m3_decode(np.arange(256))
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    ok = ~np.isnan(ref)
    assert np.array_equal(ref[ok], got[ok])


def test_e4m3_encode_roundtrip_all_nonnegative_codes():
    codes = np.arange(0x7F)            # 0x00 .. 0x7E, all finite non-negative
    assert np.array_equal(O.e4m3_encode(O.e4m3_decode(codes)), codes)


def test_e4m3_rounding_vs_torch_cast():
    # dense sweep of fp32 values over the whole E4M3 range, plus every midpoint between neighbours
    vals = O.e4m3_decode(np.arange(0x7F))
    mids = (vals[:-1] + vals[1:]) / 2
    rng = np.random.default_rng(0)
    rand = np.exp(rng.uniform(np.log(2.0 ** -12), np.log(448.0), 20000))
    x = np.concatenate([vals, mids, rand, -rand]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = O.e4m3_rne_satfinite(x.astype(np.float64))
    assert np.array_equal(ref, got)


def test_e4m3_saturates():
    assert O.e4m3_rne_satfinite(np.array([464.0, 1e6]))[0] == 448.0
    assert O.e4m3_rne_satfinite(np.array([1e6]))[0] == 448.0
    # below half the smallest subnormal -> 0
    assert O.e4m3_rne_satfinite(np.array([2.0 ** -11]))[0] == 0.0


def test_e2m1_golden_codes():
    for code, val in _read_table("e2m1_codes.txt"):
        got = O.e2m1_decode(code)
        assert got == val and (code == 8 or np.signbit(got) == np.signbit(val))


def test_e2m1_rounding_brute_force():
    """Nearest E2M1 value by exhaustive search, ties to the even code (mantissa bit 0)."""
    mags = np.array(O.E2M1_MAGNITUDES)
    x = np.concatenate([np.linspace(-8, 8, 4001), (mags[:-1] + mags[1:]) / 2,
                        -(mags[:-1] + mags[1:]) / 2])
    got = O.e2m1_rne_satfinite(x)
    for xi, gi in zip(x, got):
        a = min(abs(xi), 6.0)
        dist = np.abs(mags - a)
        best = np.flatnonzero(dist == dist.min())
        if len(best) > 1:
            best = [b for b in best if b % 2 == 0]
        assert abs(gi) == mags[best[0]], (xi, gi)


def test_bf16_round_vs_torch_on_fp32_inputs():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(50000) * np.exp(rng.uniform(-30, 30, 50000))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.bf16_round(x.astype(np.float64)), ref)


# ------------------------------------------------------------------------------------------ pack

def _block_from_codes(codes4, s, g):
    return O.e2m1_decode(codes4) * s * g


@pytest.mark.parametrize("g", [1.0, 2.0 ** -4, 8.0])
def test_pack_roundtrip_all_scales_all_codes(g):
    """Every finite positive E4M3 scale x every E2M1 code: a block whose max magnitude is 6·s·g packs
    back to exactly its codes and scale."""
    rng = np.random.default_rng(2)
    scales = O.e4m3_decode(np.arange(1, 0x7F))
    rows = []
    want_codes, want_scale = [], []
    for s in scales:
        c = rng.choice([0, 1, 2, 3, 4, 5, 6, 7, 9, 10, 11, 12, 13, 14, 15], size=32)
        c[rng.integers(32)] = rng.choice([7, 15])         # forces amax = 6 s g
        c[:16] = np.arange(16) % 16 if s == scales[40] else c[:16]
        c[c == 8] = 0
        if not np.any((c & 7) == 7):
            c[0] = 7
        rows.append(_block_from_codes(c, s, g))
        want_codes.append(c)
        want_scale.append(s)
    src = np.array(rows)
    codes, sc, rope = O.pack_fp4(src, 0, g)
    got4 = O.unpack_codes(codes, 32)
    assert np.array_equal(got4, np.array(want_codes, dtype=np.uint8))
    assert np.array_equal(O.e4m3_decode(sc[:, 0]), np.array(want_scale))
    assert np.all(sc[:, 1:] == 0)                                      # scale row padding
    assert np.array_equal(O.dequant_fp4(codes, sc, 32, g), src)


def test_pack_error_bound_and_layout():
    rng = np.random.default_rng(3)
    src = O.bf16_round(rng.standard_normal((64, 448 + 64)) * 3)
    codes, sc, rope = O.pack_fp4(src, 64, 1.0)
    assert codes.shape == (64, 224) and sc.shape == (64, 16) and rope.shape == (64, 64)
    assert np.array_equal(rope, src[:, 448:])
    deq = O.dequant_fp4(codes, sc, 448, 1.0)
    s = np.repeat(O.e4m3_decode(sc[:, :14]), 32, axis=1)
    q = src[:, :448] / s
    # half the local E2M1 spacing, or the saturation excess above 6
    spacing = np.where(np.abs(q) < 2, 0.5, np.where(np.abs(q) < 4, 1.0, 2.0))
    bound = np.maximum(spacing / 2, np.abs(q) - 6.0) * s * (1 + 1e-6)
    assert np.all(np.abs(deq - src[:, :448]) <= bound)


def test_pack_nibble_order_zero_block_and_negative_zero():
    src = np.zeros((2, 64))
    src[0, 0] = 0.5 * 1.0 * 12 / 12      # code 1 at element 0 if s = 1
    src[0, 1] = 1.0                      # code 2 at element 1
    src[0, 2] = 6.0                      # amax = 6 -> s = 1
    src[0, 3] = -1e-3                    # rounds to -0 -> written as +0
    codes, sc, _ = O.pack_fp4(src, 0, 1.0)
    assert codes[0, 0] == 0x21           # element 0 low nibble, element 1 high nibble
    assert codes[0, 1] == 0x07           # element 2 = +6, element 3 = +0 (not 0x8)
    assert O.e4m3_decode(sc[0, 0]) == 1.0
    assert np.all(codes[1] == 0) and np.all(sc[1] == 0)            # all-zero block: scale 0, codes 0
    assert np.all(codes[0, 16:] == 0) and sc[0, 1] == 0


def test_pack_tiny_block_scale_underflow_zeroes_block():
    src = np.zeros((1, 32))
    src[0, :] = 2.0 ** -14                                 # amax/6 < half the smallest E4M3 subnormal
    codes, sc, _ = O.pack_fp4(src, 0, 1.0)
    assert np.all(codes == 0) and sc[0, 0] == 0
    codes, sc, _ = O.pack_fp4(src, 0, 2.0 ** -8)           # a global scale brings it back in range
    assert sc[0, 0] != 0 and np.all(O.dequant_fp4(codes, sc, 32, 2.0 ** -8) > 0)


# ------------------------------------------------------------------------------------ FP8 window

def test_fp8_window_exact_round_trip_at_power_of_two_scales():
    """Blocks built from E4M3 grid values times 2^k with 448 * 2^k present: the block scale is exactly
    2^k and every code comes back (positive and negative codes, subnormals included)."""
    grid = O.e4m3_decode(np.arange(0, 0x7F))                  # every finite non-negative E4M3 value
    rng = np.random.default_rng(5)
    for k in (-8, 0, 3):
        vals = rng.choice(grid, size=(4, 128)) * rng.choice([-1.0, 1.0], size=(4, 128))
        vals[:, 0] = 448.0
        vals[:, 64] = -448.0
        rows = np.concatenate([vals * 2.0 ** k, rng.standard_normal((4, 32))], axis=1)
        codes, scales, rope = O.pack_fp8_window(rows, 32)
        assert np.all(scales == np.float32(2.0 ** k))
        assert np.array_equal(O.dequant_fp8_window(codes, scales, rope), rows)


def test_fp8_window_error_bound_zero_blocks_and_rope():
    """|x - x_hat| <= half an E4M3 step at |x| / s (2^-4 relative for normals, 2^-10 s for subnormals);
    an all-zero block packs to scale 0 and zero codes; the RoPE channels pass through."""
    rng = np.random.default_rng(6)
    rows = O.bf16_round(rng.standard_normal((16, 192)) * np.exp(rng.uniform(-6, 6, size=(16, 1))))
    rows[3, :64] = 0.0
    codes, scales, rope = O.pack_fp8_window(rows, 64)
    assert scales[3, 0] == 0 and not codes[3, :64].any()
    back = O.dequant_fp8_window(codes, scales, rope)
    assert np.array_equal(back[:, 128:], rows[:, 128:])
    s = np.repeat(scales.astype(np.float64), 64, axis=1)
    x = rows[:, :128]
    err = np.abs(back[:, :128] - x)
    a = np.abs(x) / np.where(s > 0, s, 1.0)
    bound = np.where(a >= 2.0 ** -6, np.ldexp(1.0, np.floor(np.log2(np.maximum(a, 2.0 ** -6))).astype(int) - 4),
                     2.0 ** -10) * s
    assert np.all(err <= bound * (1 + 1e-6) + 1e-300)
    assert np.all(np.abs(back[:, :128]).max(axis=1) <= 448.0 * s.max(axis=1) * (1 + 1e-7))


def test_paged_rows_brute_force_and_identity_table():
    """Entry i of a paged cache is slot i % page of page table[i // page]: checked element by element
    against a loop over the pages, and an identity table over a contiguous pool gives the rows back."""
    rng = np.random.default_rng(7)
    page, n_pages = 16, 12
    pool = rng.standard_normal((n_pages, page, 5))
    table = rng.permutation(n_pages)[:7]
    n = 7 * page - 3
    got = O.paged_rows(pool, table, page, n)
    want = []
    for p_i, phys in enumerate(table):
        for slot in range(page):
            if p_i * page + slot < n:
                want.append(pool[phys, slot])
    assert np.array_equal(got, np.array(want))
    flat = rng.standard_normal((4 * page, 5))
    assert np.array_equal(O.paged_rows(flat.reshape(4, page, 5), np.arange(4), page, 4 * page - 1), flat[:-1])
