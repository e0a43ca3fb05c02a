"""Planted mistakes in the CPU oracle must fail its pins.

Each case edits the oracle's source at one spot (two for the tile padding)
the way a plausible slip would (a dropped term, a wrong sign, index or rounding, a swapped operand),
compiles the edited source as a separate module in memory, and runs the pins
named beside it against that module: at least one of them must fail, while
all of them pass against the unedited oracle.  Nothing is written to disk and
the oracle module itself is not modified."""
import importlib.util
import os
import types

import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
with open(oracle.__file__) as _f:
    ORACLE_SRC = _f.read()


def _pins_against(module):
    """A fresh copy of the pin tests whose `oracle` is `module`."""
    spec = importlib.util.spec_from_file_location(
        f"_pins_{id(module)}", os.path.join(HERE, "test_oracle_pins.py"))
    pins = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(pins)
    pins.oracle = module
    return pins


def _edit(src, old, new, after):
    start = src.index(after) if after else 0
    i = src.index(old, start)
    if after is None:
        assert src.count(old) == 1, f"ambiguous edit: {old!r}"
    return src[:i] + new + src[i + len(old):]


def _edited_oracle(old, new, after=None):
    """The oracle with `old` replaced by `new` (the first occurrence after
    `after`); `old` may also be a list of (old, new) pairs, all applied."""
    edits = old if isinstance(old, list) else [(old, new)]
    src = ORACLE_SRC
    for o, n in edits:
        src = _edit(src, o, n, after)
    mod = types.ModuleType("oracle_edited")
    exec(compile(src, "oracle_edited", "exec"), mod.__dict__)
    return mod


P13_1x1_S2 = dict(symmetric=False, H=4, W=4, Cin=64, KH=1, KW=1, stride=(2, 2), pad=(0, 0))
P13_3x3_P1 = dict(symmetric=False, H=5, W=6, Cin=32, KH=3, KW=3, stride=(1, 1), pad=(1, 1))

# name: (old text, new text, edit only after this marker, [(pin, kwargs), ...]).
# Padding only one operand with raw zeros is not a mistake (its padded
# products meet the other operand's zero-point padding, (q - z) = 0), so the
# tile case pads both.
CASES = {
    "multiplier rounded down": (
        "m0 = math.floor(f * 2.0 ** 31 + 0.5)", "m0 = math.floor(f * 2.0 ** 31)", None,
        [("test_requant_params_closed_forms", {})]),
    "multiplier carry not taken": (
        "    if m0 == 2 ** 31:\n        m0 //= 2\n        e += 1\n", "", None,
        [("test_requant_params_carry_into_the_next_power_of_two", {})]),
    "requant ties rounded up": (
        "up = (r > half) | ((r == half) & ((q & 1) == 1))", "up = (r >= half)", None,
        [("test_requant_round_half_even_cases", {})]),
    "requant shift off by one": (
        "round_half_even_shift(acc * m0, 31 + shift)", "round_half_even_shift(acc * m0, 30 + shift)",
        None, [("test_requant_round_half_even_cases", {})]),
    "output zero-point dropped": (
        "y = np.clip(q + int(out_zp),", "y = np.clip(q,", None,
        [("test_requant_round_half_even_cases", {})]),
    "float64 route drops the activation zero-point": (
        "Af = A[r0:r0 + row_block].astype(np.float64) - float(za)",
        "Af = A[r0:r0 + row_block].astype(np.float64)", None,
        [("test_p5_float64_accumulation_is_exact_against_int64_loops", {})]),
    "float64 route in float32": (
        "blocks.append((Af @ Bf).astype(np.int64))",
        "blocks.append((Af.astype(np.float32) @ Bf.astype(np.float32)).astype(np.int64))",
        None, [("test_p5_float64_accumulation_is_exact_against_int64_loops", {})]),
    "float64 route skips the last row block": (
        "for r0 in range(0, A.shape[0], row_block):",
        "for r0 in range(0, A.shape[0] - row_block, row_block):", None,
        [("test_p5_float64_accumulation_is_exact_against_int64_loops", {})]),
    "weight zero-point dropped": (
        "B = np.asarray(B, dtype=np.int64) - int(zb)", "B = np.asarray(B, dtype=np.int64)", None,
        [("test_p5_float_dequant_reference", {})]),
    "activation zero-point sign": (
        "A = np.asarray(A, dtype=np.int64) - int(za)", "A = np.asarray(A, dtype=np.int64) + int(za)",
        None, [("test_p5_float_dequant_reference", {})]),
    "GEMM bias dropped": (
        "acc = acc + np.asarray(bias, dtype=np.int64)[None, :]", "acc = acc", "def int8_gemm_acc",
        [("test_p5_gemm_brute_force_loops", {})]),
    "tiles padded with raw zeros": (
        [("Ap = np.full((mt * Tm, kt * Tk), int(za), dtype=np.int64)",
          "Ap = np.zeros((mt * Tm, kt * Tk), dtype=np.int64)"),
         ("Bp = np.full((kt * Tk, nt * Tn), int(zb), dtype=np.int64)",
          "Bp = np.zeros((kt * Tk, nt * Tn), dtype=np.int64)")], None, None,
        [("test_p1_tiling_counts_match_page", {})]),
    "accumulator reset per K block": (
        "                accum += a_t @ b_t", "                accum = a_t @ b_t", None,
        [("test_p1_tiling_counts_match_page", {})]),
    "input tiles not double-buffered": (
        "s_input = 2 * (Tm * Tk + Tk * Tn)", "s_input = (Tm * Tk + Tk * Tn)", None,
        [("test_p1_buffer_budget_matches_page", {})]),
    "overflow bound magnitude 254": (
        "return INT8_MAX - INT8_MIN", "return INT8_MAX - INT8_MIN - 1", None,
        [("test_p2_overflow_constants", {})]),
    "conv pad taps read as raw 0": (
        "    xc = x - int(za)\n", "    xc = x - int(za) * 0\n", None,
        [("test_conv_brute_force_loops", {})]),
    "conv kernel rows flipped": (
        "ih = np.arange(OH) * sh + kh - ph", "ih = np.arange(OH) * sh + (KH - 1 - kh) - ph", None,
        [("test_conv_brute_force_loops", {})]),
    "range without zero": (
        "rmin = min(f32(0.0), row.min()) if K else f32(0.0)", "rmin = row.min() if K else f32(0.0)",
        None, [("test_p6_constant_row_and_error_bound", {})]),
    "scale over 256 levels": (
        "s = f32(f32(rmax) - f32(rmin)) / f32(255.0)", "s = f32(f32(rmax) - f32(rmin)) / f32(256.0)",
        None, [("test_p6_quantization_specials", {})]),
    "zero-point sign": (
        "np.rint(f32(f32(-128.0) - t))", "np.rint(f32(f32(-128.0) + t))", None,
        [("test_p6_quantization_specials", {})]),
    "codes rounded down": (
        "r = np.rint((row * inv).astype(np.float32))", "r = np.floor((row * inv).astype(np.float32))",
        None, [("test_p6_quantization_specials", {})]),
    "nibbles swapped": (
        "nib = (u[:, :, 0, :] | (u[:, :, 1, :] << 4))", "nib = (u[:, :, 1, :] | (u[:, :, 0, :] << 4))",
        None, [("test_p8_w4_pack_round_trip_and_bytes", {})]),
    "nibbles without the offset of 8": (
        "u = (qw + 8).reshape(N, K // 8, 2, 4)", "u = (qw & 0xF).reshape(N, K // 8, 2, 4)", None,
        [("test_p8_w4_pack_round_trip_and_bytes", {})]),
    "bf16 truncated": (
        "return ((u + 0x7FFF + kept_lsb) >> 16).astype(np.uint16)",
        "return (u >> 16).astype(np.uint16)", None,
        [("test_p9_bf16_rounding_hand_derived_cases", {})]),
    "bf16 ties rounded up": (
        "return ((u + 0x7FFF + kept_lsb) >> 16).astype(np.uint16)",
        "return ((u + 0x8000) >> 16).astype(np.uint16)", None,
        [("test_p9_bf16_rounding_hand_derived_cases", {})]),
    "A8W4 activation zero-point dropped": (
        "a = (qA[m].astype(np.int64) - int(za[m])).reshape(G, GROUP)",
        "a = qA[m].astype(np.int64).reshape(G, GROUP)", "def qgemm_a8w4_f32(",
        [("test_p7_a8w4_brute_force_loops", {}), ("test_p7_a8w4_float_reference", {})]),
    "A8W4 clamp before the bias": (
        "            comb = comb + np.asarray(bias, np.float64)\n"
        "        y[m] = np.minimum(np.maximum(comb.astype(np.float32), lo), hi)",
        "            comb = np.minimum(np.maximum(comb, float(lo)), float(hi))"
        " + np.asarray(bias, np.float64)\n"
        "        y[m] = comb.astype(np.float32)", "def qgemm_a8w4_f32(",
        [("test_p7_a8w4_brute_force_loops", {})]),
    "per-block codes with the first block's zero-point": (
        "- za[m].astype(np.int64)[:, None]", "- int(za[m][0])", None,
        [("test_p10_blockwise_brute_force_loops", {})]),
    "per-block codes with the first block's scale": (
        "sA[m].astype(np.float64)[None, :]", "np.float64(sA[m][0])", None,
        [("test_p10_blockwise_brute_force_loops", {})]),
    "weight-zero term dropped": (
        " + zwd * sa * S.astype(np.float64)[None, :]", "", None,
        [("test_p11_equals_dense_float_product_of_dequantized_operands", {})]),
    "group sums of raw codes": (
        "        S = a.sum(axis=1)", "        S = qA[m].astype(np.int64).reshape(G, GROUP).sum(axis=1)",
        None, [("test_p11_equals_dense_float_product_of_dequantized_operands", {})]),
    "symmetric codes clamped at 126": (
        "np.clip(r, -127, 127)", "np.clip(r, -126, 126)", None,
        [("test_p12_symmetric_hand_derived_rows", {})]),
    "unrolled rows ignore the stride": (
        "iw = ow * sw + kw - pw", "iw = ow + kw - pw", None,
        [("test_p13_dynamic_conv_equals_direct_brute_force", P13_1x1_S2)]),
    "unrolled rows with the pad added": (
        "ih = oh * sh + kh - ph", "ih = oh * sh + kh + ph", None,
        [("test_p13_dynamic_conv_equals_direct_brute_force", P13_3x3_P1)]),
    "codes entry drops the zero-point": (
        "a = (qA[m].astype(np.int64) - int(za[m])).reshape(G, GROUP)",
        "a = qA[m].astype(np.int64).reshape(G, GROUP)", "def a8w4_from_codes",
        [("test_p13_codes_entry_matches_the_linear", {})]),
}


@pytest.fixture(scope="module")
def true_pins():
    return _pins_against(oracle)


@pytest.mark.parametrize("name", list(CASES))
def test_planted_mistake_fails_a_pin(true_pins, name):
    old, new, after, checks = CASES[name]
    for pin, kw in checks:                      # the pins hold for the oracle as written
        getattr(true_pins, pin)(**kw)
    pins = _pins_against(_edited_oracle(old, new, after))
    failed = []
    for pin, kw in checks:
        try:
            getattr(pins, pin)(**kw)
        except Exception as e:                  # an assertion, or a value the pin rejects
            failed.append(f"{pin}: {type(e).__name__}")
    assert failed, f"no pin caught the planted mistake: {name}"
