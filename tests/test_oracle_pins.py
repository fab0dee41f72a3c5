"""The oracle against its pins (CPU only), and the pins against planted mistakes."""
from __future__ import annotations

import os
import re
import subprocess

import numpy as np
import pytest
import torch

import oracle
from tests import oracle_pins as P


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin, oracle_mod):
    pin(oracle_mod.default())


# ---------------------------------------------------------------------------
# element codecs: IEEE binary16 and bfloat16 from their bit-field definitions
# ---------------------------------------------------------------------------

def test_f16_decoder_all_patterns(oracle_mod):
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = oracle_mod.decode(bits, "f16")
    ref = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def test_bf16_decoder_all_patterns(oracle_mod):
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = oracle_mod.decode(bits, "bf16")
    ref = torch.from_numpy(bits.astype(np.int16)).view(torch.bfloat16).double().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def _edge_values():
    rng = np.random.default_rng(11)
    v = [0.0, -0.0, 1.0, -1.0, 65504.0, 65519.99, 65520.0, -65520.0, 1e-8, 2.0 ** -24, 2.0 ** -25,
         3 * 2.0 ** -26, 2.0 ** -14, 2.0 ** -14 - 2.0 ** -25, 1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11,
         1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, 3.3895313892515355e38, 3.4e38, 1e-40, 9.2e-41,
         float("inf"), float("-inf")]
    v += list(rng.standard_normal(3000) * 10.0 ** rng.integers(-9, 6, 3000))
    return np.array(v, dtype=np.float64)


def test_f16_encoder_matches_numpy(oracle_mod):
    v = _edge_values()
    got = oracle_mod.round_bits(v, "f16")
    with np.errstate(over="ignore"):
        ref = v.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, ref)


def test_bf16_encoder_matches_torch_on_float32_values(oracle_mod):
    # values exactly representable in float32, where torch's float32 -> bfloat16
    # cast (round to nearest even) is a single rounding
    v = _edge_values().astype(np.float32)
    v = v[np.isfinite(v) | np.isinf(v)]
    got = oracle_mod.round_bits(v.astype(np.float64), "bf16")
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)


def test_bf16_vector_encoder_matches_scalar(oracle_mod):
    v = _edge_values()
    rng = np.random.default_rng(12)
    v = np.concatenate([v, rng.standard_normal(5000) * 3.0])
    assert np.array_equal(oracle._bf16_rn_vector(v), oracle_mod.round_bits(v, "bf16"))


def test_round_to_is_nearest(oracle_mod):
    # the rounded value is never farther than half a quantum, ties to even
    v = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, 1 + 2.0 ** -8 + 2.0 ** -40])
    r = oracle_mod.round_to(v, "bf16")
    assert r[0] == 1.0 and r[1] == 1 + 2.0 ** -6 and r[2] == 1 + 2.0 ** -7


# ---------------------------------------------------------------------------
# planted mistakes: each mutated copy of the C oracle must fail some pin
# ---------------------------------------------------------------------------

_SRC = os.path.join(os.path.dirname(oracle.__file__), "conv_ref.c")

MUTATIONS = {
    "flipped_kernel": [(r"\(int64_t\)kh \* sh->d\[1\]", "(int64_t)(sh->kH - 1 - kh) * sh->d[1]"),
                       (r"\(int64_t\)kw \* sh->d\[2\]", "(int64_t)(sh->kW - 1 - kw) * sh->d[2]")],
    "pad_sign": [(r"\(int64_t\)oh \* sh->s\[1\] - sh->p\[1\]", "(int64_t)oh * sh->s[1] + sh->p[1]")],
    "dilation_dropped": [(r"\(int64_t\)kw \* sh->d\[2\]", "(int64_t)kw")],
    "stride_wrong_dim": [(r"\(int64_t\)od \* sh->s\[0\]", "(int64_t)od * sh->s[1]")],
    "group_offset_dropped": [(r"\* sh->C \+ \(int64_t\)g \* Cg;", "* sh->C;")],
    "weight_taps_transposed": [(r"\(\(\(\(int64_t\)o \* sh->kD \+ fd\) \* sh->kH \+ fh\) \* sh->kW \+ fw\)",
                                "((((int64_t)o * sh->kD + fd) * sh->kW + fw) * sh->kH + fh)")],
    "flip_ignored_in_width": [(r"const int fw = sh->flip \? sh->kW - 1 - kw : kw;", "const int fw = kw;")],
    "high_side_padding_ignored": [(r"in \+ \(int64_t\)p_lo \+ \(int64_t\)p_hi", "in + 2 * (int64_t)p_lo")],
    "magnitude_signed": [(r"mag \+= fabs\(t\);", "mag += t;")],
    "extent_off_by_one": [(r"\(int64_t\)d \* \(k - 1\) - 1;", "(int64_t)d * (k - 1);")],
    "f16_exponent_bias": [(r"e - 25\);", "e - 24);")],
    "bf16_mantissa_width": [(r"\(double\)\(128 \+ m\), e - 134\)", "(double)(128 + m), e - 133)")],
    "transpose_stride_divisibility_dropped": [(r"if \(num < 0 \|\| num % s\) return -1;", "if (num < 0) return -1;")],
    "transpose_pad_sign": [(r"int64_t num = q \+ p - \(int64_t\)k \* d;", "int64_t num = q - p - (int64_t)k * d;")],
    "transpose_points_qw_qh_swapped": [(r"int qw = \(int\)\(q % t->Qw\); q /= t->Qw;\n    int qh = \(int\)\(q % t->Qh\); q /= t->Qh;",
                                        "int qh = (int)(q % t->Qh); q /= t->Qh;\n    int qw = (int)(q % t->Qw); q /= t->Qw;")],
    "transpose_out_channel_index": [(r"\* t->kW \+ kw\) \* Cog \+ cl;", "* t->kW + kw) * Cog + (Cog - 1 - cl);")],
    "wgrad_dy_channel_reversed": [(r"\* t->Wo \+ ow\) \* t->O \+ o\];", "* t->Wo + ow) * t->O + (t->O - 1 - o)];")],
    "wgrad_tap_sign": [(r"int64_t iw = \(int64_t\)ow \* t->s\[2\] - t->p\[2\] \+ \(int64_t\)kw \* t->d\[2\];",
                        "int64_t iw = (int64_t)ow * t->s[2] - t->p[2] - (int64_t)kw * t->d[2];")],
    "padding_not_zero": [(r"if \(ih < 0 \|\| ih >= sh->H\) continue;", "if (ih < 0 || ih >= sh->H) ih = ih < 0 ? 0 : sh->H - 1;")],
    "transpose_dilation_dropped": [(r"src_index\(qw, kw, t->s\[2\], t->p\[2\], t->d\[2\], t->W\)",
                                    "src_index(qw, kw, t->s[2], t->p[2], 1, t->W)")],
    "transpose_group_offset_dropped": [(r"\* t->Ci \+ \(int64_t\)g \* Cig;", "* t->Ci;")],
    "transpose_output_padding_ignored": [(r"\(int64_t\)d \* \(k - 1\) \+ 1 \+ op;", "(int64_t)d * (k - 1) + 1;")],
    "transpose_last_input_row_dropped": [(r"return num < in \? num : -1;", "return num < in - 1 ? num : -1;")],
    "transpose_magnitude_signed": [(r"mag \+= fabs\(v\);", "mag += v;")],
    "wgrad_dilation_dropped": [(r"\+ \(int64_t\)kh \* t->d\[1\];", "+ (int64_t)kh;")],
    "wgrad_stride_wrong_dim": [(r"\(int64_t\)oh \* t->s\[1\]", "(int64_t)oh * t->s[2]")],
    "wgrad_group_offset_dropped": [(r"\(int64_t\)g \* Cg \+ c\];", "c];")],
    "wgrad_magnitude_signed": [(r"mag \+= fabs\(gy \* xv\);", "mag += gy * xv;")],
    "wgrad_taps_transposed": [(r"int64_t q = \(\(\(\(int64_t\)o \* kD \+ kd\) \* t->kH \+ kh\) \* t->kW \+ kw\) \* Cg \+ c;",
                               "int64_t q = ((((int64_t)o * kD + kd) * t->kW + kw) * t->kH + kh) * Cg + c;")],
    "dilation_dropped_depth": [(r"\+ \(int64_t\)kd \* sh->d\[0\];", "+ (int64_t)kd;")],
    "stride_height_from_width": [(r"\(int64_t\)oh \* sh->s\[1\]", "(int64_t)oh * sh->s[2]")],
    "pad_depth_sign": [(r"\(int64_t\)od \* sh->s\[0\] - sh->p\[0\]", "(int64_t)od * sh->s[0] + sh->p[0]")],
    "extent_ceil": [(r"return num / s \+ 1;", "return (num + s - 1) / s + 1;")],
    "decoder_sign_dropped": [(r"return sign \? -v : v;", "return v;")],
    "f16_subnormal_scale": [(r"ldexp\(\(double\)m, -24\)", "ldexp((double)m, -25)")],
    "encoder_truncates": [(r"double r = rint\(a / q\);", "double r = floor(a / q);")],
    "encoder_subnormal_quantum_dropped": [(r"if \(E < emin\) E = emin;", "")],
    "encoder_overflow_late": [(r"if \(rv >= ldexp\(1\.0, emax \+ 1\)\)", "if (rv >= ldexp(1.0, emax + 2))")],
}


def _build_mutant(name, edits, tmp_path):
    src = open(_SRC).read()
    for pat, rep in edits:
        src2, n = re.subn(pat, rep, src)
        assert n >= 1, f"mutation {name}: pattern {pat!r} not found"
        src = src2
    c = tmp_path / f"{name}.c"
    c.write_text(src)
    so = tmp_path / f"lib{name}.so"
    subprocess.run(["gcc", "-O1", "-std=c11", "-fopenmp", "-fPIC", "-shared", str(c), "-o", str(so), "-lm"],
                   check=True)
    return oracle.Oracle(str(so))


def _codec_pins(orc):
    """The decoders over a stride of all bit patterns and the encoders on edge
    values, against NumPy (binary16) and torch (bfloat16)."""
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    f16 = np.array([orc.lib.oracle_f16_to_f64(int(b)) for b in bits[::7]])
    ref = bits[::7].view(np.float16).astype(np.float64)
    ok = np.isnan(ref)
    assert np.array_equal(f16[~ok], ref[~ok])
    bf = np.array([orc.lib.oracle_bf16_to_f64(int(b)) for b in bits[::7]])
    refb = torch.from_numpy(bits[::7].astype(np.int16)).view(torch.bfloat16).double().numpy()
    okb = np.isnan(refb)
    assert np.array_equal(bf[~okb], refb[~okb])
    v = _edge_values()
    e16 = np.array([orc.lib.oracle_f64_to_f16_rn(float(a)) for a in v], dtype=np.uint16)
    with np.errstate(over="ignore"):
        assert np.array_equal(e16, v.astype(np.float16).view(np.uint16))
    v32 = v.astype(np.float32)
    eb = np.array([orc.lib.oracle_f64_to_bf16_rn(float(a)) for a in v32.astype(np.float64)], dtype=np.uint16)
    assert np.array_equal(eb, torch.from_numpy(v32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, tmp_path):
    orc = _build_mutant(name, MUTATIONS[name], tmp_path)
    failed = []
    for pin in P.ALL_PINS + [_codec_pins]:
        try:
            pin(orc)
        except AssertionError:
            failed.append(pin.__name__)
        except ValueError:
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {name!r}"
