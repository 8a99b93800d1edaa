"""The C oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of ``oracle/c/moe_ref.c`` (a text edit,
compiled with gcc into a temporary library), routes the C oracle's calls to
that library and checks that at least one pin of ``test_oracle_c.py`` fails.
The cross-checks against the numpy oracle are left out, so each mistake is
caught by a pin of its own.  Every edit keeps all accesses inside their arrays.
CPU only (needs gcc).
"""
import os
import subprocess

import pytest

import oracle.cref as cr
import tests.test_oracle_c as P

MUTATIONS = {  # name: (text in the source, replacement)
    "nibble order swapped": ("int nib = (c & 1) ? (byte >> 4) : (byte & 0xf);",
                             "int nib = (c & 1) ? (byte & 0xf) : (byte >> 4);"),
    "nibble read unsigned": ("return nib >= 8 ? nib - 16 : nib;", "return nib;"),
    "nibble read offset-8": ("return nib >= 8 ? nib - 16 : nib;", "return nib - 8;"),
    "int8 read unsigned": ("return (int)(int8_t)row[c];", "return (int)row[c];"),
    "scales interleaved": ("+ c / group]", "+ c % (K / group)]"),
    "fp16 exponent bias": ("ldexp((double)(0x400 | fr), ex - 25)", "ldexp((double)(0x400 | fr), ex - 24)"),
    "bf16 hidden bit dropped": ("ldexp((double)(0x80 | fr), ex - 134)", "ldexp((double)fr, ex - 134)"),
    "bf16 ties away from zero": ("if (low > half || (low == half && (keep & 1)))", "if (low >= half)"),
    "bf16 truncation": ("if (low > half || (low == half && (keep & 1)))", "if (0)"),
    "bf16 subnormal ties up": ("if (fr > 0.5 || (fr == 0.5 && fmod(fl, 2.0) != 0.0))", "if (fr >= 0.5)"),
    "router W_r transposed": ("wr[(size_t)e * H + h]", "wr[(size_t)h * E + e]"),
    "bias ignored": ("l = l + bias[e];", "l = l + 0.0f;"),
    "ties to the highest index": ("key[e] > key[best]", "key[e] >= key[best]"),
    "NaN not ranked last": ("key[e] = isnan(l) ? -INFINITY : (double)l;", "key[e] = (double)l;"),
    "weights not renormalised": ("w[(size_t)t * k + j] = exp(sel[j] - sel[0]) / sum;",
                                 "w[(size_t)t * k + j] = exp(sel[j] - sel[0]);"),
    "union not stable": ("for (int p = 0; p < P; ++p) {\n        int at = start[flat[p]]++;",
                         "for (int p = P - 1; p >= 0; --p) {\n        int at = start[flat[p]]++;"),
    "silu sign": ("return g / (1.0 + exp(-g));", "return g / (1.0 + exp(g));"),
    "gate and up swapped": ("hbuf[i] = round_bf16(silu(g) * u);", "hbuf[i] = round_bf16(silu(u) * g);"),
    "h not rounded": ("hbuf[i] = round_bf16(silu(g) * u);", "hbuf[i] = silu(g) * u;"),
    "h reversed in the down sum": ("weight_at(dq, ds, I, G, B, r, i) * hbuf[i]",
                                   "weight_at(dq, ds, I, G, B, r, i) * hbuf[I - 1 - i]"),
    "routing weight ignored": ("acc[(size_t)t * H + c] += w[(size_t)t * k + j] * y[c];",
                               "acc[(size_t)t * H + c] += y[c];"),
    "shared experts dropped": ("for (int s = 0; s < S; ++s) {", "for (int s = 0; s < 0; ++s) {"),
    "residual dropped": ("if (residual)\n", "if (0)\n"),
    "rms without sqrt": ("1.0 / sqrt(ss / H + 1e-6)", "1.0 / (ss / H + 1e-6)"),
}


def _pins():
    """The C oracle's pins, cheapest first; parametrised ones at fixed arguments."""
    plain = [getattr(P, n) for n in dir(P) if n.startswith("test_") and "agree" not in n and n not in (
        "test_dequant_group_index_and_rows", "test_batch_union_brute_force_and_inverse",
        "test_dense_identity_one_expert", "test_route_matches_brute_force_on_tie_dense_logits")]
    fixed = [lambda g=g, b=b: P.test_dequant_group_index_and_rows(g, b) for g, b in ((32, 4), (64, 4), (32, 8), (64, 8))]
    fixed += [lambda a=a: P.test_batch_union_brute_force_and_inverse(*a) for a in ((4, 16, 2), (33, 40, 3), (64, 256, 8))]
    fixed += [lambda b=b: P.test_dense_identity_one_expert(b) for b in (4, 8)]
    return plain + fixed + [P.test_route_matches_brute_force_on_tie_dense_logits]


def _build(tmp_path, text: str) -> str:
    src, lib = os.path.join(tmp_path, "moe_ref.c"), os.path.join(tmp_path, "libmutant.so")
    with open(src, "w") as f:
        f.write(text)
    r = subprocess.run([cr.CC, *cr.CFLAGS, src, "-o", lib, "-lm"], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return lib


def _first_failure(lib):
    with cr.using(lib):
        for pin in _pins():
            try:
                pin()
            except Exception as e:  # noqa: BLE001 - any failure counts as caught
                return f"{getattr(pin, '__name__', pin)}: {type(e).__name__}"
    return None


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(name, tmp_path):
    with open(cr.SRC) as f:
        text = f.read()
    old, new = MUTATIONS[name]
    assert text.count(old) == 1, f"mutation site not unique or missing: {old!r}"
    assert _first_failure(_build(str(tmp_path), text.replace(old, new))) is not None, f"no pin caught: {name}"


def test_pins_pass_unmutated(tmp_path):
    with open(cr.SRC) as f:
        assert _first_failure(_build(str(tmp_path), f.read())) is None
