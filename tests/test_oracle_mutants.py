"""Plant plausible mistakes in copies of the oracle and check that the pins catch each.

Every mutant is a textual edit of ``oracle/fpd_oracle.c`` compiled into a
temporary library (CPU only); the shipped oracle is untouched.  A mutant that
passes every pin would mean the pins leave that part of the oracle unchecked.
"""
import os
import tempfile

import pytest

import oracle
from tests import oracle_pins as P

SRC = os.path.join(os.path.dirname(oracle.__file__), "fpd_oracle.c")

MUTANTS = {
    "sink dropped from denominator": [("    Z += exp(sigma - m);\n", "")],
    "GQA head mapping h % Hkv": [("const int kvh = h / g;", "const int kvh = h % J->Hkv;")],
    "window start off by one": [("p - J->window_left", "p + 1 - J->window_left")],
    "queries not causal (all see the whole sequence)": [("p = L - Q + i;", "p = L - 1;")],
    "query positions reversed": [("p = L - Q + i;", "p = L - 1 - i;")],
    "E4M3 exponent bias 8": [("expo - 7", "expo - 8")],
    "E4M3 subnormal exponent": [("(double)mant / 8.0, -6)", "(double)mant / 8.0, -7)")],
    "E4M3 mantissa step": [("1.0 + (double)mant / 8.0", "1.0 + (double)mant / 16.0")],
    "E4M3 sign ignored": [("return sign ? -mag : mag;", "return mag;")],
    "cache read head-major (transposed operand)": [
        ("return page_row(J->kv_hnd, page", "return page_row(!J->kv_hnd, page")],
    "HND pages addressed token-major": [
        ("        return (((size_t)page * Hkv + kvh) * bt + slot) * (size_t)D;\n",
         "        return (((size_t)page * bt + slot) * Hkv + kvh) * (size_t)D;\n")],
    "fp16 exponent bias 16": [("(1.0 + (double)m / 1024.0, e - 15)",
                               "(1.0 + (double)m / 1024.0, e - 16)")],
    "fp16 subnormal scale": [("ldexp((double)m / 1024.0, -14)", "ldexp((double)m / 1024.0, -15)")],
    "NVFP4 nibble order swapped": [
        ("(d & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF)",
         "(d & 1) ? (uint8_t)(byte & 0xF) : (uint8_t)(byte >> 4)")],
    "NVFP4 scale of the neighbouring block": [("row * (J->D / 16) + d / 16]",
                                               "row * (J->D / 16) + ((d / 16) ^ 1)]")],
    "E2M1 subnormal value": [("e == 0 ? 0.5 * m :", "e == 0 ? 0.25 * m :")],
    "E2M1 exponent bias 2": [("ldexp(1.0 + 0.5 * m, e - 1)", "ldexp(1.0 + 0.5 * m, e - 2)")],
    "NVFP4 writer amax / 8": [("sf_f = (amax * (1.0f / 6.0f)) * gs;", "sf_f = (amax * (1.0f / 8.0f)) * gs;")],
    "NVFP4 writer ignores the block scale": [
        ("osc = sf_v == 0.0f ? 0.0f : 1.0f / (sf_v * (1.0f / gs));", "osc = sf_v == 0.0f ? 0.0f : gs;")],
    "NVFP4 writer nibbles swapped": [("(uint8_t)(codes[2 * i] | (codes[2 * i + 1] << 4))",
                                      "(uint8_t)(codes[2 * i + 1] | (codes[2 * i] << 4))")],
    "fp16 query decoded as bf16": [("return J->q_f16 ? fpd_oracle_f16_to_f64(bits) :",
                                    "return 0 ? fpd_oracle_f16_to_f64(bits) :")],
    "in-page slot reversed": [("j % J->bt, kvh)", "J->bt - 1 - j % J->bt, kvh)")],
    "block table ignored": [
        ("const int page = J->block_table[(size_t)b * J->max_blocks + j / J->bt];",
         "const int page = (int)((size_t)b * J->max_blocks + j / J->bt) % J->num_blocks;")],
    "wrong query row": [("const uint16_t *qr = J->q + (size_t)row * D;",
                         "const uint16_t *qr = J->q + (size_t)(b * J->Hq + kvh) * D;")],
    "lse without sink": [("J->lse[row] = m + log(Z);",
                          "J->lse[row] = m + log(Z - exp(sigma - m));")],
    "sink multiplied by sm_scale": [("(double)J->sinks[h] : -INFINITY",
                                     "J->sm_scale * (double)J->sinks[h] : -INFINITY")],
    "v_scale dropped": [("(J->v_scale * fpd_oracle_e4m3_to_f64(vr[d]))",
                         "fpd_oracle_e4m3_to_f64(vr[d])")],
    "k_scale dropped": [("(J->k_scale * fpd_oracle_e4m3_to_f64(kr[d]))",
                         "fpd_oracle_e4m3_to_f64(kr[d])")],
    "sm_scale dropped": [("s[j - start] = J->sm_scale * dot;", "s[j - start] = dot;")],
    "bf16 decode shift": [("(uint32_t)bits << 16", "(uint32_t)bits << 15")],
    "max not subtracted consistently": [("const double p = exp(s[j - start] - m);",
                                         "const double p = exp(s[j - start]);")],
    "encoder ties away from zero": [("(d == best_d && (c & 1) == 0 && (best & 1) == 1)",
                                     "(d == best_d)")],
    "encoder does not saturate infinities": [("    if (a >= 448.0)\n        return (uint8_t)(sign | 0x7E);\n", "")],
    "encoder drops the sign": [("return (uint8_t)(sign | best);", "return (uint8_t)best;")],
    "writer divides instead of the fp32 reciprocal product": [
        ("const float yk = xk * kr, yv = xv * vr;", "const float yk = xk * kr * 1.0000001f, yv = xv * vr;")],
    "writer skips slot 0 too": [("        if (slot < 0)\n            continue;\n", "        if (slot <= 0)\n            continue;\n")],
    "writer swaps K and V scales": [("const float kr = 1.0f / k_scale, vr = 1.0f / v_scale;",
                                     "const float kr = 1.0f / v_scale, vr = 1.0f / k_scale;")],
    "writer cache head-major (transposed operand)": [
        ("page_row(hnd, (int)(slot / bt)", "page_row(!hnd, (int)(slot / bt)")],
    "writer value read with the key stride": [("value[t * value_stride + (long)h * D + d]",
                                               "value[t * key_stride + (long)h * D + d]")],
    "merge drops the sink": [("        Z += exp(sigma - M);\n        for (d = 0; d < D; ++d)\n            o[d] /= Z;",
                              "        for (d = 0; d < D; ++d)\n            o[d] /= Z;")],
    "merge weights parts equally": [("const double w = l == -INFINITY ? 0.0 : exp(l - M);",
                                     "const double w = l == -INFINITY ? 0.0 : 1.0;")],
    "merge lse without the maximum": [("lse[row] = M + log(Z);", "lse[row] = log(Z);")],
    "merge sink of the wrong head": [("(double)sinks[row % Hq]", "(double)sinks[(row + 1) % Hq]")],
    "last key dropped": [("for (j = start; j < end; ++j) {\n        const int page = J->block_table"
                          "[(size_t)b * J->max_blocks + j / J->bt];\n        const uint8_t *vr",
                          "for (j = start; j < end - 1; ++j) {\n        const int page = J->block_table"
                          "[(size_t)b * J->max_blocks + j / J->bt];\n        const uint8_t *vr")],
}


@pytest.fixture(scope="module")
def source():
    with open(SRC) as f:
        return f.read()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(source, name, tmp_path):
    text = source
    for old, new in MUTANTS[name]:
        assert old in text, f"mutation site missing: {old!r}"
        text = text.replace(old, new)
    src = tmp_path / "mutant.c"
    src.write_text(text)
    so = tmp_path / "libmutant.so"
    oracle.build(str(src), str(so))
    lib = oracle.load(str(so))
    caught = []
    for pin in P.ALL_PINS:
        try:
            pin(lib)
        except (AssertionError, ValueError) as e:
            caught.append(f"{pin.__name__}: {str(e)[:80]}")
    assert caught, f"no pin catches mutant '{name}'"
