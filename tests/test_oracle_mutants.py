"""Plant plausible mistakes in a copy of the oracle source; each must trip a pin.

The mistakes are planted in a temporary copy of ``oracle/smla_oracle.c`` on the
CPU -- the oracle itself is never edited.  A mutant that passes every pin would
mean the pins leave that part of the oracle unchecked.
"""
import os
import subprocess

import pytest

import oracle
from tests import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "smla_oracle.c")

MUTANTS = {
    "e4m3_bias_off_by_one": ("ldexp(1.0 + (double)m / 8.0, e - 7)", "ldexp(1.0 + (double)m / 8.0, e - 8)"),
    "e4m3_no_subnormal": ("ldexp((double)m / 8.0, -6)", "ldexp(1.0 + (double)m / 8.0, -6)"),
    "ue8m0_bias": ("ldexp(1.0, (int)b - 127)", "ldexp(1.0, (int)b - 128)"),
    "scale_group_wrong": ("scales[d / ORC_GROUP]", "scales[d / 56]"),
    "interleaved_records": ("page_base + ORC_SCALE_BLOCK_OFFSET + (int64_t)slot * ORC_SCALE_ROW_BYTES",
                            "row + ORC_ROW_BYTES"),
    "rope_big_endian": ("(row[ORC_NOPE + 2 * r] | (row[ORC_NOPE + 2 * r + 1] << 8))",
                        "(row[ORC_NOPE + 2 * r + 1] | (row[ORC_NOPE + 2 * r] << 8))"),
    "rope_dropped": ("k[ORC_NOPE + r] = orc_bf16(u);", "k[ORC_NOPE + r] = 0.0 * orc_bf16(u);"),
    "slot_from_block": ("*slot = idx % ORC_PAGE_TOKENS;", "*slot = idx / ORC_PAGE_TOKENS;"),
    "no_seq_len_mask": ("if (idx < 0 || idx >= seq_len) return 0;", "if (idx < 0) return 0;"),
    "no_page_range_check": ("if (p < 0 || (int64_t)p >= num_pages) return 0;", "if (p < -1000) return 0;"),
    "sm_scale_dropped": ("s[j] = sm_scale * acc;", "s[j] = acc;"),
    "lse_without_max": ("*lse = M + log(l);", "*lse = log(l);"),
    "no_normalisation": ("for (d = 0; d < ORC_DIM; d++) o[d] /= l;", ";"),
    "v_is_nope_only": ("for (d = 0; d < ORC_DIM; d++) o[d] += w * K[(int64_t)j * ORC_DIM + d];",
                       "for (d = 0; d < ORC_NOPE; d++) o[d] += w * K[(int64_t)j * ORC_DIM + d];"),
    "q_head_index_swapped": ("qh[d] = orc_bf16(q[((int64_t)b * H + h) * ORC_DIM + d]);\n                orc_attend_one(qh, K, n, sm_scale, out + ((int64_t)b * H + h)",
                             "qh[d] = orc_bf16(q[((int64_t)b * H + (H - 1 - h)) * ORC_DIM + d]);\n                orc_attend_one(qh, K, n, sm_scale, out + ((int64_t)b * H + h)"),
    "combine_weights_unnormalised": ("for (d = 0; d < ORC_DIM; d++) o[d] /= W;", ";"),
    "combine_lse_plain_max": ("lse[bh] = Lmax + log(W);", "lse[bh] = Lmax;"),
    "encode_ties_to_odd": ("if (d < best_d || (d == best_d && (c & 1) == 0)) {", "if (d < best_d || (d == best_d && (c & 1) == 1)) {"),
    "encode_sign_dropped": ("uint8_t sign = signbit(x) ? 0x80 : 0x00;", "uint8_t sign = 0x00;"),
    "bf16_truncates": ("    if (dlo < dhi) return lo;", "    if (dlo < dhi + 1.0) return lo;"),
    "scale_exponent_floor": ("while (e < 127 && ldexp(448.0, e) < amax) e++;", "while (e < 127 && ldexp(448.0, e) <= amax) e++;"),
    "scale_byte_bias": ("scale_row[g] = (uint8_t)(e + 127);", "scale_row[g] = (uint8_t)(e + 128);"),
    "quantize_without_scale": ("row[d] = orc_e4m3_encode(ldexp((double)x[d], -e));", "row[d] = orc_e4m3_encode((double)x[d]);"),
    "writer_rope_big_endian": ("row[ORC_NOPE + 2 * r] = (uint8_t)(u & 0xFF);", "row[ORC_NOPE + 2 * r] = (uint8_t)(u >> 8);"),
    "writer_slot_from_block": ("page_base + (int64_t)(p % ORC_PAGE_TOKENS) * ORC_ROW_BYTES,", "page_base + (int64_t)(p / ORC_PAGE_TOKENS) * ORC_ROW_BYTES,"),
    "writer_no_page_check": ("        if (page < 0 || (int64_t)page >= num_pages) {\n            skipped++;", "        if (page < -1000) {\n            skipped++;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique/found"
    mutant = tmp_path / "mutant.c"
    mutant.write_text(src.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", str(mutant), "-o", str(so), "-lm"], check=True)
    lib = oracle.load_variant(str(so))
    failed = []
    for check in oracle_pins.ALL_CHECKS:
        try:
            check(lib)
        except AssertionError:
            failed.append(check.__name__)
    assert failed, f"mutant {name} passed every pin"
