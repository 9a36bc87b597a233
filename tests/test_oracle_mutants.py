"""The pins have teeth: each plausible mistake planted in a copy of the oracle
source (a dropped term, a wrong sign or index, an off-by-one mask, a swapped
operand) must fail at least one pin.  The mistakes are planted on the CPU, in a
temporary copy; the real oracle source is never modified."""
import os

import pytest

import oracle
from oracle.build import SOURCE, build_oracle
from oracle_pins import PINS

# (name, text in mea_oracle.c, replacement, which occurrence (0-based))
MUTANTS = [
    ("causal_off_by_one", "if (causal && pos_j > pos_i)", "if (causal && pos_j >= pos_i)", 0),
    ("top_left_causal", "int64_t pos_i = i + (N - M);", "int64_t pos_i = i;", 0),
    ("gqa_modulo_map", "const int kvh = h / group;", "const int kvh = h % Hkv;", 0),
    ("alibi_sign", "if (slopes) s -= slopes[h] * fabs", "if (slopes) s += slopes[h] * fabs", 0),
    ("alibi_slope_exponent", "-8.0 * (double)(h + 1)", "-8.0 * (double)h", 0),
    ("scale_dropped", "double s = scale * dot;", "double s = dot;", 0),
    ("lse_without_max", "*lse_row = mx + log(z);", "*lse_row = log(z);", 0),
    ("unnormalised", "const double w = score[j] / z;", "const double w = score[j];", 0),
    ("value_from_key", "const double* vj = v + ((b * N + j)", "const double* vj = k + ((b * N + j)", 0),
    ("query_head_as_kv_head", "(b * M + i) * Hq + h) * D;", "(b * M + i) * Hq + kvh) * D;", 0),
    ("blockdiag_keys_from_query_offsets", "j_lo = seqstart_k[s];", "j_lo = seqstart_q[s];", 0),
    ("blockdiag_global_position", "i_loc = i - seqstart_q[s];", "i_loc = i;", 0),
    ("blockdiag_no_causal_shift", "pos_i = i_loc + (n_len - m_len);", "pos_i = i_loc;", 0),
    ("decode_alibi_position", "(double)(n - 1 - j)", "(double)(n - j)", 0),
    ("decode_scale_dropped", "double s = scale * dot;", "double s = dot;", 1),
    ("decode_gqa_modulo", "kvh = h / group;", "kvh = h % Hkv;", 1),
    ("decode_lse_without_max", "lse[r] = mx + log(z);", "lse[r] = log(z);", 0),
    ("decode_value_from_key", "const double* vj = v_cache +", "const double* vj = k_cache +", 0),
    ("bwd_without_row_term", "const double ds = p[j] * (dp[j] - Di);",
     "const double ds = p[j] * dp[j];", 0),
    ("bwd_dk_from_key", "dkj[d] += scale * ds * qi[d];", "dkj[d] += scale * ds * kj[d];", 0),
    ("bwd_dq_unscaled", "dqi[d] += scale * ds * kj[d];", "dqi[d] += ds * kj[d];", 0),
    ("bwd_dv_from_dp", "dvj[d] += p[j] * doi[d];", "dvj[d] += dp[j] * doi[d];", 0),
    ("bwd_unnormalised", "p[j] /= z;", "p[j] /= 1.0;", 0),
    ("block_sparse_mask_ignored", "if (keep && !keep[j / block_n]) visible = 0;", "", 0),
    ("block_sparse_row_block_from_key_size", "+ i / block_m) * nblocks", "+ i / block_n) * nblocks", 0),
    ("block_sparse_head_ignored", "(((b * Hq + h) * mblocks)", "(((b * Hq) * mblocks)", 0),
    ("chunk_append_at_start", "(b * (int64_t)cap + past + r)", "(b * (int64_t)cap + r)", 0),
    ("chunk_causal_without_past", "if (causal && j > pos_i)", "if (causal && j > i)", 0),
    ("chunk_alibi_without_past", "fabs((double)(pos_i - j))", "fabs((double)(i - j))", 0),
    ("chunk_new_keys_missing", "total = past + n, pos_i", "total = past, pos_i", 0),
    ("chunk_value_from_key", "const double* vj = v_cache +", "const double* vj = k_cache +", 1),
    ("block_sparse_key_block_size_wrong", "!keep[j / block_n]", "!keep[j / (block_n + 1)]", 0),
]


def _plant(src: str, old: str, new: str, which: int) -> str:
    pos = -1
    for _ in range(which + 1):
        pos = src.find(old, pos + 1)
        assert pos >= 0, f"mutation site not found: {old!r} #{which}"
    return src[:pos] + new + src[pos + len(old):]


@pytest.mark.parametrize("name,old,new,which", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new, which):
    src = open(SOURCE).read()
    mutated = _plant(src, old, new, which)
    assert mutated != src
    path = tmp_path / f"{name}.c"
    path.write_text(mutated)
    lib = build_oracle(src=str(path), out=str(tmp_path / f"lib{name}.so"))
    orc = oracle.Oracle(lib)
    caught = []
    for pin in PINS:
        try:
            pin(orc)
        except (AssertionError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"planted mistake {name} passed every pin"
