"""Plant a plausible mistake in a copy of the oracle and require that the pins
catch it.  The mistakes are planted in the oracle source, on the CPU, in a
temporary directory; the real oracle is untouched."""
import os
import subprocess

import pytest

import oracle
import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "attn_oracle.c")

MUTANTS = {
    "window_left_off_by_one": ("if (left >= 0 && j < i - left) return 0;",
                               "if (left >= 0 && j <= i - left) return 0;"),
    "window_right_off_by_one": ("if (right >= 0 && j > i + right) return 0;",
                                "if (right >= 0 && j >= i + right) return 0;"),
    "causal_ignored": ("const int64_t right = causal ? 0 : window_right;",
                       "const int64_t right = window_right;"),
    "scale_dropped": ("s_row[j] = scale * dot;", "s_row[j] = dot;"),
    "normaliser_dropped": ("double p = exp(s_row[j] - M) / Z;", "double p = exp(s_row[j] - M);"),
    "lse_max_dropped": ("*lse_out = M + log(Z);", "*lse_out = log(Z);"),
    "exp_sign_flipped": ("double p = exp(s_row[j] - M) / Z;", "double p = exp(M - s_row[j]) / Z;"),
    "gqa_modulo_map": ("h / group", "h % Hkv"),
    "q_used_as_k": ("widen_bf16(qi[t]) * widen_bf16(kj[t])", "widen_bf16(qi[t]) * widen_bf16(qi[t])"),
    "v_ignores_sequence_start": ("const uint16_t *vj = v + ((start + j) * (int64_t)Hkv + g) * d;",
                                 "const uint16_t *vj = v + ((j) * (int64_t)Hkv + g) * d;"),
    "packed_lse_layout": ("(int64_t)h * tokens + start + i", "(int64_t)h * tokens + i"),
    "k_row_transposed": ("const uint16_t *kj = k + ((start + j) * (int64_t)Hkv + g) * d;",
                         "const uint16_t *kj = k + ((start + (i + j) % L) * (int64_t)Hkv + g) * d;"),
    "kvcache_top_left_alignment": ("const int64_t pos = L - Nq + i;", "const int64_t pos = i;"),
    "kvcache_block_table_ignored": ("                        const int64_t page = block_table\n                                                 ? block_table[(int64_t)b * pages_per_seq + j / page_size]",
                                    "                        const int64_t page = 0\n                                                 ? block_table[(int64_t)b * pages_per_seq + j / page_size]"),
    "kvcache_page_row_swapped": ("const int64_t row = page * page_size + j % page_size;\n                        const uint16_t *vj",
                                 "const int64_t row = page * page_size + (page_size - 1 - j % page_size);\n                        const uint16_t *vj"),
    "bwd_dq_scale_dropped": ("dqi[c] += scale * ds * widen_bf16(kj[c]);",
                             "dqi[c] += ds * widen_bf16(kj[c]);"),
    "bwd_D_not_subtracted": ("const double ds = exp(s_row[j] - lse_i) * (dp_row[j] - Di);",
                             "const double ds = exp(s_row[j] - lse_i) * dp_row[j];"),
    "bwd_dk_uses_k": ("dkj[c] += scale * ds * widen_bf16(qi[c]);",
                      "dkj[c] += scale * ds * widen_bf16(kj[c]);"),
    "bwd_dv_weight_dropped": ("dvj[c] += p * widen_bf16(doi[c]);", "dvj[c] += widen_bf16(doi[c]);"),
    "bwd_group_sum_one_head": ("for (int hh = 0; hh < group; ++hh) {",
                               "for (int hh = 0; hh < 1; ++hh) {"),
    "bwd_key_mask_transposed": ("                    if (!key_visible(i, j, left, right)) continue;\n                    const int64_t r",
                                "                    if (!key_visible(j, i, left, right)) continue;\n                    const int64_t r"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(tmp_path, name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert old in src, f"mutation anchor for {name} not found"
    mutated = src.replace(old, new)
    path = tmp_path / "attn_oracle_mutant.c"
    path.write_text(mutated)
    so = str(tmp_path / "liboracle_mutant.so")
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", so, str(path), "-lm"],
                   check=True)
    lib = oracle.load(so)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(lib)
        except AssertionError:
            caught.append(pin.__name__)
        except ValueError:
            caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake {name}"
