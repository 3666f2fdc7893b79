"""Plant plausible mistakes in a copy of the oracle and check that the pins
catch every one of them (CPU only; the oracle package itself is untouched)."""

import importlib.util
import os
import types

import pytest

from tests import oracle_pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "oracle", "indexer_oracle.py")

MUTATIONS = {
    "relu_dropped": ("relu = np.maximum(dots, 0.0)", "relu = dots"),
    "weight_sign": ("s = relu @ w_t", "s = relu @ (-w_t)"),
    "heads_reversed": ("dots = keys @ q_t.T", "dots = keys @ q_t[::-1].T"),
    "tie_to_higher_index": ("order = np.argsort(-s, kind=\"stable\")",
                            "order = (s.size - 1) - np.argsort(-s[::-1], kind=\"stable\")"),
    "budget_off_by_one": ("take = order[: min(ksel, n)]", "take = order[: max(min(ksel, n) - 1, 0)]"),
    "token_strict_causal": ("mask = j <= g", "mask = j < g"),
    "pool_first_token_rule": ("mask = ratio * j + ratio - 1 <= g", "mask = ratio * j <= g"),
    "tail_dropped": ("    if last <= g:\n        return np.zeros(0, dtype=np.int64)",
                     "    if True:\n        return np.zeros(0, dtype=np.int64)"),
    "e4m3_bias": ("2.0 ** (e - 7)", "2.0 ** (e - 8)"),
    "pool_coef_transposed": ("prods = kk * c[None, :, :]", "prods = kk * c[None, ::-1, :]"),
    "bf16_truncates": ("np.rint(np.ldexp(f, 8))", "np.trunc(np.ldexp(f, 8))"),
    "overlap_counts_union": ("np.count_nonzero(both[1:] == both[:-1])",
                             "np.count_nonzero(both[1:] != both[:-1])"),
    "fp8_key_scale_ignored": ("return decode_e4m3(k) * np.asarray(k_scale, dtype=np.float64)[:, None]",
                              "return decode_e4m3(k)"),
    "tail_before_pools": ("pos = np.concatenate([pos, tail])", "pos = np.concatenate([tail, pos])"),
    "regions_left_right_swapped": ("for r, members in enumerate((a & b, a - b, b - a)):",
                                   "for r, members in enumerate((a & b, b - a, a - b)):"),
    "document_start_leaks": ("            vis = np.arange(b, g + 1, dtype=np.int64)",
                             "            vis = np.arange(max(b - 1, 0), g + 1, dtype=np.int64)"),
    "pools_from_global_grid": ("            pos = (b + sel[:, None] * ratio + np.arange(ratio)[None, :]).reshape(-1)",
                               "            pos = (b // ratio * ratio + sel[:, None] * ratio + np.arange(ratio)[None, :]).reshape(-1)"),
    "regions_unsorted": ("            ordered = sorted(members)", "            ordered = sorted(members, reverse=True)"),
    "witness_counts_repeats": ("        if r >= n_vis or r <= top:", "        if r >= n_vis:"),
    "witness_counts_invisible": ("        if r >= n_vis or r <= top:", "        if r <= top:"),
    "fraction_ties_to_odd": ("rem == Fraction(1, 2) and n % 2 == 1", "rem == Fraction(1, 2) and n % 2 == 0"),
    "fraction_fallback_dropped": ("        out[p, dd] = _round_fraction_to_bf16_bits(exact)",
                                  "        out[p, dd] = out[p, dd]"),
    "fraction_subnormal_spacing": ("quantum = Fraction(2) ** (max(e, -126) - 7)", "quantum = Fraction(2) ** (e - 7)"),
    "compressed_doc_start_exclusive": ("vis = j[(j >= b // ratio) & (ratio * j + ratio - 1 <= g)]",
                                       "vis = j[(j > b // ratio) & (ratio * j + ratio - 1 <= g)]"),
    "compressed_doc_start_ignored": ("vis = j[(j >= b // ratio) & (ratio * j + ratio - 1 <= g)]",
                                     "vis = j[(ratio * j + ratio - 1 <= g)]"),
    "padding_rows_select": ("            continue                                  # a padding query row",
                            "            pass"),
    "padded_pools_on_global_grid": ("            pos = (start + sel[:, None] * ratio + np.arange(ratio)[None, :]).reshape(-1)",
                                    "            pos = (start // 8 * 8 + sel[:, None] * ratio + np.arange(ratio)[None, :]).reshape(-1)"),
    "witness_kth_off_by_one": ("taus[r] = float(np.sort(s)[::-1][ksel - 1])", "taus[r] = float(np.sort(s)[::-1][ksel - 2])"),
}


def _mutant(old, new):
    with open(SRC) as f:
        src = f.read()
    assert src.count(old) == 1, f"mutation anchor not found once: {old!r}"
    mod = types.ModuleType("oracle_mutant")
    exec(compile(src.replace(old, new), "oracle_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(name):
    mod = _mutant(*MUTATIONS[name])
    failed = []
    for pin in oracle_pins.PINS:
        try:
            pin(mod)
        except AssertionError:
            failed.append(pin.__name__)
        except Exception as e:  # a crash also counts as caught
            failed.append(f"{pin.__name__}:{type(e).__name__}")
    assert failed, f"no pin caught mutation {name}"
