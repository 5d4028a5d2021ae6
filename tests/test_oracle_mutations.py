"""Plant plausible mistakes in a copy of the oracle (on the CPU) and check the pins catch each.

Each mutation rewrites one expression of oracle/attention.py: a dropped term, a wrong sign,
a wrong index or head mapping, a swapped operand, an off-by-one in a row's key limit or in
the causal limit. The
mutated source is executed as a throw-away module; at least one pin must then fail.
"""

import math
import os
import types

import pytest

from oracle_pins import ALL_PINS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
with open(os.path.join(ROOT, "oracle", "attention.py")) as _f:
    SRC = _f.read()

MUTATIONS = {
    "scale_dropped_sqrt": ("scale = 1.0 / math.sqrt(D)", "scale = 1.0 / D"),
    "lse_drops_max": ("lse[has] = m + np.log(z)", "lse[has] = np.log(z)"),
    "lse_wrong_sign": ("lse[has] = m + np.log(z)", "lse[has] = m - np.log(z)"),
    "no_normalisation": ("out[has] = (e @ values[:N]) / z[:, None]", "out[has] = (e @ values[:N])"),
    "exp_wrong_sign": ("e = np.exp(s[has] - m[:, None])", "e = np.exp(m[:, None] - s[has])"),
    "k_v_swapped": ("s = (q_rows @ keys[:N].T) * scale", "s = (q_rows @ values[:N].T) * scale"),
    "gqa_mod_mapping": ("groups.setdefault((int(b), int(h) // G), []).append(int(h))",
                        "groups.setdefault((int(b), int(h) % Hkv), []).append(int(h))"),
    "ignores_cache_len": ("n = _clamp_len(cache_lens[b], S_cap)", "n = S_cap"),
    "len_off_by_one": ("n = _clamp_len(cache_lens[b], S_cap)",
                       "n = _clamp_len(cache_lens[b] - 1, S_cap)"),
    "row_mask_off_by_one": ("s[np.arange(N)[None, :] >= n_vis[:, None]] = -np.inf",
                            "s[np.arange(N)[None, :] > n_vis[:, None]] = -np.inf"),
    "causal_off_by_one": ("_clamp_len(int(prefix_lens[b]) + int(row_pos[p]) + 1, S_cap)",
                          "_clamp_len(int(prefix_lens[b]) + int(row_pos[p]), S_cap)"),
    "causal_top_left": ("_clamp_len(int(prefix_lens[b]) + int(row_pos[p]) + 1, S_cap)",
                        "_clamp_len(int(row_pos[p]) + 1, S_cap)"),
    "bf16_widen_shift": ("<< np.uint32(16)", "<< np.uint32(15)"),
    "empty_lse_zero": ("lse = np.full((R,), -np.inf, dtype=np.float64)",
                       "lse = np.full((R,), 0.0, dtype=np.float64)"),
    "page_index_mod": ("pg = int(block_table[b][t0 // psz])", "pg = int(block_table[b][t0 % psz])"),
    "paged_k_from_v": ("kc = gather_pages(k_pages, block_table, cache_lens, cap)",
                       "kc = gather_pages(v_pages, block_table, cache_lens, cap)"),
    "page_physical_order": ("pg = int(block_table[b][t0 // psz])", "pg = t0 // psz + b"),
    "e4m3_bias_8": ("return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)",
                    "return s * (1.0 + m / 8.0) * 2.0 ** (e - 8)"),
    "e4m3_subnormal_as_normal": ("if e == 0:\n        return s * (m / 8.0) * 2.0 ** (1 - 7)",
                                 "if e == 0:\n        return s * (1.0 + m / 8.0) * 2.0 ** (0 - 7)"),
    "e4m3_mantissa_16ths": ("return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)",
                            "return s * (1.0 + m / 16.0) * 2.0 ** (e - 7)"),
    "e4m3_sign_dropped": ("s = -1.0 if code & 0x80 else 1.0", "s = 1.0"),
    "fp8_v_scale_dropped": ("vc = DequantView(v_codes, v_scale)", "vc = DequantView(v_codes, 1.0)"),
    "fp8_scales_swapped": ("kc = DequantView(k_codes, k_scale)", "kc = DequantView(k_codes, v_scale)"),
    "fp8_paged_v_scale_for_k": ("kp = DequantView(k_pages, k_scale)",
                                "kp = DequantView(k_pages, v_scale)"),
    "fp8_view_drops_scale": ("return dequant_e4m3(self.codes[idx], self.scale)",
                             "return dequant_e4m3(self.codes[idx], 1.0)"),
}


def _mutant(name):
    old, new = MUTATIONS[name]
    assert SRC.count(old) >= 1, f"mutation anchor for {name} missing"
    mod = types.ModuleType(f"oracle_mutant_{name}")
    exec(compile(SRC.replace(old, new), f"<mutant {name}>", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(name):
    mod = _mutant(name)
    failed = []
    for pin in ALL_PINS:
        try:
            pin(mod)
        except (AssertionError, ValueError, IndexError, FloatingPointError, OverflowError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught mutation {name}"
