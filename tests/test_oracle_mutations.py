"""Planted mistakes in the oracle must be caught by its pins.

Each case edits one line of an oracle function's source (a dropped term, a
wrong index, a wrong rounding, a wrong list end), installs the edited
function in place of the real one for the duration of the test, and runs
the pin that should notice.  The pin must fail.
"""
import inspect
import textwrap

import numpy as np
import pytest

import oracle
from oracle import fp8, numerics, paged, sizing

import test_oracle_attention as att
import test_oracle_fp8 as tf8
import test_oracle_numerics as tnum
import test_oracle_pool as pool
import test_oracle_prefix as pfx
import test_oracle_swap as swp
import test_oracle_sizing as tsz


def _mutated(func, old, new):
    src = textwrap.dedent(inspect.getsource(func))
    assert src.count(old) == 1, f"mutation anchor not unique in {func.__name__}: {old!r}"
    src = src.replace(old, new)
    ns = dict(func.__globals__)
    exec(compile(src, f"<mutant {func.__name__}>", "exec"), ns)
    return ns[func.__name__]


MUTANTS = [
    # (target object, attribute, old text, new text, pin to run)
    (fp8, "encode_f32", "np.rint(", "np.floor(",
     lambda: tf8.test_encode_brute_force_random_fp32()),
    (fp8, "encode_f32", "e = np.maximum(ex - 1, -6)", "e = np.maximum(ex - 1, -7)",
     lambda: tf8.test_encode_matches_brute_force_all_bf16()),
    (fp8, "decode", "(8 + m) * np.exp2(e.astype(np.float64) - 10.0)", "(8 + m) * np.exp2(e.astype(np.float64) - 9.0)",
     lambda: tf8.test_code_values_from_definition()),
    (sizing, "kv_bytes_per_token", "return 2 * layers", "return layers",
     None),
    (sizing, "pool_blocks", "budget_bytes // (bytes_per_token * block_size)",
     "budget_bytes // bytes_per_token // block_size + 1", None),
    (paged.PagedKVOracle, "attention", "h = qh // group", "h = qh % self.H",
     lambda: att.test_matches_scalar_brute_force(2)),
    (paged.PagedKVOracle, "attention", "x = (kh @ q[i, qh]) * sc", "x = (kh @ q[i, qh])",
     lambda: att.test_matches_scalar_brute_force(1)),
    (paged.PagedKVOracle, "attention", "kh, vh = K[:, h, :], V[:, h, :]", "kh, vh = K[:, h, :], K[:, h, :]",
     lambda: att.test_matches_torch_sdpa_float64()),
    (paged.PagedKVOracle, "attention", "vh = vh * float(v_scale[layer][h])", "vh = vh * float(k_scale[layer][h])",
     lambda: att.test_fp8_matches_scalar_brute_force()),
    (paged.PagedKVOracle, "gather", "blocks = np.asarray(self.tables[seq], dtype=np.int64)[t // self.B]",
     "blocks = np.asarray(self.tables[seq], dtype=np.int64)[t % len(self.tables[seq])]",
     lambda: att.test_matches_scalar_brute_force(1)),
    (paged.PagedKVOracle, "reserve", "cow = new_len > cur and cur % self.B != 0 and self.ref[table[-1]] > 1",
     "cow = False", lambda: pool.test_parallel_sampling_cow_seven_copies_one_in_place()),
    (paged.PagedKVOracle, "reserve", "if int(cow) + grow > len(self.free) + len(self.cached):",
     "if grow > len(self.free) + len(self.cached):",
     lambda: pool.test_cow_and_growth_need_is_checked_before_any_change()),
    (paged.PagedKVOracle, "release", "self.free.append(b)", "self.free.appendleft(b)",
     lambda: pool.test_release_returns_blocks_in_logical_order_once_unreferenced()),
    (paged.PagedKVOracle, "slot", "if self.ref[b] > 1 or", "if self.ref[b] > 2 or",
     lambda: pool.test_invalid_calls()),
    (paged.PagedKVOracle, "append", "self.k[layer][b, :, o, :] = k_bits[t]", "self.k[layer][b, :, o - 1, :] = k_bits[t]",
     lambda: pool.test_append_writes_the_slot_and_nothing_else()),
    # fp16 storage widened as if it were bf16 (caught by the definition and by
    # the fp16 brute force, which decodes with the struct binary16 codec)
    (numerics, "bits_to_f64", "return b.view(np.float16).astype(np.float64)",
     "return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)",
     lambda: tnum.test_fp16_values_from_definition()),
    (numerics, "bits_to_f64", "return b.view(np.float16).astype(np.float64)",
     "return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)",
     lambda: att.test_fp16_matches_scalar_brute_force(4)),
    (numerics, "bits_to_f64", "return b.view(np.float16).astype(np.float64)",
     "return b.view(np.float16).astype(np.float32).astype(np.float64) * (1 + 2.0 ** -11)",
     lambda: tnum.test_named_fp16_values()),
    # block-granular prefix cache
    (paged.PagedKVOracle, "_prefix", "tokens[: (i + 1) * self.B]", "tokens[i * self.B : (i + 1) * self.B]",
     lambda: pfx.test_conversations_under_pool_pressure_keep_exact_contents(0)),
    (paged.PagedKVOracle, "_take", "popitem(last=False)", "popitem(last=True)",
     lambda: pfx.test_lru_trace_by_hand()),
    (paged.PagedKVOracle, "_take", "del self.registry[self.key_of.pop(b)]", "self.key_of.pop(b)",
     lambda: pfx.test_conversations_under_pool_pressure_keep_exact_contents(0)),
    (paged.PagedKVOracle, "release", "for b in reversed(self.tables[seq]):", "for b in self.tables[seq]:",
     lambda: pfx.test_lru_trace_by_hand()),
    (paged.PagedKVOracle, "release", "if self.ref[b] == 0 and b not in self.key_of:", "if self.ref[b] == 0:",
     lambda: pfx.test_lru_trace_by_hand()),
    (paged.PagedKVOracle, "slot", "or b in self.key_of", "or False",
     lambda: pfx.test_registered_blocks_are_immutable_and_first_registration_wins()),
    (paged.PagedKVOracle, "register", "if key not in self.registry and b not in self.key_of:",
     "if b not in self.key_of:",
     lambda: pfx.test_registered_blocks_are_immutable_and_first_registration_wins()),
    (paged.PagedKVOracle, "reserve_prefix", "if need > len(self.free) + len(self.cached) - idle:",
     "if need > len(self.free) + len(self.cached):",
     lambda: pfx.test_reusing_every_idle_block_and_needing_one_more_fails_cleanly()),
    (paged.PagedKVOracle, "register", "if b in self.key_of and self.key_of[b] != self._prefix(tokens, i):",
     "if False:",
     lambda: pfx.test_registered_blocks_are_immutable_and_first_registration_wins()),
    (paged.PagedKVOracle, "reserve_prefix", "self.ref[b] += 1", "pass",
     lambda: pfx.test_conversations_under_pool_pressure_keep_exact_contents(0)),
    (paged.PagedKVOracle, "match", "while (m + 1) * self.B <= len(tokens)", "while (m + 2) * self.B <= len(tokens)",
     lambda: pfx.test_worked_103_token_prompt_reuses_96()),
    # swap-out / swap-in
    (paged.PagedKVOracle, "swap_bytes", "(2 * _ceil_div(n_tokens, self.B)", "(_ceil_div(n_tokens, self.B)",
     lambda: swp.test_swap_bytes_are_the_exercise_allocated_bytes()),
    (paged.PagedKVOracle, "swap_out", "image[c, j, i] = cache[layer][b]", "image[c, i % len(table), j % len(layers)] = cache[layer][b]",
     lambda: swp.test_image_layout_holds_each_appended_row_at_its_place()),
    (paged.PagedKVOracle, "swap_out", "self.release(seq)", "None",
     lambda: swp.test_round_trip_restores_attention_exactly_and_frees_blocks()),
    (paged.PagedKVOracle, "swap_in", "self.v[layer][b] = image[1][j][i]", "self.v[layer][b] = image[0][j][i]",
     lambda: swp.test_round_trip_restores_attention_exactly_and_frees_blocks()),
    (paged.PagedKVOracle, "swap_in", "for j, b in enumerate(self.tables[seq]):",
     "for j, b in enumerate(reversed(self.tables[seq])):",
     lambda: swp.test_round_trip_restores_attention_exactly_and_frees_blocks()),
]


def _sizing_pins(golden_dir):
    import json
    import os
    with open(os.path.join(golden_dir, "printed_sizing.json")) as f:
        printed = json.load(f)
    tsz.test_bytes_per_token_printed(printed)
    tsz.test_capacity_12gib(printed)


@pytest.mark.parametrize("case", range(len(MUTANTS)))
def test_planted_mistake_is_caught(case, monkeypatch, golden_dir):
    target, name, old, new, pin = MUTANTS[case]
    real = getattr(target, name)
    func = real if inspect.isfunction(real) else real.__func__
    mutant = _mutated(func, old, new)
    monkeypatch.setattr(target, name, mutant)
    if target is numerics:
        # the pool model holds its own reference to the widening function
        monkeypatch.setattr(paged, name, mutant)
    if target is sizing:
        # sizing helpers call each other through module globals, so the
        # capacity pins see the mutant too
        with pytest.raises(AssertionError):
            _sizing_pins(golden_dir)
        return
    # an assertion, or the mutant crashing on a state the real code never reaches
    with pytest.raises((AssertionError, IndexError, KeyError)):
        pin()


def test_unmutated_pins_pass(golden_dir):
    _sizing_pins(golden_dir)
    tf8.test_code_values_from_definition()
    att.test_matches_scalar_brute_force(2)
    pool.test_invalid_calls()
    assert oracle.PagedKVOracle is paged.PagedKVOracle
    assert np.isfinite(fp8.decode(np.arange(0x7F, dtype=np.uint8))).all()
