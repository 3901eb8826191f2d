"""The oracle's pins catch plausible mistakes (CPU only).

Each case copies the oracle's C source, plants one mistake in the copy (an
off-by-one in the mask predicate, a dropped term, a wrong sign, a transposed
operand, a wrong index), compiles it, routes the oracle through the mutant and
checks that at least one pin of ``test_oracle_pins.py`` now fails.  A control
case compiles the unchanged source the same way and checks that the same pins
pass.  Every planted mistake keeps all memory accesses in bounds.

The head and batch mapping lives in the oracle's Python layer; those mistakes
are planted in a copy of the module's source, executed as a separate module.
"""
import types

import pytest

import oracle
import test_balance
import test_oracle_pins as pins

FWD = [
    lambda o: pins.test_unmasked_equals_sdpa(o, 33, 50, 16),
    lambda o: pins.test_causal_encoding_equals_sdpa_causal(o, 40, 32),
    lambda o: pins.test_random_mask_equals_sdpa_boolean_mask(o),
    lambda o: pins.test_zero_query_closed_form_random_masks(o, 0),
    lambda o: pins.test_golden_hand_example(o),
]
BWD = [
    lambda o: pins.test_backward_finite_differences(o, 2, 4, 2),
    lambda o: pins.test_backward_equals_torch_autograd_sdpa(o),
]
CLASSIFY = [lambda o, s=s: pins.test_classify_sound_random(o, s) for s in range(6)] + [
    lambda o: pins.test_classify_causal_closed_form(o),
]
CLASSIFY_GOLDEN = [lambda o: pins.test_classify_golden_clauses(o)]
LOCALIZE = [lambda o, s=s: pins.test_localize_reproduces_dense_rows(o, s) for s in range(3)]
LOCALIZE_MULTI = [lambda o, s=s: pins.test_localize_multi_reproduces_dense_rows(o, s) for s in range(3)]
COUNT = [lambda o: pins.test_count_unmasked(o)]
TILE_COSTS = [lambda o: test_balance.test_tile_costs_sum_to_pair_count(o),
              lambda o: test_balance.test_tile_costs_causal_closed_form(o)]
COUNT_HEADS = [lambda o: pins.test_count_unmasked_batches_and_per_head_masks(o)]
GQA = [
    lambda o: pins.test_gqa_and_batches_equal_sdpa_with_repeated_kv(o),
    lambda o: pins.test_gqa_backward_equals_torch_autograd_repeated_kv(o),
]
PER_HEAD = [lambda o: pins.test_per_head_masks_equal_sdpa_per_head(o)]

# (name, text in the source, planted replacement, pins expected to catch it)
MUTATIONS = [
    ("predicate_lts_strict", "(lts[j] <= i && i < lte[j])", "(lts[j] < i && i < lte[j])", FWD),
    ("predicate_ute_inclusive", "(uts[j] <= i && i < ute[j])", "(uts[j] <= i && i <= ute[j])", FWD),
    ("scale_dropped", "s_buf[j] = scale * dot(qi, k + j * d, d);", "s_buf[j] = dot(qi, k + j * d, d);", FWD),
    ("lse_without_max", "      lse[r] = m + log(l);\n", "      lse[r] = log(l);\n", FWD),
    ("softmax_unnormalised", "const double p = exp(s[j] - m) / l;", "const double p = exp(s[j] - m);", FWD),
    ("ds_sign", "const double ds = s[j] * (dp[j] - D);", "const double ds = s[j] * (dp[j] + D);", BWD),
    ("dq_wrong_operand", "g[c] += scale * ds * k[j * d + c];", "g[c] += scale * ds * v[j * d + c];", BWD),
    ("dk_scale_dropped", "gk[c] += scale * ds * q[i * d + c];", "gk[c] += ds * q[i * d + c];", BWD),
    ("dv_wrong_operand", "gv[c] += p * dout[i * d + c];", "gv[c] += p * q[i * d + c];", BWD),
    ("row_sum_D_wrong_operand", "D += exp(s[j] - lse[i]) * dot(dout + i * d, v + j * d, d);",
     "D += exp(s[j] - lse[i]) * dot(dout + i * d, k + j * d, d);", BWD),
    ("classify_skip_uses_min", "if ((mx[0] <= r0 && mn[1] >= r1)", "if ((mn[0] <= r0 && mn[1] >= r1)", CLASSIFY),
    ("classify_full_uses_max", "else if ((mn[0] >= r1 ||", "else if ((mx[0] >= r1 ||", CLASSIFY),
    # conservative slips (sound, so the soundness pins pass them): the golden catches each
    ("classify_drop_empty_lt", "(mn[0] >= r1 || mx[1] <= r0 || mn[0] >= mx[1])", "(mn[0] >= r1 || mx[1] <= r0)",
     CLASSIFY_GOLDEN),
    ("classify_drop_empty_ut", "(mn[2] >= r1 || mx[3] <= r0 || mn[2] >= mx[3])", "(mn[2] >= r1 || mx[3] <= r0)",
     CLASSIFY_GOLDEN),
    ("classify_lt_ends_strict", "mx[1] <= r0", "mx[1] < r0", CLASSIFY_GOLDEN),
    ("classify_ut_ends_strict", "mx[3] <= r0", "mx[3] < r0", CLASSIFY_GOLDEN),
    ("classify_lt_starts_strict", "(mn[0] >= r1 ||", "(mn[0] > r1 ||", CLASSIFY_GOLDEN),
    ("classify_ut_starts_strict", "(mn[2] >= r1 ||", "(mn[2] > r1 ||", CLASSIFY_GOLDEN),
    ("classify_skip_lt_covers_strict", "mx[0] <= r0 && mn[1] >= r1", "mx[0] <= r0 && mn[1] > r1", CLASSIFY_GOLDEN),
    ("classify_skip_ut_starts_strict", "mx[2] <= r0 && mn[3] >= r1", "mx[2] < r0 && mn[3] >= r1", CLASSIFY_GOLDEN),
    ("classify_skip_ut_covers_strict", "mx[2] <= r0 && mn[3] >= r1", "mx[2] <= r0 && mn[3] > r1", CLASSIFY_GOLDEN),
    ("classify_skip_lt_starts_strict", "mx[0] <= r0 && mn[1] >= r1", "mx[0] < r0 && mn[1] >= r1", CLASSIFY_GOLDEN),
    ("localize_shift_off_by_one", "x = x - a;", "x = x - a - 1;", LOCALIZE),
    ("localize_multi_first_offset", "acc += x - a[t];", "acc += x - a[0];", LOCALIZE_MULTI),
    ("count_negated", "cnt += !is_masked(lts, lte, uts, ute, j, i);\n    total += cnt;",
     "cnt += is_masked(lts, lte, uts, ute, j, i);\n    total += cnt;", COUNT),
    ("tile_costs_row_past_tile", "for (int64_t i = t * bm; i < r1; ++i)", "for (int64_t i = t * bm; i <= r1; ++i)",
     TILE_COSTS),
]

# (name, text in oracle/__init__.py, planted replacement, pins expected to catch it)
PY_MUTATIONS = [
    ("kv_head_interleaved", "return (lambda h: h // G), (lambda h: 0 if Hm == 1 else h)",
     "return (lambda h: h % Hkv), (lambda h: 0 if Hm == 1 else h)", GQA),
    ("mask_head_always_first", "(lambda h: 0 if Hm == 1 else h)", "(lambda h: 0)", PER_HEAD),
    ("dkdv_group_interleaved", "for h in range(hk * G, (hk + 1) * G):", "for h in range(hk, Hq, Hkv):", GQA),
    ("forward_mask_of_first_batch",
     "vecs = [np.ascontiguousarray(x[b, hm]) for x in m4]\n        if sel is None:\n            qb = _f64(",
     "vecs = [np.ascontiguousarray(x[0, hm]) for x in m4]\n        if sel is None:\n            qb = _f64(", GQA),
    ("dq_mask_of_first_batch",
     "vecs = [np.ascontiguousarray(x[b, hm]) for x in m4]\n        if sel is None:\n            qb, gb,",
     "vecs = [np.ascontiguousarray(x[0, hm]) for x in m4]\n        if sel is None:\n            qb, gb,", GQA),
    ("count_per_head_masks_broadcast", "total += per_head[0] * Hq if Hm == 1 else sum(per_head)",
     "total += per_head[0] * Hq", COUNT_HEADS),
    ("count_last_batch_only", "        total += per_head[0] * Hq if Hm == 1 else sum(per_head)\n",
     "        total = per_head[0] * Hq if Hm == 1 else sum(per_head)\n", COUNT_HEADS),
]


def _python_source() -> str:
    with open(oracle.__file__) as f:
        return f.read()


def _python_variant(text: str):
    """Executes a version of the oracle's Python layer as a module of its own (same C library)."""
    mod = types.ModuleType("oracle_python_variant")
    mod.__file__ = oracle.__file__
    exec(compile(text, oracle.__file__, "exec"), mod.__dict__)
    return mod


def _fails_with(mod, check) -> bool:
    try:
        check(mod)
    except AssertionError:
        return True
    return False


def _fails(check) -> bool:
    try:
        check(oracle)
    except AssertionError:
        return True
    return False


@pytest.fixture(scope="module")
def source():
    oracle.build_oracle()
    return oracle.source()


def test_control_unchanged_source_passes_every_pin(source, tmp_path):
    lib = oracle.build_variant(source, str(tmp_path))
    with oracle.use_library(lib):
        for check in FWD + BWD + CLASSIFY + CLASSIFY_GOLDEN + LOCALIZE + LOCALIZE_MULTI + COUNT + TILE_COSTS:
            assert not _fails(check)


@pytest.mark.parametrize("name,old,new,checks", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(source, tmp_path, name, old, new, checks):
    assert source.count(old) == 1, f"{name}: the text to mutate must occur exactly once"
    lib = oracle.build_variant(source.replace(old, new), str(tmp_path))
    with oracle.use_library(lib):
        caught = [i for i, check in enumerate(checks) if _fails(check)]
    assert caught, f"{name}: no pin caught the planted mistake"


def test_control_unchanged_python_layer_passes_its_pins():
    oracle.build_oracle()
    mod = _python_variant(_python_source())
    for check in GQA + PER_HEAD + COUNT_HEADS + FWD[:1] + BWD[:1]:
        assert not _fails_with(mod, check)


@pytest.mark.parametrize("name,old,new,checks", PY_MUTATIONS, ids=[m[0] for m in PY_MUTATIONS])
def test_planted_mapping_mistake_is_caught(name, old, new, checks):
    oracle.build_oracle()
    text = _python_source()
    assert text.count(old) == 1, f"{name}: the text to mutate must occur exactly once"
    mod = _python_variant(text.replace(old, new))
    caught = [i for i, check in enumerate(checks) if _fails_with(mod, check)]
    assert caught, f"{name}: no pin caught the planted mistake"
