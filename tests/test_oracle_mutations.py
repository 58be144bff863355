"""Planted mistakes in the oracle: every one must fail at least one pin.

Each case copies the oracle package (``oracle.c`` and ``__init__.py``) into a
temporary directory, makes one plausible slip in the copy -- a dropped ReLU,
the wrong tie direction, a missing softmax scale or normaliser, an index
taken from the wrong operand, a shared layer reading the wrong cache --
builds that copy with gcc and runs the pins of ``test_oracle_pins.py``
against it.  A slip that passes every pin would be a gap in the pinning, so
the test fails on it.  The mistakes live only in the temporary copies, on the
CPU; the oracle itself is untouched.
"""
import importlib.util
import inspect
import os
import shutil

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PINS = os.path.join(ROOT, "tests", "test_oracle_pins.py")
GOLDEN = os.path.join(ROOT, "tests", "golden")

# (name, file, [(original text, replacement), ...]); every original must
# occur exactly as often as its count in the list says (once by default).
MUTANTS = [
    # ---- indexer
    ("relu_dropped", "oracle.c",
     [("double relu = dot > 0.0 ? dot : 0.0;", "double relu = dot;")]),
    ("relu_after_the_head_weight", "oracle.c",
     [("double relu = dot > 0.0 ? dot : 0.0;\n                acc += (double)wr[j] * relu;",
       "double wd = (double)wr[j] * dot;\n                acc += wd > 0.0 ? wd : 0.0;")]),
    ("weight_of_head_0_for_every_head", "oracle.c",
     [("acc += (double)wr[j] * relu;", "acc += (double)wr[0] * relu;")]),
    ("query_head_0_for_every_head", "oracle.c",
     [("bf16_val(q[(int64_t)j * dI + c])", "bf16_val(q[c])")]),
    ("key_features_reversed", "oracle.c",
     [("bf16_val(kb[s * dI + c])", "bf16_val(kb[s * dI + (dI - 1 - c)])")]),
    ("diagonal_masked", "oracle.c",
     [("if (s > t) { o[s] = -INFINITY; continue; }", "if (s >= t) { o[s] = -INFINITY; continue; }")]),
    ("causal_mask_missing", "oracle.c",
     [("if (s > t) { o[s] = -INFINITY; continue; }", "if (s >= Lk) { o[s] = -INFINITY; continue; }")]),
    ("head_weights_of_batch_0", "oracle.c",
     [("const float *wr = w + (b * Lq + i) * (int64_t)H;", "const float *wr = w + i * (int64_t)H;")]),
    ("indexer_position_without_offset", "oracle.c",
     [("int64_t t = (int64_t)q_offset + i;\n        const uint16_t *q = qI",
       "int64_t t = i;\n        const uint16_t *q = qI")]),
    # ---- top-k
    ("ties_to_the_higher_position", "oracle.c",
     [("return (x->s < y->s) ? -1 : (x->s > y->s);", "return (x->s > y->s) ? -1 : (x->s < y->s);"),
      ("(S[s2] == S[s] && s2 < s)", "(S[s2] == S[s] && s2 > s)")]),
    ("ties_to_the_higher_position_in_the_sort_only", "oracle.c",
     [("return (x->s < y->s) ? -1 : (x->s > y->s);", "return (x->s > y->s) ? -1 : (x->s < y->s);")]),
    ("smallest_scores_kept", "oracle.c",
     [("if (x->v > y->v) return -1;\n    if (x->v < y->v) return 1;",
       "if (x->v < y->v) return -1;\n    if (x->v > y->v) return 1;"),
      ("if (S[s2] > S[s] ||", "if (S[s2] < S[s] ||")]),
    ("selection_left_in_score_order", "oracle.c",
     [("qsort(o, (size_t)m, sizeof(int32_t), int_cmp);", "")]),
    ("visible_set_without_the_query_position", "oracle.c",
     [("int64_t n = t + 1 < Lk ? t + 1 : Lk;", "int64_t n = t < Lk ? t : Lk;", 2)]),
    ("padded_with_position_0", "oracle.c",
     [("for (int64_t j = m; j < k; ++j) o[j] = -1;", "for (int64_t j = m; j < k; ++j) o[j] = 0;"),
      ("for (; m < k; ++m) o[m] = -1;", "for (; m < k; ++m) o[m] = 0;")]),
    ("signed_zeros_compared_by_bits", "oracle.c",
     [("if (x->v > y->v) return -1;\n    if (x->v < y->v) return 1;",
       "if (x->v > y->v) return -1;\n    if (x->v < y->v) return 1;\n"
       "    if (signbit(x->v) != signbit(y->v)) return signbit(x->v) ? 1 : -1;")]),
    # ---- attention
    ("softmax_scale_missing", "oracle.c",
     [("z[i] = scale * dot;", "z[i] = dot;")]),
    ("softmax_not_normalised", "oracle.c",
     [("for (int c = 0; c < d; ++c) oh[c] /= den;", "")]),
    ("max_not_subtracted", "oracle.c",
     [("double e = exp(z[i] - m);", "double e = exp(z[i]);")]),
    ("lse_without_the_max", "oracle.c",
     [("if (lse) lse[h] = m + log(den);", "if (lse) lse[h] = log(den);")]),
    ("values_read_from_K", "oracle.c",
     [("oh[c] += e * bf16_val(Vb[s * d + c]);", "oh[c] += e * bf16_val(Kb[s * d + c]);")]),
    ("key_of_the_query_position", "oracle.c",
     [("dot += bf16_val(qh[c]) * bf16_val(Kb[s * d + c]);",
       "dot += bf16_val(qh[c]) * bf16_val(Kb[t * d + c]);")]),
    ("query_head_0_for_every_attention_head", "oracle.c",
     [("const uint16_t *qh = qrow + (int64_t)h * d;", "const uint16_t *qh = qrow;")]),
    ("index_row_of_the_flattened_row", "oracle.c",
     [("V + b * (int64_t)Lk * d, idx + r * (int64_t)k, k,",
       "V + b * (int64_t)Lk * d, idx + rid * (int64_t)k, k,")]),
    ("beyond_the_query_accepted", "oracle.c",
     [("if (s < 0 || s > t) { rc = -2; z[i] = -INFINITY; continue; }",
       "if (s < 0) { rc = -2; z[i] = -INFINITY; continue; }"),
      ("if (s < 0 || s > t) continue;", "if (s < 0) continue;")]),
    # ---- cross-layer overlap
    ("overlap_counts_the_union", "oracle.c",
     [("both += in_a[s] & in_b[s];", "both += in_a[s] | in_b[s];")]),
    ("overlap_counts_repeats", "oracle.c",
     [("if (x >= 0 && x < Lk) in_a[x] = 1;", "if (x >= 0 && x < Lk) in_a[x] += 1;"),
      ("both += in_a[s] & in_b[s];", "both += in_a[s] < in_b[s] ? in_a[s] : in_b[s];")]),
    ("overlap_fraction_over_the_set_size", "__init__.py",
     [("return np.asarray(counts)[:, 0] / float(k)",
       "return np.asarray(counts)[:, 0] / np.asarray(counts)[:, 1]")]),
    ("jaccard_over_the_sum", "__init__.py",
     [("c[:, 0] / (c[:, 1] + c[:, 2] - c[:, 0] + 1e-8)", "c[:, 0] / (c[:, 1] + c[:, 2] + 1e-8)")]),
    ("bf16_sign_dropped", "oracle.c",
     [("uint32_t u = ((uint32_t)h) << 16;", "uint32_t u = ((uint32_t)(h & 0x7fffu)) << 16;")]),
    ("count_form_off_by_one", "oracle.c",
     [("if (beat < k) o[m++] = (int32_t)s;", "if (beat <= k && m < k) o[m++] = (int32_t)s;")]),
    ("softmax_in_base_2", "oracle.c",
     [("double e = exp(z[i] - m);", "double e = exp2(z[i] - m);")]),
    ("default_scale_over_d", "oracle.c",
     [("if (scale <= 0.0) scale = 1.0 / sqrt((double)d);",
       "if (scale <= 0.0) scale = 1.0 / (double)d;", 2)]),
    ("dense_attention_without_the_query_position", "oracle.c",
     [("for (int64_t s = 0; s <= t; ++s) all[s] = (int32_t)s;",
       "for (int64_t s = 0; s <= t; ++s) all[s] = (int32_t)(s < t ? s : -1);")]),
    ("overlap_ignores_bad_entries", "oracle.c",
     [("else if (x != -1) rc = rc < -2 ? rc : -2;", ""),
      ("else if (y != -1) rc = rc < -2 ? rc : -2;", "")]),
    ("row_positions_of_the_sequence_index", "__init__.py",
     [("return (r % Lq) + q_offset", "return (r // Lq) + q_offset")]),
    ("stack_attention_ignores_the_row_sample", "__init__.py",
     [('o, lse = sparse_attn(L["q"], L["k"], L["v"], cached, q_offset, scale, rows)',
       'o, lse = sparse_attn(L["q"], L["k"], L["v"], cached, q_offset, scale)')]),
    # ---- index cache and layer stack
    ("shared_layers_keep_the_first_full_layer", "__init__.py",
     [("            cached = topk_sort(sc.astype(np.float32), row_positions(B, Lq, q_offset, rows), k)",
       "            cached = cached if cached is not None else topk_sort(\n"
       "                sc.astype(np.float32), row_positions(B, Lq, q_offset, rows), k)")]),
    ("leading_shared_layer_not_rejected", "__init__.py",
     [("elif cached is None:", "elif cached is None and False:")]),
    ("row_positions_without_offset", "__init__.py",
     [("return (r % Lq) + q_offset", "return r % Lq")]),
    ("pattern_characters_unchecked", "__init__.py",
     [('raise ValueError(f"pattern character {c!r} is neither F/1 nor S/0")', "return False")]),
]


def _load_module(name, path, package_dir=None):
    kw = {"submodule_search_locations": [package_dir]} if package_dir else {}
    spec = importlib.util.spec_from_file_location(name, path, **kw)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _mutant_oracle(tmp_path, tag, fname, edits):
    d = tmp_path / f"oracle_{tag}"
    d.mkdir()
    for f in ("oracle.c", "__init__.py"):
        shutil.copy(os.path.join(ROOT, "oracle", f), d / f)
    p = d / fname
    text = p.read_text()
    for e in edits:
        old, new = e[0], e[1]
        count = e[2] if len(e) > 2 else 1
        assert text.count(old) == count, f"{tag}: expected {count} x {old!r}"
        text = text.replace(old, new)
    p.write_text(text)
    mod = _load_module(f"oracle_{tag}", str(d / "__init__.py"), str(d))
    mod._load()            # a slip that does not build is a broken case, not a caught one
    return mod


def _pin_calls():
    """(label, function, kwargs) for every pin, parametrised cases expanded;
    functions are bound later to a fresh copy of the pins module."""
    mod = _load_module("pins_listing", PINS)
    out = []
    for name, fn in sorted(vars(mod).items()):
        if not (name.startswith("test_") and callable(fn)):
            continue
        params = inspect.signature(fn).parameters
        cases = [{}]
        for mark in getattr(fn, "pytestmark", []):
            if mark.name == "parametrize":
                argname, values = mark.args[0], mark.args[1]
                assert "," not in argname
                cases = [dict(c, **{argname: v}) for c in cases for v in values]
        for c in cases:
            if "golden_dir" in params:
                c = dict(c, golden_dir=GOLDEN)
            label = name + ("[" + ",".join(str(v) for k, v in c.items() if k != "golden_dir") + "]"
                            if len(c) > ("golden_dir" in c) else "")
            out.append((label, name, c))
    return out


def _failing_pins(oracle_mod, stop_at_first):
    pins = _load_module(f"pins_under_{oracle_mod.__name__}", PINS)
    pins.oracle = oracle_mod
    failed = []
    for label, name, kw in _pin_calls():
        try:
            getattr(pins, name)(**kw)
        except (Exception, pytest.fail.Exception) as e:   # an assertion, pytest.raises
            # that saw no error, or the mutant's own error
            failed.append((label, type(e).__name__))
            if stop_at_first:
                break
    return failed


def test_unmodified_copy_passes_every_pin(tmp_path):
    """The harness itself: a verbatim copy of the oracle passes all pins."""
    mod = _mutant_oracle(tmp_path, "verbatim", "oracle.c", [])
    assert _failing_pins(mod, stop_at_first=False) == []


@pytest.mark.parametrize("tag,fname,edits", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_fails_a_pin(tmp_path, tag, fname, edits):
    mod = _mutant_oracle(tmp_path, tag, fname, edits)
    assert _failing_pins(mod, stop_at_first=True), f"no pin catches the slip {tag!r}"


def test_concurrent_first_use_builds_and_loads_once(tmp_path):
    """Host threads of a row-per-core pool may all make the first oracle call
    at once; a fresh copy (no library built yet) must come up in every one."""
    from concurrent.futures import ThreadPoolExecutor
    mod_dir = tmp_path / "oracle_fresh"
    mod_dir.mkdir()
    for f in ("oracle.c", "__init__.py"):
        shutil.copy(os.path.join(ROOT, "oracle", f), mod_dir / f)
    mod = _load_module("oracle_fresh", str(mod_dir / "__init__.py"), str(mod_dir))
    with ThreadPoolExecutor(max_workers=8) as ex:
        got = list(ex.map(lambda _: mod.num_threads(), range(8)))
    assert all(n >= 1 for n in got)
    assert sorted(p.name for p in mod_dir.iterdir() if p.suffix == ".tmp") == []
