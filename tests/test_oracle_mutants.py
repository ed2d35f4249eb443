"""The oracle's pins catch plausible mistakes (CPU only).

Each mutant is a copy of the oracle with one plausible mistake planted in its C source: a
dropped term, a wrong sign or index, an off-by-one, a swapped operand.  The copy is compiled
into its own directory and run through the pin suite of test_oracle_pins.py, which must fail
for it.  Pins run cheapest first and a mutant stops at its first failing pin.  Nothing here
touches the real oracle or the CUDA library.
"""
import importlib.util
import inspect
import itertools
import os
import shutil
import time

import pytest

from conftest import ROOT

ORACLE_DIR = os.path.join(ROOT, "oracle")

# (name, text in pa_oracle.c, replacement); each text occurs exactly once
MUTANTS = [
    ("slot offset", "+ logical] * block_size\n                + p % block_size;",
     "+ logical] * block_size\n                + (p + 1) % block_size;"),
    ("causal limit off by one", "int limit = ctx - q_len + i; /* last key this query may see */",
     "int limit = ctx - q_len + i - 1;"),
    ("GQA map", "int h = g * group + hh;", "int h = hh * num_kv_heads + g;"),
    ("missing softmax scale", "s[p] = scale * acc;", "s[p] = acc;"),
    ("halved LSE", "return mx + log(sum);", "return mx + 0.5 * log(sum);"),
    ("E4M3 ties to odd", "return sign | (uint8_t)((lo & 1) == 0 ? lo : hi);",
     "return sign | (uint8_t)((lo & 1) == 1 ? lo : hi);"),
    ("E4M3 exponent bias", "mag = ldexp(1.0 + (double)m / 8.0, e - 7);",
     "mag = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    ("K written as V", "= v[src];", "= k[src];"),
    ("FP8 reciprocal multiply", "float yk = bf16_to_float(k[src]) / k_scale[h];",
     "float yk = bf16_to_float(k[src]) * (1.0f / k_scale[h]);"),
    ("allocator does not stop", "if (stopped || total > max_blocks_per_seq || need > count) {",
     "if (total > max_blocks_per_seq || need > count) {"),
    ("allocator counts new tokens only", "need = total - have;",
     "need = oracle_blocks_needed(n, block_size);"),
    ("allocator takes from the tail", "queue[(head + j) % capacity]",
     "queue[(head + count - 1 - j) % capacity]"),
    ("free at the head", "tail = ((int64_t)state[0] + state[1]) % capacity;",
     "tail = state[0];"),
    ("window off by one",
     "if (window > 0 && limit - window + 1 > lo) lo = limit - window + 1;",
     "if (window > 0 && limit - window > lo) lo = limit - window;"),
    ("window 1 read as full attention",
     "if (window > 0 && limit - window + 1 > lo) lo = limit - window + 1;",
     "if (window > 1 && limit - window + 1 > lo) lo = limit - window + 1;"),
    ("local chunk off by one",
     "if (local_chunk > 0 && limit / local_chunk * local_chunk > lo) lo = limit / local_chunk * local_chunk;",
     "if (local_chunk > 0 && (limit - 1) / local_chunk * local_chunk > lo) lo = (limit - 1) / local_chunk * local_chunk;"),
    ("DCP shares interleave tokens", "if ((p / block_size) % world == rank) ++n;",
     "if (p % world == rank) ++n;"),
    ("DCP local block index",
     "local_table[(int64_t)r * max_blocks_per_seq + j / world] * block_size",
     "local_table[(int64_t)r * max_blocks_per_seq + j % world] * block_size"),
    ("merge LSE in log2", "lse[n] = L + log(wsum);", "lse[n] = L + log2(wsum);"),
    ("merge weighs empty parts", "if (w == 0.0) continue;", ""),
]


def _load_pins():
    spec = importlib.util.spec_from_file_location(
        "oracle_pins_for_mutants", os.path.join(ROOT, "tests", "test_oracle_pins.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _pin_calls(pins):
    """Every (name, function, kwargs) of the pin suite that takes the oracle, parametrize
    marks expanded."""
    calls = []
    for name, fn in vars(pins).items():
        if not name.startswith("test_") or not callable(fn):
            continue
        if "oracle_mod" not in inspect.signature(fn).parameters:
            continue
        grids = []
        for mark in getattr(fn, "pytestmark", []):
            if mark.name != "parametrize":
                continue
            names = [n.strip() for n in mark.args[0].split(",")]
            values = [v if len(names) > 1 else (v,) for v in mark.args[1]]
            grids.append([dict(zip(names, v)) for v in values])
        for combo in itertools.product(*grids) if grids else [()]:
            kw = {}
            for part in combo:
                kw.update(part)
            calls.append((name, fn, kw))
    return calls


def _variant(tmp_path, idx, old, new):
    d = tmp_path / f"oracle_mutant_{idx}"
    d.mkdir()
    for f in ("__init__.py", "brute.py"):
        shutil.copy(os.path.join(ORACLE_DIR, f), d / f)
    src = open(os.path.join(ORACLE_DIR, "pa_oracle.c")).read()
    assert src.count(old) == 1, f"mutation anchor not unique: {old!r}"
    (d / "pa_oracle.c").write_text(src.replace(old, new))
    spec = importlib.util.spec_from_file_location(f"oracle_mutant_{idx}", d / "__init__.py",
                                                  submodule_search_locations=[str(d)])
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    return mod


def test_every_planted_mistake_fails_a_pin(tmp_path, oracle_mod):
    pins = _load_pins()
    calls = _pin_calls(pins)
    assert len(calls) > 60
    # cheapest pins first: time each once on the real oracle (which must pass them all)
    cost = []
    for name, fn, kw in calls:
        t0 = time.perf_counter()
        fn(oracle_mod=oracle_mod, **kw)
        cost.append(time.perf_counter() - t0)
    order = sorted(range(len(calls)), key=lambda i: cost[i])
    survivors = []
    for idx, (label, old, new) in enumerate(MUTANTS):
        mutant = _variant(tmp_path, idx, old, new)
        killed = None
        for i in order:
            name, fn, kw = calls[i]
            try:
                fn(oracle_mod=mutant, **kw)
            except Exception:  # an assertion, or the oracle refusing its own output
                killed = name
                break
        if killed is None:
            survivors.append(label)
    assert not survivors, f"mistakes no pin catches: {survivors}"
