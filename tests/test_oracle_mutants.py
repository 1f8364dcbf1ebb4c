"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a temporary copy of the oracle (its C source or its
layout module, never the real files), builds it, swaps it in for the duration of the
case, and runs the pin tests: at least one must fail.  A pin set that let a mutant
through would not pin the oracle.
"""
import ctypes
import importlib.util
import os
import subprocess
import tempfile

import pytest

import oracle
import oracle.layout as real_layout

import test_oracle_adamw as T_adamw
import test_oracle_fp16 as T_fp16
import test_oracle_ring as T_ring
import test_oracle_stages as T_stages
import test_oracle_wire as T_wire

ORACLE_DIR = os.path.dirname(oracle.__file__)

PINS = [
    T_fp16.test_half_to_float_exhaustive, T_fp16.test_float_to_half_special_cases,
    T_ring.test_three_gpu_walkthrough_scatter_reduce, T_ring.test_three_gpu_walkthrough_all_gather,
    lambda: [T_ring.test_order_probe(k) for k in range(3)],
    T_ring.test_brute_force_exact_inputs_equal_direct_sum, T_ring.test_brute_force_general_inputs_within_summation_bound,
    T_adamw.test_first_step_closed_form, T_adamw.test_zero_gradient_only_decays,
    T_adamw.test_matches_torch_adamw_single_rank, T_adamw.test_nonfinite_counted_per_bucket_and_propagated,
    T_stages.test_allgather_is_concatenation_of_partitions, T_stages.test_literal_send_counts_match_closed_form,
    T_stages.test_memory_and_comm_closed_forms_match_pages, T_stages.test_layout_brute_force,
    T_stages.test_three_gpu_thirds,
    T_wire.test_one_wire_hop_is_the_rounded_fp16_sum, T_wire.test_wire_rounds_at_every_hop,
    T_wire.test_wire_overflow_depends_on_ring_order, T_wire.test_scaler_follows_hand_trace,
    T_wire.test_dynamic_run_skips_overflowing_steps,
]

# (name, original text, mutated text) in oracle.c
C_MUTANTS = [
    ("fold starts one rank late", "const int64_t k = imod(r - h, n_ranks);", "const int64_t k = imod(r - h + 1, n_ranks);"),
    ("receiver drops its own value", "wire16 ? wire16_add(incoming, own) : incoming + own;",
     "wire16 ? wire16_add(incoming, own) : incoming;"),
    ("sum read from the wrong rank", "const int64_t holder = imod(k - 1, n_ranks);", "const int64_t holder = imod(k, n_ranks);"),
    ("all-gather passes the wrong chunk", "const int64_t k = imod(r + 1 - h, n_ranks);", "const int64_t k = imod(r - h, n_ranks);"),
    ("no weight decay", "float pp = *p * s[1];", "float pp = *p;"),
    ("beta2 used for the first moment", "const float mm = *m * s[2] + g * s[3];", "const float mm = *m * s[4] + g * s[3];"),
    ("no second-moment bias correction", "const float denom = root / s[7] + s[8];", "const float denom = root + s[8];"),
    ("eps inside the correction", "const float denom = root / s[7] + s[8];", "const float denom = root / (s[7] + s[8]);"),
    ("no mean over ranks", "s[0] = (float)(1.0 / ((double)n_ranks * loss_scale));", "s[0] = (float)(1.0 / loss_scale);"),
    ("no first-moment bias correction", "s[6] = (float)(lr / (1.0 - pow(beta1, (double)t)));", "s[6] = (float)lr;"),
    ("gradient not squared", "const float gg = g * g;", "const float gg = g;"),
    ("update sign flipped", "pp = pp - s[6] * ratio;", "pp = pp + s[6] * ratio;"),
    ("fp16 rounding truncates", "const double q = rint(a / ulp);", "const double q = floor(a / ulp);"),
    ("fp16 subnormal scale off", "mag = ldexp((double)f, -24);", "mag = ldexp((double)f, -25);"),
    ("fp16 exponent bias off", "mag = ldexp((double)(1024 + f), e - 25);", "mag = ldexp((double)(1024 + f), e - 24);"),
    ("non-finite count misses inf", "if (!isfinite(reduced[i])) ++c;", "if (isnan(reduced[i])) ++c;"),
    ("sender counter not kept", "if (sent) sent[r] += chi - clo;", "if (sent) sent[r] += 0;"),
    ("wire sum not rounded to fp16", "return oracle_half_to_float(oracle_double_to_half((double)incoming + (double)own));",
     "return incoming + own;"),
    ("wire sum rounded through fp32", "oracle_double_to_half((double)incoming + (double)own)",
     "oracle_double_to_half((double)(float)((double)incoming + (double)own) * 1.0000001)"),
]

# (name, original, mutated) in layout.py
PY_MUTANTS = [
    ("shard not rounded up", "S = roundup(ceil_div(psi, n_ranks), pad_align) if psi > 0 else 0",
     "S = (psi // n_ranks) if psi > 0 else 0"),
    ("buckets cut from the head", "lo = max(0, hi - bucket_elems)\n                buckets.append((lo, hi))",
     "lo = max(0, hi - bucket_elems)\n                buckets.insert(0, (lo, hi))"),
    ("ZeRO-3 without the backward gather", "phases = 3 if stage == 3 else 2", "phases = 2"),
    ("ZeRO-2 keeps full gradients", "p16, g16, os_ = 2 * psi, 2 * S, 12 * S", "p16, g16, os_ = 2 * psi, 2 * psi, 12 * S"),
    ("DDP optimizer state sharded", "p16, g16, os_ = 2 * psi, 2 * psi, 12 * psi", "p16, g16, os_ = 2 * psi, 2 * psi, 12 * S"),
]

# (name, original, mutated) in the oracle's Python composition (oracle/__init__.py)
INIT_MUTANTS = [
    ("scaler never grows", "                self.scale *= self.factor\n", "                self.scale *= 1.0\n"),
    ("scaler counts skipped steps as applied", "            self.skipped += 1\n", "            self.skipped += 1\n            self.step += 1\n"),
    ("overflow step still updates", "        if bad == 0:\n            h = Hyper(", "        if True:\n            h = Hyper("),
    ("scale window not reset", "                self.clean_steps = 0\n", "                pass\n"),
]


def _some_pin_fails():
    for pin in PINS:
        try:
            pin()
        except (AssertionError, ValueError, IndexError):
            return True
    return False


@pytest.fixture(scope="module")
def workdir():
    with tempfile.TemporaryDirectory() as d:
        yield d


@pytest.mark.parametrize("name,old,new", C_MUTANTS, ids=[m[0] for m in C_MUTANTS])
def test_c_mutant_is_caught(name, old, new, workdir, monkeypatch):
    src = open(os.path.join(ORACLE_DIR, "oracle.c")).read()
    assert old in src, name
    tag = str(abs(hash(name)))
    c_path = os.path.join(workdir, f"mutant_{tag}.c")
    so_path = os.path.join(workdir, f"mutant_{tag}.so")
    open(c_path, "w").write(src.replace(old, new, 1))     # the first occurrence only
    subprocess.run(["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fPIC", "-shared", "-o", so_path, c_path, "-lm"],
                   check=True)
    monkeypatch.setattr(oracle, "_LIB", oracle.configure(ctypes.CDLL(so_path)))
    assert _some_pin_fails(), f"no pin caught the planted mistake: {name}"


@pytest.mark.parametrize("name,old,new", PY_MUTANTS, ids=[m[0] for m in PY_MUTANTS])
def test_layout_mutant_is_caught(name, old, new, workdir, monkeypatch):
    src = open(real_layout.__file__).read()
    assert src.count(old) == 1, name
    path = os.path.join(workdir, f"layout_mutant_{abs(hash(name))}.py")
    open(path, "w").write(src.replace(old, new))
    spec = importlib.util.spec_from_file_location(f"layout_mutant_{abs(hash(name))}", path)
    mutant = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mutant)
    for mod in (oracle, T_ring, T_adamw, T_stages):
        for fn in ("make_layout", "counters"):
            if hasattr(mod, fn):
                monkeypatch.setattr(mod, fn, getattr(mutant, fn))
    assert _some_pin_fails(), f"no pin caught the planted mistake: {name}"


def test_unmutated_oracle_passes_every_pin():
    assert not _some_pin_fails()


@pytest.mark.parametrize("name,old,new", INIT_MUTANTS, ids=[m[0] for m in INIT_MUTANTS])
def test_composition_mutant_is_caught(name, old, new, monkeypatch):
    src = open(os.path.join(ORACLE_DIR, "__init__.py")).read()
    assert old in src, name
    ns = {"__name__": "oracle_mutant"}
    mutated = src.replace(old, new, 1).replace("from . import build as _build", "from oracle import build as _build")
    mutated = mutated.replace("from .layout import", "from oracle.layout import")
    exec(compile(mutated, "oracle_mutant", "exec"), ns)
    monkeypatch.setattr(oracle, "LossScaler", ns["LossScaler"])
    monkeypatch.setattr(oracle, "run_steps_dynamic", ns["run_steps_dynamic"])
    assert _some_pin_fails(), f"no pin caught the planted mistake: {name}"
