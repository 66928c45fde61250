"""The oracle's pins must catch plausible mistakes in it.

Each mutant is a copy of ``oracle/kda_oracle.c`` with one deliberate slip
(a dropped term, a flipped sign, a wrong index, a transposed operand, the
epsilon moved out of the root ...), compiled to a temporary library on the
CPU.  With the mutant swapped in, at least one pin of
``test_oracle_pins.py`` has to fail.  The real oracle source is never
modified.
"""
import ctypes
import inspect
import os
import subprocess

import pytest

import oracle as oracle_pkg
from tests import test_oracle_backward as bwd_pins
from tests import test_oracle_decode as dec_pins
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle_pkg.__file__), "kda_oracle.c")

MUTANTS = {
    "no_decay": ("S[(int64_t)d * V + c] *= e;", "(void)e;"),
    "residual_sign": ("r[c] = vt[c] - acc;", "r[c] = vt[c] + acc;"),
    "no_beta": ("const double bk = bt * kt[d];", "const double bk = kt[d];"),
    "output_uses_k": ("acc += (scale * qt[d])", "acc += (scale * kt[d])"),
    "no_scale": ("acc += (scale * qt[d])", "acc += (qt[d])"),
    "transposed_update": ("S[(int64_t)d * V + c] += bk * r[c];", "S[(int64_t)c * V + d] += bk * r[c];"),
    "eps_outside_sqrt": ("sqrtf(ss + 1e-6f)", "(sqrtf(ss) + 1e-6f)"),
    "gqa_modulo": ("const int hq = h / group;", "const int hq = h % H;"),
    "gate_wrong_channel": ("const double e = exp(gt[d]);", "const double e = exp(gt[K - 1 - d]);"),
    "norm_truncates": ("u += 0x7fffu + lsb;", "u += 0u * lsb;"),
    "decay_after_update_output": ("ot[c] = acc;", "ot[c] = acc * exp(gt[0]);"),
}

# slips in the reverse mode (each site occurs only in the backward)
BWD_MUTANTS = {
    "bwd_dq_no_scale": ("dqt[d] = scale * acc;", "dqt[d] = acc;"),
    "bwd_dq_from_previous_state": ("acc += St[(int64_t)d * V + c] * dot[c];", "acc += Sp[(int64_t)d * V + c] * dot[c];"),
    "bwd_dr_no_beta": ("dr[c] = bt * acc;", "dr[c] = acc;"),
    "bwd_dbeta_uses_v": ("db += acc * r[c];", "db += acc * vt[c];"),
    "bwd_dk_sign": ("dkt[d] = bt * a1 - a2;", "dkt[d] = bt * a1 + a2;"),
    "bwd_dropped_rank1_term": ("const double x = dS[(int64_t)d * V + c] - kt[d] * dr[c];",
                               "const double x = dS[(int64_t)d * V + c];"),
    "bwd_dg_from_undecayed_state": ("acc += Sd[(int64_t)d * V + c] * x;", "acc += Sp[(int64_t)d * V + c] * x;"),
    "bwd_adjoint_not_decayed": ("dS[(int64_t)d * V + c] = e * x;", "dS[(int64_t)d * V + c] = x;"),
    "bwd_wrong_checkpoint": ("memcpy(blk, ckpt + (size_t)m * KV,", "memcpy(blk, ckpt + (size_t)(m > 0 ? m - 1 : 0) * KV,"),
}


def _pin_functions():
    out = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if name.startswith("test_") and "oracle" in inspect.signature(fn).parameters:
            if "chunk" in inspect.signature(fn).parameters:
                out.append((name, lambda o, fn=fn: fn(o, 64)))
            else:
                out.append((name, fn))
    return out


def _run_mutant(old, new, tmp_path, pin_functions):
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site {old!r} not found"
    mutated = src.replace(old, new, 1)
    c_path = tmp_path / "mut.c"
    so_path = tmp_path / "libmut.so"
    c_path.write_text(mutated)
    subprocess.run(["gcc", *oracle_pkg.GCC_FLAGS, str(c_path), "-o", str(so_path), "-lm"], check=True)

    real = oracle_pkg._load()
    lib = ctypes.CDLL(str(so_path))
    for fname in ("kda_oracle_l2norm_bf16", "kda_oracle_recurrence_f64", "kda_oracle_forward",
                  "kda_oracle_max_threads", "kda_oracle_f64_to_bf16", "kda_oracle_backward_f64"):
        f, r = getattr(lib, fname), getattr(real, fname)
        f.argtypes, f.restype = r.argtypes, r.restype
    caught = []
    oracle_pkg._lib = lib
    try:
        for name, fn in pin_functions:
            try:
                fn(oracle_pkg)
            except AssertionError:
                caught.append(name)
    finally:
        oracle_pkg._lib = real
    return caught


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_pins_catch_mutant(mutant, tmp_path):
    old, new = MUTANTS[mutant]
    assert _run_mutant(old, new, tmp_path, _pin_functions()), f"no pin caught mutant {mutant}"


def _bwd_pin_functions():
    return [(name, fn) for name, fn in inspect.getmembers(bwd_pins, inspect.isfunction)
            if name.startswith("test_") and "oracle" in inspect.signature(fn).parameters]


@pytest.mark.parametrize("mutant", sorted(BWD_MUTANTS))
def test_backward_pins_catch_mutant(mutant, tmp_path):
    old, new = BWD_MUTANTS[mutant]
    assert _run_mutant(old, new, tmp_path, _bwd_pin_functions()), f"no pin caught mutant {mutant}"


# slips in the decode step's row and slot bookkeeping (``oracle.decode_step``, Python); the arithmetic under it is
# the recurrence above, whose mutants are caught by the forward pins
DECODE_MUTANTS = {
    "dec_output_at_slot": ('o[rows] = res["o64"][:, 0]', 'o[idx[rows] % B] = res["o64"][:, 0]'),
    "dec_state_not_written_back": ('pool[idx[rows]] = res["state"]', "pass"),
    "dec_state_written_to_row": ('pool[idx[rows]] = res["state"]', 'pool[rows % pool.shape[0]] = res["state"]'),
    "dec_start_from_row_slot": ("s0 = np.ascontiguousarray(pool[idx[rows]], dtype=np.float32)",
                                "s0 = np.ascontiguousarray(pool[rows % pool.shape[0]], dtype=np.float32)"),
    "dec_padding_rows_kept": ("rows = np.nonzero(idx >= 0)[0]", "rows = np.arange(B)"),
}


def _python_pins_failing(monkeypatch, func, old, new, pins):
    """Swap a copy of oracle function ``func`` with one slip into the oracle module and run ``pins``
    (name, callable) against it; returns the names of the pins that failed."""
    src = inspect.getsource(getattr(oracle_pkg, func))
    assert src.count(old) == 1, f"mutation site {old!r} not found"
    namespace = dict(vars(oracle_pkg))
    exec(compile(src.replace(old, new), "<oracle mutant>", "exec"), namespace)
    monkeypatch.setattr(oracle_pkg, func, namespace[func])
    caught = []
    for name, fn in pins:
        try:
            fn()
        except (AssertionError, IndexError, ValueError):
            caught.append(name)
    return caught


def _decode_pins_failing(monkeypatch, old, new):
    pins = [(n, f) for n, f in inspect.getmembers(dec_pins, inspect.isfunction) if n.startswith("test_")]
    return _python_pins_failing(monkeypatch, "decode_step", old, new, pins)


def test_decode_mutant_harness_passes_the_unchanged_function(monkeypatch):
    old = "rows = np.nonzero(idx >= 0)[0]"
    assert _decode_pins_failing(monkeypatch, old, old) == []


@pytest.mark.parametrize("mutant", sorted(DECODE_MUTANTS))
def test_decode_pins_catch_mutant(mutant, monkeypatch):
    old, new = DECODE_MUTANTS[mutant]
    assert _decode_pins_failing(monkeypatch, old, new), f"no pin caught mutant {mutant}"


# slips in the backward's raw-input wrapper (group sums over the value heads of a Q/K head, the normalisation's
# Jacobian); each is caught by the differences of the smooth forward or of the normalisation
WRAPPER_MUTANTS = {
    "wrap_no_group_sum": ("backward", "dqn = dqn.reshape(B, T, H, grp, K).sum(3)",
                          "dqn = dqn.reshape(B, T, H, grp, K)[:, :, :, 0]"),
    "wrap_dk_through_q": ("backward", "dk = l2norm_backward_f64(bits_to_f32(kb), dkn)",
                          "dk = l2norm_backward_f64(bits_to_f32(qb), dkn)"),
    "jac_no_projection": ("l2norm_backward_f64", "return dy / n - x * (x * dy).sum(-1, keepdims=True) / n ** 3",
                          "return dy / n"),
    "jac_wrong_power": ("l2norm_backward_f64", "/ n ** 3", "/ n ** 2"),
}


def _wrapper_pins():
    return [(name, lambda fn=fn: fn(oracle_pkg)) for name, fn in inspect.getmembers(bwd_pins, inspect.isfunction)
            if name in ("test_raw_input_backward_matches_differences_loosely", "test_l2norm_jacobian")]


def test_wrapper_mutant_harness_passes_the_unchanged_functions(monkeypatch):
    for func, old, _ in WRAPPER_MUTANTS.values():
        assert _python_pins_failing(monkeypatch, func, old, old, _wrapper_pins()) == []
        monkeypatch.undo()  # the next site is read from the real function's source


@pytest.mark.parametrize("mutant", sorted(WRAPPER_MUTANTS))
def test_wrapper_pins_catch_mutant(mutant, monkeypatch):
    func, old, new = WRAPPER_MUTANTS[mutant]
    assert _python_pins_failing(monkeypatch, func, old, new, _wrapper_pins()), f"no pin caught mutant {mutant}"
