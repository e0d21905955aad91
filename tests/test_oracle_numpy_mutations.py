"""The pins of the numpy oracles (linear cross-attention, the Mix-FFN temporal
convolution) must reject plausible mistakes.

Each case plants one mistake in a private copy of the oracle function's source
(on the CPU), swaps it in for the real one, and runs the pin tests against it:
at least one of them has to fail. Mirrors the planted-mistake test of the C
oracle.
"""
import importlib.util
import inspect
import os
import typing

import numpy as np
import pytest

import oracle
from oracle import tconv

HERE = os.path.dirname(os.path.abspath(__file__))


def _load(name):
    spec = importlib.util.spec_from_file_location("_pins_" + name, os.path.join(HERE, name))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _mutant_function(fn, old, new):
    src = inspect.getsource(fn)
    assert src.count(old) == 1, "mutation anchor not found: " + old
    ns = {"np": np, "Optional": typing.Optional, "Tuple": typing.Tuple}
    exec(compile(src.replace(old, new), "<mutant>", "exec"), ns)
    return ns[fn.__name__]


def _any_fails(calls):
    for call in calls:
        try:
            call()
        except AssertionError:
            return True
    return False


TCONV_MUTANTS = {
    "taps_reversed": ("w[0] * framed[:, 0:T] + w[1] * framed[:, 1:T + 1] + w[2] * framed[:, 2:T + 2]",
                      "w[2] * framed[:, 0:T] + w[1] * framed[:, 1:T + 1] + w[0] * framed[:, 2:T + 2]"),
    "no_shortcut": ("y = x + w[0] * framed", "y = w[0] * framed"),
    "cache_ignored": ("prev = zero if cache is None else", "prev = zero if True else"),
    "next_frame_from_cache": ("framed = np.concatenate([prev, x, zero], axis=1)",
                              "framed = np.concatenate([prev, x, prev], axis=1)"),
    "centre_tap_shifted": ("w[1] * framed[:, 1:T + 1]", "w[1] * framed[:, 2:T + 2]"),
    "bias_dropped": ("y = y + np.asarray(bias, dtype=np.float64)", "y = y + 0.0"),
    "cache_is_first_frame": ("return y, x[:, T - 1].copy()", "return y, x[:, 0].copy()"),
}


@pytest.mark.parametrize("name", sorted(TCONV_MUTANTS))
def test_tconv_pins_reject_mutant(name, monkeypatch):
    old, new = TCONV_MUTANTS[name]
    pins = _load("test_oracle_tconv.py")
    mutant = _mutant_function(tconv.temporal_conv, old, new)
    monkeypatch.setattr(tconv, "temporal_conv", mutant)
    calls = [pins.test_hand_worked_case, pins.test_matches_scipy_correlation,
             pins.test_zero_initialised_conv_is_the_identity, pins.test_blocks_versus_whole_sequence,
             pins.test_causality_across_blocks, pins.test_channels_and_positions_are_independent,
             pins.test_golden_two_block_chain]
    calls += [lambda T=T, c=c, b=b: pins.test_matches_loops(T, c, b)
              for T in (1, 2, 5) for c, b in ((False, False), (True, False), (True, True))]
    assert _any_fails(calls), name + " passed every pin"


CROSS_MUTANTS = {
    "no_relu_q": ("q = np.maximum(np.asarray(q, dtype=np.float64), 0.0)",
                  "q = np.asarray(q, dtype=np.float64)"),
    "no_relu_k": ("k = np.maximum(np.asarray(k, dtype=np.float64), 0.0)",
                  "k = np.asarray(k, dtype=np.float64)"),
    "state_transposed": ('np.einsum("bhia,bhac->bhic", q, S)', 'np.einsum("bhia,bhca->bhic", q, S)'),
    "z_from_values": ("z = k.sum(axis=2)", "z = v.sum(axis=2)"),
    "no_eps": ("den = np.einsum(\"bhia,bha->bhi\", q, z) + eps",
               "den = np.einsum(\"bhia,bha->bhi\", q, z)"),
    "gate_sign": ("out = out / (1.0 + np.exp(-np.asarray(g, dtype=np.float64)))",
                  "out = out / (1.0 + np.exp(np.asarray(g, dtype=np.float64)))"),
}


@pytest.mark.parametrize("name", sorted(CROSS_MUTANTS))
def test_cross_pins_reject_mutant(name, monkeypatch):
    old, new = CROSS_MUTANTS[name]
    oracle.build()
    pins = _load("test_oracle.py")
    mutant = _mutant_function(oracle.cross_forward, old, new)
    monkeypatch.setattr(oracle, "cross_forward", mutant)
    calls = [pins.test_cross_matches_bruteforce_with_gate,
             pins.test_cross_with_equal_lengths_is_the_self_attention_oracle,
             pins.test_cross_closed_forms, pins.test_cross_golden_worked_example]
    assert _any_fails(calls), name + " passed every pin"


def test_the_harness_passes_the_real_oracles(monkeypatch):
    # control: the same calls against the unmutated functions all pass
    pins = _load("test_oracle_tconv.py")
    monkeypatch.setattr(tconv, "temporal_conv",
                        _mutant_function(tconv.temporal_conv, "y = x + w[0] * framed",
                                         "y = x + w[0] * framed"))
    assert not _any_fails([pins.test_hand_worked_case, pins.test_matches_scipy_correlation,
                           pins.test_blocks_versus_whole_sequence,
                           lambda: pins.test_matches_loops(5, True, True)])
    oracle.build()
    cross = _load("test_oracle.py")
    monkeypatch.setattr(oracle, "cross_forward",
                        _mutant_function(oracle.cross_forward, "z = k.sum(axis=2)",
                                         "z = k.sum(axis=2)"))
    assert not _any_fails([cross.test_cross_matches_bruteforce_with_gate,
                           cross.test_cross_with_equal_lengths_is_the_self_attention_oracle,
                           cross.test_cross_closed_forms])
