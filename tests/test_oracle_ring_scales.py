"""Pins for the oracle's amax ring, scale rule, static values and export.

vLLM docs, "FP8 ViT encoder attention": a circular buffer of 16 observed
Q/K/V amax values drives the per-forward scale (usage section); calibration
runs 16 dynamic passes and saves the learned scales multiplied by the save
margin, default 1.5 (usage section); the scale file holds per-layer q/k/v
values such as 224/198/210 (scale file format section).
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from tests.fp_helpers import fl32_of_rational


def test_ring_holds_last_16_and_reduces_with_max():
    r = oracle.Ring()
    for v in range(1, 21):
        r.push(float(v))
    assert r.count == 16
    assert r.bound() == 20.0
    assert sorted(r.slots.tolist()) == [float(v) for v in range(5, 21)]
    assert r.head == 20 % 16


def test_ring_evicts_oldest():
    r = oracle.Ring()
    for v in range(20, 4, -1):          # 20, 19, ..., 5 : 16 pushes
        r.push(float(v))
    assert r.bound() == 20.0
    r.push(1.0)                         # evicts 20
    assert r.bound() == 19.0
    for _ in range(3):
        r.push(1.0)                     # evicts 19, 18, 17
    assert r.bound() == 16.0


def test_partial_ring_uses_only_filled_slots():
    r = oracle.Ring()
    assert r.bound() == 0.0
    r.push(3.0)
    r.push(2.0)
    assert r.count == 2 and r.bound() == 3.0


def test_empty_bound_gives_unit_scales():
    qs, ds = oracle.scales_from_bound(0.0)
    assert qs == 1.0 and ds == 1.0


@pytest.mark.parametrize("A", [224.0, 198.0, 210.0, 218.0, 195.0, 207.0, 3.7, 1e-3, 448.0, 1e6])
def test_scales_are_correctly_rounded_quotients(A):
    qs, ds = oracle.scales_from_bound(A)
    a = Fraction(float(np.float32(A)))
    assert qs == fl32_of_rational(Fraction(448) / a)
    assert ds == fl32_of_rational(a / Fraction(448))


def test_page_static_values(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "static_scale_file.json")))
    cf = g["closed_forms"]
    qs, ds = oracle.scales_from_bound(224.0)
    assert (qs, ds) == (cf["q_224"]["qs"], cf["q_224"]["ds"])
    qs, ds = oracle.scales_from_bound(210.0)
    assert ds == cf["v_210"]["ds"]
    assert qs == fl32_of_rational(Fraction(*cf["v_210"]["qs_rational"]))
    qs, ds = oracle.scales_from_bound(198.0)
    assert ds == fl32_of_rational(Fraction(*cf["k_198"]["ds_rational"]))
    assert qs == fl32_of_rational(Fraction(*cf["k_198"]["qs_rational"]))


def test_dynamic_step_is_current_inclusive():
    # first pass on an empty ring: the scale comes from the pass's own amax
    r = oracle.Ring()
    qs, ds = r.dynamic_step(3.5)
    assert ds == fl32_of_rational(Fraction(7, 2) / 448)
    assert qs == 128.0
    # a larger amax later dominates immediately
    qs, ds = r.dynamic_step(7.0)
    assert qs == 64.0


def test_nonfinite_amax_leaves_ring_unchanged():
    r = oracle.Ring()
    r.dynamic_step(2.0)
    qs, ds = r.dynamic_step(float("inf"), nonfinite=True)
    assert r.count == 1 and r.bound() == 2.0
    assert qs == 224.0
    r2 = oracle.Ring()
    qs, ds = r2.dynamic_step(float("inf"), nonfinite=True)
    assert r2.count == 0 and (qs, ds) == (1.0, 1.0)


def test_export_applies_margin_once():
    r = oracle.Ring()
    for _ in range(16):
        r.push(3.0)
    assert r.export_value() == 4.5
    assert r.export_value(2.0) == 6.0
    r = oracle.Ring()
    for v in [1.0, 149.0, 2.0]:
        r.push(v)
    assert r.export_value() == fl32_of_rational(Fraction(149) * Fraction(3, 2))


def test_selector_examples(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "selectors.json")))
    for c in g["cases"]:
        assert oracle.parse_selector(c["text"], c["max_index"]) == set(c["expect"])
    for c in g["invalid"]:
        with pytest.raises(ValueError):
            oracle.parse_selector(c["text"], c["max_index"])
    assert oracle.parse_selector("", 5) == set()
    assert oracle.parse_selector(" 1 , 3 - 4 ", 5) == {1, 3, 4}


def test_layer_modes():
    skip = oracle.parse_selector("0-2", 24)
    assert oracle.layer_mode(0, skip, False) == oracle.SKIP
    assert oracle.layer_mode(3, skip, False) == oracle.DYNAMIC
    assert oracle.layer_mode(3, skip, True) == oracle.STATIC
    assert oracle.layer_mode(2, skip, True) == oracle.SKIP


def test_step_and_layer_modes_follow_both_selectors():
    # vLLM-Omni parameters table: listed steps or layers skip FP8 attention;
    # the table's own examples, "0,1,4-6" for steps and "0-2,10" for layers
    steps = oracle.parse_selector("0,1,4-6", 50)
    layers = oracle.parse_selector("0-2,10", 24)
    for step in range(50):
        for layer in range(24):
            want_skip = step in (0, 1, 4, 5, 6) or layer in (0, 1, 2, 10)
            m = oracle.step_layer_mode(layer, step, layers, steps, False)
            assert m == (oracle.SKIP if want_skip else oracle.DYNAMIC), (step, layer)
            m = oracle.step_layer_mode(layer, step, layers, steps, True)
            assert m == (oracle.SKIP if want_skip else oracle.STATIC), (step, layer)
