"""Per-call mode selection in a denoising loop, through the C ABI, against
the oracle (vLLM-Omni docs, parameters table: kv_cache_skip_steps and
kv_cache_skip_layers; listed steps or layers keep the native dtype)."""
import numpy as np
import pytest

import oracle
import quantization_amax_reduce_b200 as qar

pytestmark = pytest.mark.gpu


def _mask(sel, n):
    m = np.zeros(n, np.uint8)
    m[sorted(sel)] = 1
    return m


def test_step_and_layer_modes_match_the_oracle():
    n_layers, n_steps = 24, 50
    ctx = qar.Context(n_layers)
    ctx.set_static_scales(7, 224.0, 198.0, 210.0)   # one layer with static bounds
    rng = np.random.default_rng(5)
    cases = [("0,1,4-6", "0-2,10")]
    for _ in range(20):
        s = sorted(set(rng.integers(0, n_steps, size=rng.integers(0, 6)).tolist()))
        l = sorted(set(rng.integers(0, n_layers, size=rng.integers(0, 6)).tolist()))
        cases.append((",".join(map(str, s)), ",".join(map(str, l))))
    for step_text, layer_text in cases:
        steps = qar.parse_selector(step_text, n_steps)
        layers = qar.parse_selector(layer_text, n_layers)
        assert steps == oracle.parse_selector(step_text, n_steps)
        assert layers == oracle.parse_selector(layer_text, n_layers)
        ms, ml = _mask(steps, n_steps), _mask(layers, n_layers)
        for step in range(n_steps):
            for layer in range(n_layers):
                got = ctx.select_mode_at_step(layer, step, ml, ms)
                want = oracle.step_layer_mode(layer, step, layers, steps, layer == 7)
                assert got == want, (step_text, layer_text, step, layer)
    # no step mask: the layer rule alone
    assert ctx.select_mode_at_step(3, 0, None, None) == qar.DYNAMIC
    assert ctx.select_mode_at_step(7, 0, None, None) == qar.STATIC
    with pytest.raises(qar.FP8AttnError):
        ctx.select_mode_at_step(0, n_steps, None, np.zeros(n_steps, np.uint8))
    with pytest.raises(qar.FP8AttnError):
        ctx.select_mode_at_step(n_layers, 0, None, None)
