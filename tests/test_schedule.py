"""The per-layer and progressive sparsity policy (host only, no GPU)."""
import numpy as np
import pytest

from contextual_sparsity_lora_svd_b200 import synth
from contextual_sparsity_lora_svd_b200.schedule import (LayerRatios, ProgressiveSchedule,
                                                        llama2_7b_stack)


def test_llama2_stack_table_matches_the_workload_recipe():
    t = llama2_7b_stack()
    assert t.layers == 32
    for layer in range(32):
        assert (t.ffn[layer], t.qk[layer]) == pytest.approx(synth.stack_sparsity(layer))


def test_llama2_stack_table_shape():
    """Layers 0-3 dense; 4 starts at (0.5, 0.3); 31 ends at (0.9, 0.6); the
    ratios never fall with depth (deep layers tolerate more sparsity)."""
    t = llama2_7b_stack()
    assert t.ffn[:4] == (0.0,) * 4 and t.qk[:4] == (0.0,) * 4
    assert (t.ffn[4], t.qk[4]) == pytest.approx((0.5, 0.3))
    assert (t.ffn[31], t.qk[31]) == pytest.approx((0.9, 0.6))
    assert np.all(np.diff(t.ffn[4:]) > 0) and np.all(np.diff(t.qk[4:]) > 0)


def test_progressive_dense_first_tenth_then_table():
    sch = ProgressiveSchedule(llama2_7b_stack(), total_steps=1000)
    assert sch.dense_steps == 100
    assert all(r == (0.0, 0.0) for r in sch.ratios(0))
    assert all(r == (0.0, 0.0) for r in sch.ratios(99))
    full = sch.ratios(100)
    assert full == list(zip(sch.table.ffn, sch.table.qk))
    assert sch.ratios(999) == full
    assert sch.phases() == [(0, 100, 0.0), (100, 900, 1.0)]


def test_progressive_warmup_ramp():
    sch = ProgressiveSchedule(LayerRatios.uniform(2, 0.8, 0.4), total_steps=100, dense_frac=0.1,
                              warmup_frac=0.1)
    f = [sch.factor(s) for s in range(100)]
    assert f[:10] == [0.0] * 10
    np.testing.assert_allclose(f[10:20], np.arange(1, 11) / 10)
    assert f[20:] == [1.0] * 80
    assert sch.ratios(14)[1] == pytest.approx((0.8 * 0.5, 0.4 * 0.5))
    ph = sch.phases()
    assert sum(n for _, n, _ in ph) == 100 and ph[0] == (0, 10, 0.0) and ph[-1] == (20, 80, 1.0)


@pytest.mark.parametrize("bad", [dict(total_steps=0), dict(dense_frac=1.5),
                                 dict(warmup_frac=-0.1)])
def test_progressive_rejects_bad_arguments(bad):
    kw = dict(table=LayerRatios.uniform(1, 0.5, 0.5), total_steps=10)
    kw.update(bad)
    with pytest.raises(ValueError):
        ProgressiveSchedule(**kw)


def test_ratio_table_rejects_bad_values():
    with pytest.raises(ValueError):
        LayerRatios((0.5, 1.0), (0.1, 0.1))
    with pytest.raises(ValueError):
        LayerRatios((0.5,), (0.1, 0.1))
    with pytest.raises(ValueError):
        ProgressiveSchedule(LayerRatios.uniform(1, 0.5, 0.5), 10).factor(10)
