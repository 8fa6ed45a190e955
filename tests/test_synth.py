"""The seeded input recipe (mixture_memories_layer_b200/synth.py) produces the
shapes, distributions and structure the workloads claim: it stands in for
the pages' public benchmarks, so its properties are checked, not assumed."""
import numpy as np
import pytest

from mixture_memories_layer_b200 import synth


def test_varlen_packing_follows_its_recipe():
    # lengths drawn U{512..2048} until the total is reached; the last one is
    # clipped to the remainder (and may fall below 512)
    w = synth.WORKLOADS["mom380m_skew_varlen"]
    cu = synth.make_cu_seqlens(w, np.random.default_rng(w.seed))
    lens = np.diff(cu)
    assert cu[0] == 0 and cu[-1] == w.varlen_total == 16384
    assert np.all(lens[:-1] >= 512) and np.all(lens <= 2048) and lens[-1] >= 1
    assert 8 <= len(lens) <= 32
    # same seed, same packing
    assert np.array_equal(cu, synth.make_cu_seqlens(w, np.random.default_rng(w.seed)))


@pytest.mark.parametrize("name", ["mom380m", "mom1p3b_m16"])
def test_fixed_length_batches(name):
    w = synth.WORKLOADS[name]
    cu = synth.make_cu_seqlens(w)
    assert np.array_equal(np.diff(cu), np.full(w.batch, w.seq_len))
    assert w.n_tokens == w.batch * w.seq_len


def test_weights_and_tokens_have_the_stated_distributions():
    w = synth.WORKLOADS["mom380m"]
    rng = np.random.default_rng(0)
    p = synth.make_weights(w, rng)
    Hd = w.heads * w.d_head
    shapes = {"w_r": (w.n_mem, w.d_model), "w_q": (Hd, w.d_model), "w_k_sh": (Hd, w.d_model),
              "w_v_sh": (Hd, w.d_model), "w_beta": (w.heads, w.d_model), "w_a": (w.heads, w.d_model),
              "w_k": (w.n_mem, Hd, w.d_model), "w_v": (w.n_mem, Hd, w.d_model)}
    for key, shape in shapes.items():
        assert p[key].shape == shape, key
    # N(0, 1/d_model) weights: sample std within 2 % of 1/sqrt(d_model)
    for key in ("w_q", "w_k", "w_v"):
        assert abs(p[key].std() * np.sqrt(w.d_model) - 1.0) < 0.02, key
    assert np.all((p["A"] >= 0) & (p["A"] <= 2.7)) and np.all((p["b_a"] >= -4) & (p["b_a"] <= 0))
    assert np.all(p["b_r"] == 0)
    x = synth.make_tokens(w, rng, 4096)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01
    # bf16 workloads hold bf16-representable values (both sides read the same numbers)
    assert np.array_equal(x, synth.bf16_round(x))
    assert np.array_equal(p["w_q"], synth.bf16_round(p["w_q"]))


def test_skewed_workload_biases_memory_zero_only():
    w = synth.WORKLOADS["mom380m_skew_varlen"]
    p = synth.make_weights(w, np.random.default_rng(w.seed))
    assert p["b_r"][0] == w.router_bias0 == 2.0 and np.all(p["b_r"][1:] == 0)


def test_decode_problem_layout():
    w = synth.small_workload(synth.WORKLOADS["decode_b256"], batch=4, prefill_len=8)
    p = synth.make_decode_problem(w, steps=3)
    assert p["x_prefill"].shape == (4 * 8, w.d_model)
    assert np.array_equal(p["cu_prefill"], np.arange(0, 5 * 8, 8))
    assert p["x_steps"].shape == (3, 4, w.d_model)
