"""The seeded input generator: deterministic, right shapes and value sets."""
import numpy as np

from sparse_attention_decode_relu_b200 import synth


def test_deterministic_and_independent_streams():
    a = synth.make_workload("a", L=500, T=2, key_dtype="fp8", recipe="normal", seed=4)
    b = synth.make_workload("b", L=500, T=2, key_dtype="fp8", recipe="normal", seed=4)
    for f in ("q", "q_idx", "w_idx", "k_idx", "k_scale", "pos"):
        assert np.array_equal(getattr(a, f), getattr(b, f)), f
    assert np.array_equal(a.kv, b.kv)
    c = synth.make_workload("c", L=900, T=2, key_dtype="fp8", recipe="normal", seed=4)
    assert np.array_equal(a.q, c.q) and np.array_equal(a.q_idx, c.q_idx)   # same stream, other L
    assert np.array_equal(a.kv, c.kv[:500])


def test_shapes_and_recipes():
    w = synth.config("tiny_decode")
    assert (w.L, w.T, w.key_dtype) == (4096, 1, "bf16") and w.pos.tolist() == [4095]
    assert w.q.shape == (1, 64, 128) and w.q.dtype == np.uint16
    assert w.kv.shape == (4096, 2, 4, 128) and w.k_scale is None
    qi = synth.bf16_bits_to_f32(w.q_idx)
    ki = synth.bf16_bits_to_f32(w.k_idx)
    assert set(np.unique(qi)) <= set(range(-3, 4)) and set(np.unique(ki)) <= set(range(-3, 4))
    assert set(np.unique(w.w_idx)) <= {0.0, 1.0, 2.0, 3.0}
    v = synth.config("verify_block")
    assert v.pos.tolist() == list(range(32760, 32768))
    twin = synth.config("long_decode_int")
    assert twin.k_idx.dtype == np.uint8 and set(np.unique(twin.k_scale)) <= {0.5, 1.0, 2.0}
    assert synth.config("sweep_L200_T8").pos.tolist() == list(range(192, 200))


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 3.0e38], np.float32)
    bits = synth.f32_to_bf16_bits(x)
    back = synth.bf16_bits_to_f32(bits)
    assert back.tolist()[:4] == [1.0, 1.0, 1.0 + 2 ** -6, -2.5]   # ties to even
    assert np.isfinite(back[4])


def test_planted_runs_do_not_overlap():
    rng = np.random.default_rng(0)
    for L in (4096, 1 << 20):
        starts = synth._planted_starts(L, rng)
        assert len(starts) == 32
        assert np.all(np.diff(starts) >= 64) and starts.min() >= 0 and starts.max() <= L - 8 - 64
