"""The seeded input generator: determinism, storage rounding, distributions."""
import numpy as np

from synth import CONFIGS, gen


def test_streams_are_deterministic_and_distinct():
    k1 = gen.stream_key(0, 2, gen.T_W1, 5)
    k2 = gen.stream_key(0, 2, gen.T_W1, 6)
    a = gen.raw_u64(k1, 1000)
    np.testing.assert_array_equal(a, gen.raw_u64(k1, 1000))
    assert not np.array_equal(a, gen.raw_u64(k2, 1000))
    # a window of a stream equals the tail of the full stream
    np.testing.assert_array_equal(gen.raw_u64(k1, 100, start=900), a[900:])


def test_chunked_stream_matches_scalar_definition():
    key = gen.stream_key(1, 2, 3)
    n = gen._CHUNK + 5
    u = gen.raw_u64(key, n)
    for i in (0, 1, gen._CHUNK - 1, gen._CHUNK, n - 1):
        assert int(u[i]) == gen._mix64_int(key + (i + 1) * gen.GOLDEN)


def test_bf16_storage_and_moments():
    cfg = CONFIGS[1]
    w = gen.make_expert_weight(cfg, 0, "w2", 3)
    assert w.shape == (cfg.d, cfg.f) and w.dtype == np.float32
    bits = w.view(np.uint32)
    assert np.all((bits & 0xFFFF) == 0)                 # bf16 values
    assert abs(w.std() * np.sqrt(cfg.f) - 1.0) < 0.01
    assert abs(w.mean()) < 1e-3
    b = gen.make_bias(cfg)
    assert b.dtype == np.float32 and b.min() >= -0.01 and b.max() <= 0.01


def test_quantile_table_symmetry():
    q = gen.normal_quantiles()
    np.testing.assert_allclose(q, -q[::-1], atol=1e-12)
    assert abs(q.mean()) < 1e-12 and abs(q.std() - 1.0) < 1e-3
