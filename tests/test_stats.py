"""Host checks of the error/bias statistics (no GPU)."""
import numpy as np

from flashattention_bf16_fwd_b200.stats import bias_stats, lse_rel_err, max_rel_err, normwise_rel_err


def test_bias_stats_detects_planted_bias():
    rng = np.random.default_rng(0)
    ref = rng.standard_normal((4000, 64))
    noise = 1e-3 * rng.standard_normal(ref.shape)
    rows = np.ones(4000, bool)
    clean = bias_stats(ref + noise, ref, rows)
    assert abs(clean["z_mean"]) < 4 and abs(clean["z_aligned"]) < 4
    shrunk = bias_stats(ref * (1 - 2e-4) + noise, ref, rows)     # pulls every value toward 0
    assert shrunk["z_aligned"] < -5
    shifted = bias_stats(ref + 2e-4 + noise, ref, rows)
    assert shifted["z_mean"] > 5


def test_error_measures():
    ref = np.array([[1.0, -2.0], [0.5, 4.0]])
    x = ref + np.array([[0.1, 0.0], [0.0, -0.2]])
    assert abs(max_rel_err(x, ref) - 0.05) < 1e-12
    assert abs(normwise_rel_err(x, ref) - np.sqrt(0.05) / np.sqrt(1 + 4 + 0.25 + 16)) < 1e-12
    assert abs(lse_rel_err([0.0005, 10.01], [0.0, 10.0]) - 1e-3) < 1e-12


def test_normwise_floor_for_vanishing_gradients():
    ref = np.zeros((4, 64))
    assert normwise_rel_err(ref + 1e-8, ref) < 1e-4
    assert normwise_rel_err(ref + 1e-3, ref) >= 0.99
