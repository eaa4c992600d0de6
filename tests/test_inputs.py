"""The seeded input generators (shared by the tests, the benchmark and the smoke check).

* the torch evaluation of the draws, which makes the benchmark's large inputs, gives the
  numpy draws (up to the last fp64 bit of log/cos, i.e. a rare bf16 ulp);
* moving the slow mode of the bimodal a_k shifts exactly those draws and nothing else, so a
  workload with another slow mean is the same draw of every other tensor.
"""
import numpy as np
import pytest

from kv_cache_compression_ua_b200 import inputs as I


@pytest.mark.parametrize("name,slow_mean", [("decode_1b", -6.0), ("decode_1b", -20.0), ("prefill_1b", -6.0),
                                            ("fwdbwd_3b", -6.0)])
def test_torch_draws_equal_numpy_draws(name, slow_mean):
    w = I.WORKLOADS[name].resized(ak_slow_mean=slow_mean)
    a = I.make_prefill_inputs(w, T=96, B=2, b0=1)
    t = I.make_prefill_inputs_torch(w, "cpu", T=96, B=2, b0=1)
    assert set(a) == set(t)
    for n in a:
        got = t[n].float().numpy()
        assert got.shape == a[n].shape, n
        exact = np.mean(got == a[n])
        assert exact > 0.999, (n, exact)
        np.testing.assert_allclose(got, a[n], rtol=8e-3, atol=1e-6, err_msg=n)


def test_slow_mean_shifts_only_the_slow_draws():
    w0 = I.WORKLOADS["decode_1b"]
    w1 = w0.resized(ak_slow_mean=-20.0)
    a0 = I.make_prefill_inputs(w0, T=512, B=2, names=["k", "a_q", "a_k"])
    a1 = I.make_prefill_inputs(w1, T=512, B=2, names=["k", "a_q", "a_k"])
    np.testing.assert_array_equal(a0["k"], a1["k"])
    np.testing.assert_array_equal(a0["a_q"], a1["a_q"])
    slow = a0["a_k"] < -3.5                     # 5 standard deviations from either mode
    assert 0.05 < slow.mean() < 0.15
    np.testing.assert_array_equal(a1["a_k"][~slow], a0["a_k"][~slow])
    np.testing.assert_allclose(a1["a_k"][slow] - a0["a_k"][slow], -14.0, atol=1e-5)
    t0 = I.make_decode_token(w0, 3)
    t1 = I.make_decode_token(w1, 3)
    np.testing.assert_array_equal(t0["q"], t1["q"])
    sl = t0["a_k"] < -3.5
    np.testing.assert_array_equal(t1["a_k"][~sl], t0["a_k"][~sl])


def test_retention_matched_draw_is_the_calibrated_one():
    """The constant the benchmark uses is the one the committed calibration wrote, and that
    calibration reached the pages' 16k average compression (21.38 at p = 0.15)."""
    import json
    import os
    rec = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "decode_retention.json")))
    assert rec["ak_slow_mean"] == I.DECODE_RETAINED_AK_SLOW_MEAN
    assert rec["p"] == I.DECODE_RETAINED_P
    assert abs(rec["target_retention"] - 1 / 21.38) < 1e-12
    assert abs(rec["retention_at_that_mean"] / rec["target_retention"] - 1) < 0.02
