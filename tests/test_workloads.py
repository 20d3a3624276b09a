"""Input generators: the outlier-channel map used by the parity tests matches the tensors."""
import numpy as np

import workloads as wl


def test_outlier_scale_marks_the_scaled_channels():
    w = wl.WORKLOADS["cross_varlen_outliers_h32"]
    for which in "qkv":
        x = wl.make_tensor(w, which, tokens=512)
        s = wl.outlier_scale(w, which)
        assert s.shape == (w.heads, 128)
        assert set(np.unique(s).tolist()) == {1.0, w.outlier_gain}
        assert int((s == w.outlier_gain).sum()) == int(round(w.outlier_frac * w.heads * 128))
        rms = np.sqrt((x.astype(np.float64) ** 2).mean(axis=0))   # (heads, 128)
        # Outlier channels are ~64x the others: every marked channel exceeds every unmarked one.
        assert rms[s > 1].min() > 8 * rms[s == 1].max()


def test_outlier_scale_is_one_without_outliers():
    w = wl.WORKLOADS["dense_4x2048_h16"]
    assert np.all(wl.outlier_scale(w, "v") == 1.0)
