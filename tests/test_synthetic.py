"""The seeded input generator: reproducible, shaped like the pages' workloads."""
import numpy as np

from fp8_linear_layers_b200 import synthetic


def test_reproducible_and_tag_separated():
    a = synthetic.make_x(4, 256, seed=0, tag="X", outliers=3)
    b = synthetic.make_x(4, 256, seed=0, tag="X", outliers=3)
    c = synthetic.make_x(4, 256, seed=0, tag="Y", outliers=3)
    assert a.dtype == np.uint16 and np.array_equal(a, b) and not np.array_equal(a, c)


def test_outlier_channels_are_scaled():
    K = 4096
    x = synthetic.make_x(64, K, seed=0, outliers=synthetic.outlier_count(K))
    cols = synthetic.outlier_channels(64, K, seed=0, outliers=synthetic.outlier_count(K))
    assert len(cols) == 41
    xf = (x.astype(np.uint32) << 16).view(np.float32)
    rms = np.sqrt((xf.astype(np.float64) ** 2).mean(0))
    mask = np.zeros(K, bool)
    mask[cols] = True
    assert 15 < rms[mask].mean() < 25 and 0.8 < rms[~mask].mean() < 1.2


def test_weight_std():
    w = synthetic.make_w(512, 1024, seed=1)
    wf = (w.astype(np.uint32) << 16).view(np.float32)
    assert abs(wf.std() - 0.02) < 0.001


def test_shape_tables():
    assert sum(n * k for _, n, k in synthetic.LLAMA31_8B) == 218_103_808
    assert sum(n * k for _, n, k in synthetic.QWEN3_8B) == 192_937_984
