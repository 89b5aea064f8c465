"""The seeded input generator: reproducible, prefix-consistent, and with the distributions its
docstring states (no layer arithmetic is involved)."""
import numpy as np

from group_wise_affine_qlinear_b200 import synthetic as S


def test_regeneration_is_byte_identical():
    w = S.WORKLOADS["tiny"]
    assert S.digest(w.x(), *w.w()) == S.digest(w.x(), *w.w())
    w8 = S.WORKLOADS["text_proj_w8"]
    assert S.digest(*S.weights8(3, 1, 16, 512)) == S.digest(*S.weights8(3, 1, 16, 512))
    assert w8.bits == 8


def test_leading_rows_equal_a_shorter_draw():
    """Rows come in 128-row Philox blocks: the first M rows of a draw of 300 rows are a draw of M rows."""
    full = S.activations(3, 0, 300, 256, block_means=True)
    for M in (1, 8, 32, 129):
        assert np.array_equal(S.activations(3, 0, M, 256, block_means=True), full[:M])


def test_weight_distributions():
    c, s, b = S.weights(1, 0, 64, 1024)
    sf, bf = s.astype(np.float64), b.astype(np.float64)
    assert c.dtype == np.uint32 and c.shape == (64, 128)
    assert np.all((sf >= 0.999e-3) & (sf <= 2.001e-2))
    assert np.all(np.abs(bf + 7.5 * sf) <= 0.6 * sf + 1e-3 * sf)          # -7.5 s + N(0, (0.1 s)^2), |z| < 6
    c8, s8, b8 = S.weights8(1, 0, 64, 1024)
    s8f, b8f = s8.astype(np.float64), b8.astype(np.float64)
    assert c8.shape == (64, 256)
    assert np.all((s8f >= 0.999e-3 / 17) & (s8f <= 2.001e-2 / 17))
    assert np.all(np.abs(b8f + 127.5 * s8f) <= 6 * 1.7 * s8f + 1e-2 * s8f)
    q8 = (c8[:, :, None] >> (8 * np.arange(4, dtype=np.uint32))) & 0xFF       # uniform codes over [0, 255]
    assert q8.min() == 0 and q8.max() == 255


def test_text_features_have_block_means():
    """13 channel blocks of 4096 with log-sigma means -1.5 + 0.25 b."""
    sig = S.channel_sigma(3, 0, 53248, block_means=True).astype(np.float64)
    means = np.log(sig).reshape(13, 4096).mean(axis=1)
    assert np.all(np.abs(means - (-1.5 + 0.25 * np.arange(13))) < 0.06)
