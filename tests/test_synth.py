"""The input generators: published SplitMix64 outputs, distribution shapes, and the VBQ
allocation statistics the pages report."""
import numpy as np

from cell_updates_b200 import synth


def test_splitmix64_published_outputs():
    # SplitMix64 started from state 0 (the first outputs of Vigna's reference generator)
    out = synth.mix64(np.arange(1, 4, dtype=np.uint64) * synth.GAMMA)
    assert [hex(int(v)) for v in out] == ["0xe220a8397b1dcdaf", "0x6e789e6aa1b965f4",
                                          "0x6c45d188009454f"]


def test_hashed_normal_moments():
    v = synth.hashed_normal_f32(7, synth.STREAM_WEIGHT, np.arange(1 << 20), 0.02).astype(np.float64)
    assert abs(v.mean()) < 1e-4 and abs(v.std() - 0.02) < 2e-4
    assert np.abs(v).max() <= 0.02 * np.sqrt(12.0) + 1e-6   # Irwin-Hall(4) support


def test_vbq_bits_follow_page_statistics():
    # VBQ abstract: 69% of groups at 1 bit; mean about 1.82 bits on the learned recipe
    b = synth.vbq_bits(262144, seed=2)
    frac1 = (b == 1).mean()
    assert abs(frac1 - 0.69) < 0.005
    assert abs(b.mean() - 1.79) < 0.02


def test_student_t_outliers():
    w = synth.student_t_weights(128, 1024, seed=1)
    assert w.dtype == np.float32 and w.shape == (128, 1024)
    assert np.abs(w).max() > 0.2
