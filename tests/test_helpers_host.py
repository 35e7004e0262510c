"""Host-side checks of the test metrics: the block-by-block comparison used
for the long workloads must give the same acceptance numbers as comparing the
whole tensor at once, so that splitting the oracle into channel blocks
changes nothing about what the parity tests accept."""
import numpy as np
import pytest

from .helpers import MAX_ABS_TOL, StreamedCompare, metrics


def _pair(seed, shape=(2, 300, 96)):
    rng = np.random.default_rng(seed)
    ref = rng.standard_normal(shape) * rng.uniform(0.01, 100.0, shape[-1])
    y = ref * (1 + 3e-3 * rng.standard_normal(shape))
    return y, ref


@pytest.mark.parametrize("block", [1, 7, 32, 96])
def test_streamed_compare_equals_whole_tensor_metrics(block):
    y, ref = _pair(0)
    cmp = StreamedCompare(ref.shape[-1])
    order = list(range(0, ref.shape[-1], block))[::-1]  # any order of blocks
    for c0 in order:
        cmp.add(y[..., c0:c0 + block], ref[..., c0:c0 + block], c0)
    rel, mabs, ch_mabs, ch_rel = cmp.result()
    rel_w, mabs_w = metrics(y, ref)
    assert rel == pytest.approx(rel_w, rel=1e-12)
    assert mabs == pytest.approx(mabs_w, rel=1e-12)
    for c in (0, 5, ref.shape[-1] - 1):
        r_c, m_c = metrics(y[..., c], ref[..., c])
        assert ch_rel[c] == pytest.approx(r_c, rel=1e-12)
        assert ch_mabs[c] == pytest.approx(m_c, rel=1e-12)


def test_streamed_compare_catches_a_bad_element_and_a_missing_block():
    y, ref = _pair(1)
    y[1, 123, 17] += 50.0 * np.sqrt(np.mean(ref ** 2))
    cmp = StreamedCompare(ref.shape[-1])
    for c0 in range(0, 96, 32):
        cmp.add(y[..., c0:c0 + 32], ref[..., c0:c0 + 32], c0)
    with pytest.raises(AssertionError):
        cmp.check("planted error")
    assert cmp.result()[1] > MAX_ABS_TOL
    partial = StreamedCompare(96)
    partial.add(ref[..., :64], ref[..., :64], 0)
    with pytest.raises(AssertionError):
        partial.result()
