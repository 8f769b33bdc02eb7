"""The counter-based synthetic KV generator: SplitMix64 against its published
first outputs for seed 0, and the stated value distribution."""
import numpy as np

from synthetic import TINY, DORY
from synthetic.kvgen import splitmix64, kv_rows, counter


def test_splitmix64_reference_outputs():
    # successive outputs of the SplitMix64 generator started from state 0
    gamma = np.uint64(0x9E3779B97F4A7C15)
    assert int(splitmix64(np.uint64(0))) == 0xE220A8397B1DCDAF
    assert int(splitmix64(gamma)) == 0x6E789E6AA1B965F4


def test_counter_fields_do_not_overlap():
    a = counter(0, 1, 0, 0, 0, 0, 0)
    b = counter(0, 0, 0, 0, 0, (1 << 20) - 1, 511)
    assert int(a) > int(b)
    assert int(counter(1, 63, 7, 4095, 63, (1 << 20) - 1, 511)) < 1 << 58


def test_kv_rows_distribution_and_bf16():
    K, V = kv_rows(DORY, 2, 3, 1, 0, 2, np.arange(4096))
    assert K.shape == (4096, DORY.head_dim)
    assert abs(np.mean(np.sum(K.astype(np.float64) ** 2, axis=1)) - 1) < 0.02
    assert abs(np.var(V.astype(np.float64)) * DORY.d - 1) < 0.02
    assert np.all((K.view(np.uint32) & 0xFFFF) == 0)       # BF16-exact
    K2, _ = kv_rows(DORY, 2, 3, 1, 0, 2, np.arange(4096))
    assert np.array_equal(K, K2)
    K3, _ = kv_rows(DORY, 2, 3, 1, 0, 3, np.arange(4096))   # other head
    assert not np.array_equal(K, K3)
