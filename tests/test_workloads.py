"""The seeded input generator follows its stated recipe: N(0, 1) rows rounded
to the 16-bit format with ties to even, key outlier channels scaled by 20
(fixed in the tiny case, drawn once per workload otherwise and shared by every
row), value outlier tokens scaled by 10 (2 % of a batch row's tokens, shared
across its heads), the TurboQuant workloads' channel outliers on both K and V,
and the same arrays for the same seed.  CPU only."""
import numpy as np
import pytest

from quantized_kv_cache_18_b200 import workloads as W


def _f32(bits, dtype):
    return W.bits_to_float32(bits, dtype).astype(np.float64)


def test_rounding_to_16_bits_is_nearest_even():
    # bf16: 1 + 2^-8 is halfway between 1 and 1 + 2^-7 (ties to the even 1.0);
    # 1 + 3 * 2^-8 is halfway between 1 + 2^-7 and 1 + 2^-6 (ties to 1 + 2^-6)
    x = np.array([1 + 2**-8, 1 + 3 * 2**-8, 1 + 2**-8 + 2**-20, -2.5], np.float32)
    got = _f32(W.to_bits(x, "bf16"), "bf16")
    assert got.tolist() == [1.0, 1 + 2**-6, 1 + 2**-7, -2.5]
    y = np.array([1 + 2**-11, 1 + 3 * 2**-11, 65504.0], np.float32)
    assert _f32(W.to_bits(y, "fp16"), "fp16").tolist() == [1.0, 1 + 2**-9, 65504.0]


def test_tiny_key_outlier_channels_are_scaled():
    w = W.with_sizes(W.WORKLOADS["tiny"], seq_len=512)
    K, _ = W.prefill(w, seq_len=512)
    k = _f32(K, w.dtype)                                # [B][Hkv][S][d]
    std = k.reshape(-1, w.head_dim).std(axis=0)
    out = [3, 17]
    assert np.all(std[out] > 15) and np.all(std[out] < 25)
    rest = np.delete(std, out)
    assert np.all(rest > 0.85) and np.all(rest < 1.15)


@pytest.mark.parametrize("name", ["8b2", "70b"])
def test_drawn_key_outlier_channels_are_shared_by_every_row(name):
    w = W.with_sizes(W.WORKLOADS[name], batch=1, seq_len=1024)
    ch = W.k_outlier_channels(w)
    assert ch.size == w.n_k_outlier_channels and np.unique(ch).size == ch.size
    K, _ = W.prefill(w, seq_len=1024)
    k = _f32(K, w.dtype)
    for h in range(w.num_kv_heads):
        std = k[0, h].std(axis=0)
        assert np.all(std[ch] > 14)
        assert np.all(np.delete(std, ch) < 1.4)


def test_value_outlier_tokens_are_shared_across_heads():
    w = W.with_sizes(W.WORKLOADS["8b2"], batch=2, seq_len=2000)
    _, V = W.prefill(w, seq_len=2000)
    v = _f32(V, w.dtype)
    for b in range(w.batch):
        toks = W.v_outlier_tokens(w, b)
        assert toks.size == round(0.02 * w.seq_len)
        rms = np.sqrt((v[b] ** 2).mean(axis=2))      # [Hkv][S]
        for h in range(w.num_kv_heads):
            big = np.sort(np.argsort(rms[h])[-toks.size:])
            assert np.array_equal(big, np.sort(toks))
    assert not np.array_equal(W.v_outlier_tokens(w, 0), W.v_outlier_tokens(w, 1))


def test_turbo_workload_puts_channel_outliers_on_values_too():
    w = W.with_sizes(W.WORKLOADS["tq"], batch=1, seq_len=1024)
    ch = W.k_outlier_channels(w)
    _, V = W.prefill(w, seq_len=1024)
    std = _f32(V, w.dtype)[0, 0].std(axis=0)
    assert np.all(std[ch] > 14) and np.all(np.delete(std, ch) < 1.4)


def test_same_seed_same_inputs_and_rows_differ():
    w = W.with_sizes(W.WORKLOADS["tiny"], seq_len=256)
    K1, V1 = W.prefill(w, seq_len=256)
    K2, V2 = W.prefill(w, seq_len=256)
    assert np.array_equal(K1, K2) and np.array_equal(V1, V2)
    assert not np.array_equal(K1[0, 0], K1[0, 1])
    q1, q2 = W.query(w, 3), W.query(w, 3)
    assert np.array_equal(q1, q2) and not np.array_equal(q1, W.query(w, 4))
