"""The seeded input generator shared by the CUDA path's tests, the bench and the
oracle: determinism, storage rounding and the stated distributions."""
import numpy as np
import pytest
import torch

from post_weight_quantization_20_b200 import synthetic as S


def test_bytes_do_not_depend_on_thread_count():
    a = S.gen_activations(20000, 48, S.F16, S.ActSpec(mix_rank=3), seed=5, tag=2, threads=1)
    b = S.gen_activations(20000, 48, S.F16, S.ActSpec(mix_rank=3), seed=5, tag=2, threads=4)
    assert np.array_equal(a.view(np.uint16), b.view(np.uint16))
    w1 = S.gen_weight(300, 2000, S.BF16, S.WeightSpec(outlier_frac=0.01), seed=5, threads=1)
    w3 = S.gen_weight(300, 2000, S.BF16, S.WeightSpec(outlier_frac=0.01), seed=5, threads=3)
    assert np.array_equal(w1, w3)


def test_chunks_are_seeded_by_position():
    # the first CHUNK tokens do not depend on how many tokens follow
    short = S.gen_activations(S.CHUNK, 32, S.F32, S.ActSpec(), seed=9)
    long = S.gen_activations(2 * S.CHUNK + 5, 32, S.F32, S.ActSpec(), seed=9)
    assert np.array_equal(short, long[:S.CHUNK])
    other = S.gen_activations(S.CHUNK, 32, S.F32, S.ActSpec(), seed=9, tag=1)
    assert not np.array_equal(short, other)


def test_bf16_rounding_is_round_to_nearest_even():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(100000) * np.exp(rng.uniform(-20, 20, 100000))).astype(np.float32)
    bits = S.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bits, ref)
    # exact ties go to the even neighbour
    ties = np.array([0x3F808000, 0x3F818000, 0xBF808000], dtype=np.uint32).view(np.float32)
    assert S.f32_to_bf16_bits(ties).tolist() == [0x3F80, 0x3F82, 0xBF80]
    # widening is exact
    assert np.array_equal(S.f32_to_bf16_bits(S.bf16_bits_to_f32(bits)), bits)


def test_student_t4_quantile():
    t = S._student_t4(np.random.Generator(np.random.PCG64(3)), 2_000_000)
    # two-sided 95% point of Student's t with 4 degrees of freedom: 2.7764
    frac = np.mean(np.abs(t) > 2.7764)
    assert abs(frac - 0.05) < 1.5e-3
    assert abs(np.median(t)) < 5e-3


def test_outlier_channels_and_weight_outliers():
    spec = S.ActSpec(dist="normal", outlier_frac=0.05, outlier_mult=20.0)
    X = S.gen_activations(20000, 200, S.F32, spec, seed=4)
    idx = S.outlier_channels(200, spec, seed=4, tag=0)
    assert len(idx) == 10
    sd = X.std(axis=0)
    rest = np.setdiff1d(np.arange(200), idx)
    assert np.allclose(sd[idx] / sd[rest].mean(), 20.0, rtol=0.05)
    W = S.gen_weight(400, 500, S.F32, S.WeightSpec(sigma=0.02, outlier_frac=0.01, outlier_mult=8.0),
                     seed=4)
    big = np.abs(W) > 0.02 * 4.5      # a N(0, 0.02^2) entry exceeds 4.5 sigma with p ~ 7e-6
    assert abs(big.mean() - 0.01 * 0.57) < 1.5e-3   # P(|N(0, 8^2)| > 4.5) = 0.574


def test_low_rank_mix_correlates_channels():
    plain = S.gen_activations(8000, 40, S.F32, S.ActSpec(dist="normal", outlier_frac=0.0), seed=6)
    mixed = S.gen_activations(8000, 40, S.F32,
                              S.ActSpec(dist="normal", outlier_frac=0.0, mix_rank=2), seed=6)

    def mean_abs_corr(x):
        c = np.corrcoef(x.T)
        return np.abs(c[~np.eye(len(c), dtype=bool)]).mean()

    assert mean_abs_corr(plain) < 0.02
    assert mean_abs_corr(mixed) > 0.1


@pytest.mark.parametrize("dtype", S.DTYPES)
def test_to_f64_is_exact_widening(dtype):
    X = S.gen_activations(100, 16, dtype, S.ActSpec(), seed=8)
    x64 = S.to_f64(X, dtype)
    x32 = S.to_f32(X, dtype)
    assert x64.dtype == np.float64 and np.array_equal(x64, x32.astype(np.float64))


def test_a_token_range_equals_the_same_rows_of_one_call():
    spec = S.ActSpec(mix_rank=2)
    whole = S.gen_activations(3 * S.CHUNK + 17, 24, S.F16, spec, seed=3, tag=4)
    part = S.gen_activations(S.CHUNK + 17, 24, S.F16, spec, seed=3, tag=4,
                             first_token=2 * S.CHUNK)
    assert np.array_equal(part.view(np.uint16), whole[2 * S.CHUNK:].view(np.uint16))
    with pytest.raises(ValueError):
        S.gen_activations(10, 24, S.F16, spec, seed=3, first_token=5)
