"""Host generator checks (CPU): published SplitMix64 outputs, distributions,
random access, recipes."""
import numpy as np
import pytest

from gen import counter_hash as ch
from gen import recipes


def test_splitmix64_published_stream_seed_zero():
    """SplitMix64 seeded with 0 (splitmix64.c): first three outputs."""
    got = [int(v) for v in ch.stream_outputs(0, 0, np.arange(3))]
    assert got == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_integer_values_uniform_in_range():
    v = ch.int_values(1, 3, 0, 90000)
    assert v.min() == -4 and v.max() == 4
    counts = np.bincount(v + 4)
    assert np.all(np.abs(counts - 10000) < 500)
    # stored as bf16 they are exact
    np.testing.assert_array_equal(ch.bf16_bits_to_f64(ch.int_bf16(1, 3, 0, 1000)), v[:1000])


def test_normal_values_moments_and_grid():
    v = ch.normal_values(7, 9, 0, 200000)
    assert abs(v.mean()) < 0.01 and abs(v.var() - 1.0) < 0.02
    assert np.all(np.abs(v) <= 6.0)
    assert np.all(v * 65536 == np.round(v * 65536))


def test_bf16_rounding_is_nearest_even():
    # 1 + 2^-8 lies halfway between bf16 neighbours 1 and 1 + 2^-7 -> even (1.0)
    x = np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 1.0 + 2 ** -8 + 2 ** -12])
    b = ch.f32_to_bf16_bits(x)
    np.testing.assert_array_equal(ch.bf16_bits_to_f64(b), [1.0, 1.0 + 2 ** -6, -1.0, 1.0 + 2 ** -7])


def test_random_access_matches_sequential():
    full = recipes.host_normal_tensor(3, recipes.tid(recipes.KIND_K, 2), (2, 50, 4, 8))
    rows = np.array([0, 17, 49])
    got = recipes.host_rows(3, recipes.tid(recipes.KIND_K, 2), (4, 8), rows, normal=True,
                            prefix_index=1, rows_total=50)
    np.testing.assert_array_equal(got, full[1, rows])
    fi = recipes.host_int_tensor(3, recipes.tid(recipes.KIND_K_IDX, 0), (1, 30, 16))
    gi = recipes.host_rows(3, recipes.tid(recipes.KIND_K_IDX, 0), (16,), np.array([29, 3]),
                           normal=False, prefix_index=0, rows_total=30)
    np.testing.assert_array_equal(gi, fi[0, [29, 3]])


def test_needle_pairs_are_valid():
    pairs = recipes.needle_pairs(recipes.PREFILL_64K)
    assert len(pairs) == 32
    ps = [p for p, _ in pairs]
    assert len(set(ps)) == 32
    assert all(0 <= p < t < recipes.PREFILL_64K.L for p, t in pairs)


def test_recipe_sizes():
    c5 = recipes.DECODE_1M
    kv_bytes = c5.n_layers * c5.Hkv * c5.D * 2 * 2 * c5.N
    assert kv_bytes / 2 ** 30 == 56.0
    assert recipes.GIST_128K.rows_cap == 64 * 17 + 16
    assert recipes.GIST_128K.Tk_max == 8192 * 17 + 16


def test_e4m3_codes_of_integers_and_rejections():
    """Integers in [-4, 4] have the E4M3 codes the format gives them (sign
    bit, exponent field e + 7, mantissa of |v| / 2^e - 1 in eighths); values
    E4M3 cannot hold exactly are rejected; the integer stream in E4M3 is the
    bf16 stream's values."""
    codes = ch.e4m3_codes(np.arange(-4, 5))
    assert [int(c) for c in codes] == [0xC8, 0xC4, 0xC0, 0xB8, 0x00, 0x38, 0x40, 0x44, 0x48]
    for bad in (4.25, 1000.0, 2.0 ** -10, 1.0625):
        with pytest.raises(ValueError):
            ch.e4m3_codes(np.array([bad]))
    ints = ch.int_values(5, 77, count=4096)
    np.testing.assert_array_equal(ch.int_e4m3(5, 77, count=4096), ch.e4m3_codes(ints))


def test_device_e4m3_conversion_matches_the_host_codes_on_cpu_tensors():
    """The conversion the fp8 workload's device inputs take (torch's E4M3
    cast of the integer bf16 tensor) gives the host generator's codes; the
    same check runs on the GPU in the parity tests."""
    import torch
    from gen import torch_inputs as TI
    bits = ch.int_bf16(13, 9, count=5000)
    t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
    np.testing.assert_array_equal(TI.to_e4m3(t).numpy(), ch.int_e4m3(13, 9, count=5000))
