"""The seeded input generator: distribution, determinism and addressability."""
import numpy as np

import synthetic as syn


def test_weight_distribution_moments():
    x = syn.bf16_bits_to_f32(syn.host_bf16(1 << 20, 1001, 5, 0.02)).astype(np.float64)
    assert abs(x.mean()) < 1e-4
    assert abs(x.std() - 0.02) < 2e-4
    assert np.abs(x).max() < 6.1 * 0.02
    g = syn.bf16_bits_to_f32(syn.host_bf16(4096, 1001, 6, 0.0, 1.0))
    assert np.all(g == 1.0)


def test_elements_are_addressable_by_offset():
    full = syn.host_bf16(10000, 7, 3, 1.0)
    part = syn.host_bf16(100, 7, 3, 1.0, offset=4321)
    np.testing.assert_array_equal(part, full[4321:4421])
    assert not np.array_equal(syn.host_bf16(100, 7, 4, 1.0), full[:100])   # other tensor id
    assert not np.array_equal(syn.host_bf16(100, 8, 3, 1.0), full[:100])   # other seed


def test_kv_contents_depend_only_on_logical_position():
    cfg = syn.TINY
    a = syn.host_kv(cfg, 3001, 1, "k", 2, 0, 40)
    b = syn.host_kv(cfg, 3001, 1, "k", 2, 17, 23)
    np.testing.assert_array_equal(a[17:23], b)
    c = syn.host_kv(cfg, 3001, 1, "v", 2, 0, 40)
    assert not np.array_equal(a, c)


def test_tokens_pages_and_lengths():
    t = syn.host_tokens(1000, 2002, 128256)
    assert t.min() >= 0 and t.max() < 128256 and len(np.unique(t)) > 990
    perm = syn.page_permutation(8192, 3005)
    assert sorted(perm.tolist()) == list(range(8192)) and not np.array_equal(perm, np.arange(8192))
    lens = syn.ragged_lengths(64, 3004)
    assert lens.min() >= 512 and lens.max() <= 8192


def test_tensor_specs_pointer_order_and_bytes():
    specs = syn.tensor_specs(syn.LLAMA8B)
    assert specs[0].name == "tok_emb" and specs[-1].name == "lm_head"
    assert len(specs) == 1 + 9 * 32 + 2
    assert abs(syn.weight_bytes(syn.LLAMA8B) / 1e9 - 16.06) < 0.01
    moe = syn.tensor_specs(syn.MOE30B)
    assert len(moe) == 1 + 10 * 48 + 2
    assert len({s.tensor_id for s in moe}) == len(moe)
