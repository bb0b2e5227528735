"""Checks of the seeded input generator and of the five workload shapes."""
import numpy as np
import pytest

from prefix_aware_decode_b200 import workload as wl


def test_streams_are_deterministic_and_distinct():
    a = wl.normal_bf16(1, 2, 3, 1000)
    b = wl.normal_bf16(1, 2, 3, 1000)
    c = wl.normal_bf16(1, 2, 4, 1000)
    assert np.array_equal(a, b)
    assert not np.array_equal(a, c)


def test_normal_moments():
    z = wl.normal_stream(42, 1, 0, 400_000)
    assert abs(z.mean()) < 0.01
    assert abs(z.std() - 1.0) < 0.01
    # tails roughly gaussian: P(|z| > 3) ~ 0.0027
    assert 0.0018 < np.mean(np.abs(z) > 3) < 0.0036


def test_bf16_rounding_is_rne_of_float():
    z = wl.normal_stream(5, 9, 0, 10_000).astype(np.float32)
    bits = wl.normal_bf16(5, 9, 0, 10_000)
    import torch
    ref = torch.from_numpy(z).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bits, ref)


def test_permutation_is_a_permutation():
    p = wl.permutation(3, 5, 1000)
    assert np.array_equal(np.sort(p), np.arange(1000))


def test_fill_pages_independent_of_threads():
    ids = np.array([3, 0, 2], dtype=np.int32)
    a = np.zeros((4, 2, 16, 8), dtype=np.uint16)
    b = np.zeros((4, 2, 16, 8), dtype=np.uint16)
    wl._gen().pagen_fill_pages(9, 1, ids.ctypes.data, 3, 2 * 16 * 8, a.ctypes.data, 1)
    wl._gen().pagen_fill_pages(9, 1, ids.ctypes.data, 3, 2 * 16 * 8, b.ctypes.data, 3)
    assert np.array_equal(a, b)
    assert (a[1] == 0).all()  # untouched page
    assert np.array_equal(a[2].ravel(), wl.normal_bf16(9, 1, 2, 2 * 16 * 8))


@pytest.mark.parametrize("config", [1, 2, 3, 4, 5])
def test_config_shapes(config):
    w = wl.make_config(config, with_values=False)
    spec = {1: (4, 8, 2, 64), 2: (64, 32, 8, 128), 3: (256, 32, 8, 128), 4: (128, 32, 8, 128),
            5: (512, 32, 8, 128)}[config]
    assert (w.B, w.Hq, w.Hkv, w.D) == spec
    assert w.P == 16
    used = np.concatenate([w.block_table[b, : -(-int(w.kv_lens[b]) // 16)] for b in range(w.B)])
    assert used.min() >= 0 and used.max() < w.num_pages
    # spare pages: about 5% of the used ones
    n_used = len(np.unique(used))
    assert w.num_pages - n_used == max(1, int(np.ceil(0.05 * n_used)))
    if config == 1:
        assert all(256 + 16 <= n <= 256 + 64 for n in w.kv_lens)
    if config == 2:
        assert all(2048 + 128 <= n <= 2048 + 1024 for n in w.kv_lens)
        assert 140e6 < w.unique_kv_bytes < 180e6
    if config == 3:
        assert all(4096 + 1024 + 64 <= n <= 4096 + 1024 + 2048 for n in w.kv_lens)
        # 8 branches of 32 requests each
        assert len({tuple(w.block_table[b, 256:320]) for b in range(w.B)}) == 8
    if config == 4:
        assert all(32 <= n <= 32768 for n in w.kv_lens)
        assert w.prefix_ratio == 0.0
        assert len(np.unique(used)) == len(used)
    if config == 5:
        assert all(32768 + 1 <= n <= 131072 + 1 for n in w.kv_lens)
        assert w.prefix_ratio > 0.99
        assert 9e9 < w.unique_kv_bytes < 12.5e9


def test_config1_values_and_poison():
    w = wl.make_config(1)
    assert w.q.shape == (4, 8, 64)
    nan = wl.BF16_NAN
    for b in range(w.B):
        n = int(w.kv_lens[b])
        last = w.block_table[b, (n - 1) // 16]
        tail = n % 16
        if tail:
            assert (w.k_pool[last, :, tail:, :] == nan).all()
            assert (w.v_pool[last, :, :tail, :] != nan).all()
    used = set(np.concatenate([w.block_table[b, : -(-int(w.kv_lens[b]) // 16)] for b in range(w.B)]).tolist())
    spare = [p for p in range(w.num_pages) if p not in used]
    assert spare and all((w.k_pool[p] == nan).all() for p in spare)
    # the shared root is the same physical pages for every request
    assert (w.block_table[:, :16] == w.block_table[0, :16]).all()


def test_config5_copy_on_write_tail():
    w = wl.make_config(5, scale=1 / 16)  # 2 sessions, shortened contexts
    assert w.B == 32
    for s in range(2):
        rows = range(16 * s, 16 * s + 16)
        n = int(w.kv_lens[16 * s])
        r = (n - 1) % 16
        pages = [w.block_table[b, (n - 1) // 16] for b in rows]
        assert len(set(pages)) == 16  # private pages
        if r:
            for p in pages[1:]:
                assert np.array_equal(w.k_pool[p, :, :r], w.k_pool[pages[0], :, :r])
        own = [w.k_pool[p, :, r].tobytes() for p in pages]
        assert len(set(own)) == 16  # each query's own token differs


def test_workload_is_reproducible():
    a = wl.make_config(1)
    b = wl.make_config(1)
    assert np.array_equal(a.block_table, b.block_table)
    assert np.array_equal(a.k_pool, b.k_pool) and np.array_equal(a.q, b.q)
    c = wl.make_config(1, seed=5)
    assert not np.array_equal(a.q, c.q)
