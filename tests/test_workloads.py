"""The seeded input generator: determinism, bf16 rounding, needle planting."""
import numpy as np
import torch

import workloads


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32),
                        np.array([1.0, -1.0, 0.0, 1.00390625, 1.01171875, 3.0e-39], np.float32)])
    ours = workloads.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = workloads.bf16_bits_to_f32(ours)
    assert np.array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_generation_is_deterministic_and_row_independent():
    wl = workloads.small("t", B=3, H=2, L=40, g=4, w=4, d_c=16, d_r=8)
    a = workloads.generate(wl, threads=1)
    b = workloads.generate(wl, threads=3)
    for name in ("q_c", "q_r", "c_kv", "k_r"):
        assert np.array_equal(getattr(a, name), getattr(b, name))
    one = workloads.generate(wl.with_(B=1), threads=1)   # sequence 0 alone is the same stream
    assert np.array_equal(one.c_kv[0], a.c_kv[0])


def test_distribution_scales():
    wl = workloads.WORKLOADS["v2lite"].with_(B=1, L=4096)
    x = workloads.generate(wl, threads=1)
    c = workloads.bf16_bits_to_f32(x.c_kv)
    q = workloads.bf16_bits_to_f32(x.q_c)
    assert abs(c.std() - 1.0) < 0.02
    assert abs(q.std() * np.sqrt(576) - 1.0) < 0.05


def test_needles_are_planted():
    wl = workloads.WORKLOADS["needle"].with_(B=2, H=8, L=8192)
    x = workloads.generate(wl, threads=2)
    for b in range(2):
        pos = x.needle_pos[b]
        assert len(pos) == workloads.NEEDLES_PER_SEQ and np.all(np.diff(pos) > 0)
        rows = x.c_kv[b][pos]
        assert np.all(rows == rows[0])
        norm = np.linalg.norm(np.concatenate([workloads.bf16_bits_to_f32(rows[0]),
                                              workloads.bf16_bits_to_f32(x.k_r[b][pos[0]])]))
        assert abs(norm - 4 * 24.0) < 0.5


def test_registry_shapes():
    W = workloads.WORKLOADS
    assert (W["v2lite"].B, W["v2lite"].H, W["v2lite"].L, W["v2lite"].g, W["v2lite"].w) == (8, 16, 32768, 16, 1024)
    assert W["v2lite"].n_groups == 1984 and W["v2"].n_groups == 3968 and W["needle"].n_groups == 3968
    assert len(W["sweep"].sweep) == 10


def test_paged_layout_places_every_token_once():
    wl = workloads.small("paged", B=3, H=2, L=300, g=8, w=20, d_c=16, d_r=8, dtype="bf16", seed=5)
    x = workloads.generate(wl, threads=1)
    lens = [300, 65, 1]
    cache = workloads.paged_layout(x, lens, 64, seed=5, spare_pages=2)
    ps = cache.page_size
    owned = np.zeros(cache.c_pool.shape[0], bool)
    for b, L in enumerate(lens):
        need = -(-L // ps)
        pages = cache.block_table[b, :need]
        assert np.all((pages >= 0) & (pages < cache.num_pages))
        assert np.all(cache.block_table[b, need:] == -1)
        for t in (0, L // 2, L - 1):
            row = pages[t // ps] * ps + t % ps
            assert np.array_equal(cache.c_pool[row], x.c_kv[b, t])
            assert np.array_equal(cache.k_pool[row], x.k_r[b, t])
        rows = pages[:, None].astype(np.int64) * ps + np.arange(ps)[None]
        owned[rows.reshape(-1)[:L]] = True
    assert cache.num_pages == (5 + 2 + 1) + 2
    nan = workloads.nan_fill("bf16")
    assert np.all(cache.c_pool[~owned] == nan) and np.all(cache.k_pool[~owned] == nan)
    assert not np.any(cache.c_pool[owned] == nan)
    again = workloads.paged_layout(x, lens, 64, seed=5, spare_pages=2)
    assert np.array_equal(again.block_table, cache.block_table)
