"""Context sharding (CPU): partial softmax sums over slices of the context
and their exact merge, the slice partition, and the exchange between ranks
over gloo.

The oracle's slice partials are checked against the whole-sequence oracle
(itself pinned in oracle_pins.py): for any partition of the context on group
boundaries, merging the slices' (M, Z, O) with the online-softmax merge (the
Pulsar Attention page, "Fase 2") gives the whole decode, and the slices'
anchors concatenate to the whole anchors.  The two-rank test runs the
package's exchange (all-gather of the partial tensors) over gloo and merges
on every rank.
"""
import os
import socket
import sys

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle_pins as pins  # noqa: E402
import workloads  # noqa: E402
from kv_compression_b200.shard import exchange_partials, slice_bounds  # noqa: E402
from oracle import oracle as orc  # noqa: E402


def _inputs(seed, B=2, H=3, L=203, d_c=16, d_r=8, dtype="f32"):
    rng = np.random.default_rng(seed)
    return pins.rand_inputs(rng, B, H, L, d_c, d_r, dtype)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_partials_merge_to_the_whole(dtype):
    qc, qr, C, K = _inputs(40, dtype=dtype)
    L = C.shape[1]
    for (g, w) in ((4, 17), (8, 0), (1, 30), (16, 250), (5, 3)):
        whole = orc.lca(qc, qr, C, K, g=g, w=w)
        nG = orc.num_groups(L, g, w)
        win0 = nG * g
        cuts_options = [[], [win0], [g * (nG // 2)] if nG else [], [0, 0], [L, L],
                        sorted({g * (nG // 3), win0, min(L, win0 + 7)})]
        for cuts in cuts_options:
            b = [0] + cuts + [L]
            slices = [(b[i], b[i + 1] - b[i]) for i in range(len(b) - 1)]
            parts = [orc.partial(qc, qr, C, K, g, w, p0, n) for (p0, n) in slices]
            out = orc.merge(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]),
                            np.stack([p[2] for p in parts]))
            assert pins.rel_err(out, whole.out) < 1e-12, (g, w, cuts)
            anc = np.concatenate([p[3] for p in parts], axis=2)
            assert np.array_equal(anc, whole.anchor), (g, w, cuts)


def test_partial_refuses_a_cut_group():
    qc, qr, C, K = _inputs(41)
    with pytest.raises(RuntimeError):
        orc.partial(qc, qr, C, K, 4, 17, 6, 50)      # starts inside group 1


@pytest.mark.parametrize("L,g,w,parts", [(1000, 16, 100, 3), (100, 8, 200, 4), (130, 2, 3, 5),
                                         (65536, 16, 2048, 8), (7, 4, 0, 3)])
def test_slice_bounds_cover_the_context_on_group_boundaries(L, g, w, parts):
    sl = slice_bounds(L, g, w, parts)
    assert len(sl) == parts
    assert sl[0][0] == 0 and sum(n for _, n in sl) == L
    win0 = ((L - w) // g if L > w else 0) * g
    for i, (p0, n) in enumerate(sl):
        assert n >= 0
        if i:
            assert p0 == sl[i - 1][0] + sl[i - 1][1]
        if p0 < win0:
            assert p0 % g == 0


WORLD = 2


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, port: int, result_dir: str) -> None:
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=WORLD)
    try:
        wl = workloads.small("shard", B=2, H=3, L=300, g=8, w=40, d_c=16, d_r=8, dtype="f32", seed=5)
        x = workloads.generate(wl, threads=1)
        pos0, n = slice_bounds(wl.L, wl.g, wl.w, WORLD)[rank]
        m, z, o, anc = orc.partial(x.q_c, x.q_r, x.c_kv, x.k_r, wl.g, wl.w, pos0, n)
        mz = torch.from_numpy(np.stack([m, z], axis=-1))
        all_mz, all_o = exchange_partials(mz, torch.from_numpy(o))
        out = orc.merge(all_mz[..., 0].numpy(), all_mz[..., 1].numpy(), all_o.numpy())
        whole = orc.lca(x.q_c, x.q_r, x.c_kv, x.k_r, g=wl.g, w=wl.w)
        err = pins.rel_err(out, whole.out)
        with open(os.path.join(result_dir, f"rank{rank}.txt"), "w") as f:
            f.write(f"{err!r} {all_mz.shape[0]} {anc.shape[2]}\n")
    finally:
        dist.destroy_process_group()


def test_two_ranks_exchange_and_merge(tmp_path):
    mp.spawn(_rank_main, args=(_free_port(), str(tmp_path)), nprocs=WORLD, join=True)
    for r in range(WORLD):
        err, n, ng = open(tmp_path / f"rank{r}.txt").read().split()
        assert float(err) < 1e-12 and int(n) == WORLD
