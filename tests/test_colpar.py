"""Column-parallel sharding, host side (no GPU): the channel ranges, the
all-gather that assembles whole rows (gloo ranks on CPU, world sizes 2 and 3,
uneven shards), and the premise of the split pinned in the oracle: a shard's
round-to-nearest codes and scales are the full layer's for its channels, and
the layer on a shard gives exactly the full layer's columns."""
import os
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

from oracle import spear_oracle as O
from w4_gemm_gated_b200 import colpar, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("N,world", [(4096, 1), (4096, 2), (11008 - 11008 % 256, 3), (768, 2), (14336, 8)])
def test_column_ranges_cover_aligned_balanced(N, world):
    r = colpar.column_ranges(N, world)
    assert len(r) == world and r[0][0] == 0 and r[-1][1] == N
    for (a0, a1), (b0, _) in zip(r, r[1:]):
        assert a1 == b0
    widths = [n1 - n0 for n0, n1 in r]
    assert all(w > 0 and w % colpar.ALIGN == 0 for w in widths)
    assert max(widths) - min(widths) <= colpar.ALIGN


def test_column_ranges_reject():
    with pytest.raises(ValueError):
        colpar.column_ranges(4000, 2)       # not a multiple of 256
    with pytest.raises(ValueError):
        colpar.column_ranges(512, 3)        # fewer 256-channel blocks than ranks
    with pytest.raises(ValueError):
        colpar.column_ranges(512, 0)


def _gather_worker(rank, world, port, N, out):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from w4_gemm_gated_b200 import colpar as C
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        M = 5
        n0, n1 = C.column_ranges(N, world)[rank]
        # element (m, n) of the whole output is 1000 m + n: each rank holds its columns
        rows = torch.arange(M, dtype=torch.float32)[:, None] * 1000.0
        part = rows + torch.arange(n0, n1, dtype=torch.float32)[None, :]
        y = C.gather_columns(part, N)
        want = rows + torch.arange(N, dtype=torch.float32)[None, :]
        out[rank] = bool(torch.equal(y, want))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("N,world", [(1024, 2), (768, 2), (1280, 3)])
def test_gather_columns_on_gloo_ranks(N, world):
    port = 29700 + (os.getpid() % 200) + N % 97 + world
    with mp.Manager() as man:
        out = man.dict()
        mp.spawn(_gather_worker, args=(world, port, N, out), nprocs=world, join=True)
        res = dict(out)
    assert res == {p: True for p in range(world)}


@pytest.mark.parametrize("group", [0, 128])
def test_shard_premise_in_the_oracle(group):
    # quantisation is per output channel (and per 128-row group along K), so a
    # shard's codes and scales are the full layer's; the layer on the shard is
    # the full layer's columns
    M, K, N, r = 3, 256, 768, 16
    L = synth.make_layer(M, K, N, r, b_g=-0.5, seed=77)
    q, s = O.quantize_rtn(L.W, group)
    y, g = O.linear(L.x, q, s, group, L.A, L.B, L.w_g, L.b_g)
    for n0, n1 in colpar.column_ranges(N, 2):
        qs, ss = O.quantize_rtn(np.ascontiguousarray(L.W[:, n0:n1]), group)
        assert np.array_equal(qs, q[n0:n1])            # q is N x K
        assert np.array_equal(ss, s[..., n0:n1])       # s is [N] or [K/128, N]
        ys, gs = O.linear(L.x, qs, ss, group, L.A, np.ascontiguousarray(L.B[:, n0:n1]), L.w_g, L.b_g)
        np.testing.assert_allclose(ys, y[:, n0:n1], rtol=1e-12, atol=1e-12 * np.max(np.abs(y)))
        np.testing.assert_array_equal(gs, g)
