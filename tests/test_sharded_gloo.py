"""The token- and row-sharded layer orchestration on two CPU ranks (gloo).

The orchestration (post_weight_quantization_07_b200.sharded) is run with the
float64 oracle as its compute steps: every rank computes H and D over its
token shard, the all-reduce sums them, and every rank quantises its row shard.
Gathered, the shards must reproduce the oracle run on the whole layer.
"""
import os
import socket

import numpy as np
import pytest

import oracle
from synthetic import random_layer_host

torch = pytest.importorskip("torch")
dist = pytest.importorskip("torch.distributed")
mp = pytest.importorskip("torch.multiprocessing")

from post_weight_quantization_07_b200.sharded import quantize_layer_sharded, shard_range  # noqa: E402

M, N, N_TOK, WBITS, G, DAMP, ALPHA = 48, 64, 600, 3, 16, 0.01, 0.5


def _terms(X, Xh):
    return torch.from_numpy(oracle.hessian(Xh)), torch.from_numpy(oracle.qep_cross(X, Xh))


def _finish(W, H, D, alpha, damp, wbits, groupsize, act_order):
    Wp = oracle.qep_correct(W, None, None, alpha, damp, H=H.numpy(), d=D.numpy())
    q = oracle.gptq_quantize(Wp, H.numpy(), wbits, groupsize, damp, act_order)
    return Wp, q


def _rank_main(rank, world, port, act_order, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        L = random_layer_host(M, N, N_TOK, seed=8100)
        t0, t1 = shard_range(N_TOK, rank, world)
        r0, r1 = shard_range(M, rank, world)
        W = L["W"].astype(np.float64)
        H, D, (Wp, q) = quantize_layer_sharded(W[r0:r1], L["X"][t0:t1], L["Xhat"][t0:t1], ALPHA, DAMP, WBITS,
                                               G, act_order, terms=_terms, finish=_finish)
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), H=H.numpy(), D=D.numpy(), Wp=Wp, codes=q["codes"],
                 scales=q["scales"], zeros=q["zeros"], rows=np.array([r0, r1]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("act_order", [False, True])
def test_sharded_layer_on_two_ranks_matches_whole_layer(tmp_path, act_order):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), act_order, str(tmp_path)), nprocs=world, join=True)
    L = random_layer_host(M, N, N_TOK, seed=8100)
    W = L["W"].astype(np.float64)
    Hw = oracle.hessian(L["Xhat"])
    Dw = oracle.qep_cross(L["X"], L["Xhat"])
    Wpw = oracle.qep_correct(W, L["X"], L["Xhat"], ALPHA, DAMP, H=Hw)
    ref = oracle.gptq_quantize(Wpw, Hw, WBITS, G, DAMP, act_order)
    seen = np.zeros(M, dtype=bool)
    for r in range(world):
        z = np.load(tmp_path / f"rank{r}.npz")
        # the all-reduced terms are the whole layer's (summation order aside)
        assert np.allclose(z["H"], Hw, rtol=1e-12, atol=1e-9 * np.abs(Hw).max())
        assert np.allclose(z["D"], Dw, rtol=1e-12, atol=1e-9 * np.abs(Dw).max())
        r0, r1 = z["rows"]
        seen[r0:r1] = True
        assert np.allclose(z["Wp"], Wpw[r0:r1], rtol=0, atol=1e-10 * np.abs(W).max())
        assert np.array_equal(z["codes"], ref["codes"][r0:r1])
        assert np.allclose(z["scales"], ref["scales"][r0:r1], rtol=1e-10, atol=0)
        assert np.array_equal(z["zeros"], ref["zeros"][r0:r1])
    assert seen.all()


def test_shard_range_covers_and_aligns():
    for total in (0, 1, 7, 64, 1000):
        for world in (1, 2, 3, 8):
            spans = [shard_range(total, r, world, align=4) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == total
            for (a, b), (c, d) in zip(spans, spans[1:]):
                assert b == c and a <= b
            assert all(a % 4 == 0 for a, _ in spans if a < total)
