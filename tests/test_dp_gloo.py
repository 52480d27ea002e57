"""The data-parallel exchange on CPU ranks (gloo, world size 2).

The per-rank compute is the float64 oracle on the rank's shard of token rows; the test
checks that the sharded result (global mean, summed dW, local dH rows) equals the oracle
on the whole batch, and that a rank that leaves before the exchange makes the other rank
fail with an error instead of waiting for ever.
"""

import os
import socket
import tempfile
from datetime import timedelta

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(kind):
    from lm_head_loss_streaming_b200 import synthetic
    return synthetic.make(kind, 37, 16, 53, w_std=0.3, ignore_frac=0.2, seed=5,
                          with_labels=True)


class _OracleRes:
    def __init__(self, f):
        self.loss_sum = torch.tensor([f["loss_sum"]], dtype=torch.float64)
        self.n_valid = torch.tensor([f["n_valid"]], dtype=torch.int64)


def _worker(rank, world, port, kind, outdir, mode):
    import sys
    sys.path.insert(0, ROOT)
    import oracle
    from lm_head_loss_streaming_b200 import dp

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=timedelta(seconds=20))
    try:
        inp = _inputs(kind)
        rows = np.array_split(np.arange(inp.N), world)[rank]
        sl = torch.from_numpy(rows)
        Hq, W = inp.Hq[sl], inp.W
        Hp = None if kind == "ce" else inp.Hp[sl]
        lab = inp.labels[sl]

        if mode == "leave" and rank == 1:
            raise SystemExit(0)  # leaves between steps, before the exchange

        def fwd():
            return _OracleRes(oracle.forward(kind, Hq, W, lab, Hp, inp.ignore_index))

        # Vocabulary-row sharding of dW (FSDP-style): the backward writes the first V rows
        # of a buffer padded to world * ceil(V / world) rows, which is reduce-scattered.
        V, d = W.shape
        dW_full = None
        if mode in ("shard", "fused_shard"):
            dW_full = torch.zeros(world * dp.shard_rows(V, world), d, dtype=torch.float64)

        def as_dW(dW):
            if dW_full is None:
                return torch.from_numpy(dW)
            dW_full[:V].copy_(torch.from_numpy(dW))
            return dW_full[:V]

        def bwd(res, n_valid_global):
            valid = (lab != inp.ignore_index).numpy()
            g = np.where(valid, 1.0 / max(int(n_valid_global.item()), 1), 0.0)
            dH, dW = oracle.backward(kind, Hq, W, lab, Hp, g, inp.ignore_index)
            if dW_full is not None:
                return torch.from_numpy(dH), as_dW(dW)
            if mode == "ready3":
                # The overlapped form's result: (dH, dW, ready); without an event or a
                # side stream the exchange runs in line.
                return torch.from_numpy(dH), torch.from_numpy(dW), None
            return torch.from_numpy(dH), torch.from_numpy(dW)

        def count():
            return torch.tensor([int((lab != inp.ignore_index).sum())], dtype=torch.int64)

        def fused(scale):
            # A single call whose gradient is that of the local mean, scaled by `scale`.
            res = fwd()
            n_local = max(int(res.n_valid.item()), 1)
            valid = (lab != inp.ignore_index).numpy()
            g = np.where(valid, float(scale.item()) / n_local, 0.0)
            dH, dW = oracle.backward(kind, Hq, W, lab, Hp, g, inp.ignore_index)
            return res, torch.from_numpy(dH), as_dW(dW)

        try:
            if mode in ("fused", "fused_shard"):
                r = dp.fused_fwd_bwd(count, fused, dW_full=dW_full)
            else:
                r = dp.fwd_bwd(fwd, bwd, dW_full=dW_full)
        except Exception as e:  # noqa: BLE001
            with open(os.path.join(outdir, f"err{rank}.txt"), "w") as f:
                f.write(type(e).__name__)
            return
        dw_rows = np.array(r.dW_rows if r.dW_rows is not None else (0, V))
        np.savez(os.path.join(outdir, f"rank{rank}.npz"), loss=r.loss_mean.numpy(),
                 n_valid=r.n_valid.numpy(), dH=r.dH.numpy(), dW=r.dW.numpy(), rows=rows,
                 dw_rows=dw_rows)
    finally:
        try:
            dist.destroy_process_group()
        except Exception:  # noqa: BLE001
            pass


@pytest.mark.parametrize("kind,mode", [("ce", "ok"), ("kl_div", "ok"), ("lk_hybrid", "ok"),
                                       ("kl_div", "ready3"), ("ce", "fused"),
                                       ("kl_div", "fused"), ("ce", "shard"),
                                       ("tv", "shard"), ("kl_div", "fused_shard")])
def test_two_rank_data_parallel_matches_whole_batch(kind, mode):
    import oracle
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_worker, args=(2, _free_port(), kind, d, mode), nprocs=2,
                           join=True, start_method="spawn")
        inp = _inputs(kind)
        Hp = None if kind == "ce" else inp.Hp
        ref = oracle.forward(kind, inp.Hq, inp.W, inp.labels, Hp, inp.ignore_index)
        rdH, rdW = oracle.backward(kind, inp.Hq, inp.W, inp.labels, Hp, None, inp.ignore_index)
        covered = []
        for rank in range(2):
            r = np.load(os.path.join(d, f"rank{rank}.npz"))
            assert int(r["n_valid"][0]) == ref["n_valid"]
            assert abs(float(r["loss"][0]) - ref["loss"]) <= 1e-12 * max(1.0, abs(ref["loss"]))
            if mode in ("shard", "fused_shard"):
                # Rank r holds vocabulary rows [r * Vs, (r + 1) * Vs) of the summed dW, the
                # rows past V being the zero padding.
                a, b = (int(x) for x in r["dw_rows"])
                Vs = r["dW"].shape[0]
                assert a == min(rank * Vs, inp.V) and b == min((rank + 1) * Vs, inp.V)
                covered.extend(range(a, b))
                tol = 1e-6 if mode == "fused_shard" else 1e-10
                assert np.abs(r["dW"][:b - a] - rdW[a:b]).max() <= tol * np.abs(rdW).max()
                assert not r["dW"][b - a:].any()
                assert np.abs(r["dH"] - rdH[r["rows"]]).max() <= tol * np.abs(rdH).max()
            elif mode == "fused":
                # The fused form passes its scale as the library's float32 grad_scale:
                # relative-to-max-norm agreement at float32 resolution.
                for got, want in ((r["dW"], rdW), (r["dH"], rdH[r["rows"]])):
                    assert np.abs(got - want).max() <= 1e-6 * np.abs(want).max()
            else:
                assert np.allclose(r["dW"], rdW, rtol=1e-10, atol=1e-14)
                assert np.allclose(r["dH"], rdH[r["rows"]], rtol=1e-10, atol=1e-14)
        if mode in ("shard", "fused_shard"):
            assert covered == list(range(inp.V))  # the shards tile the vocabulary once


def test_rank_that_leaves_makes_the_other_fail_not_hang():
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_worker, args=(2, _free_port(), "ce", d, "leave"), nprocs=2,
                           join=True, start_method="spawn")
        assert os.path.exists(os.path.join(d, "err0.txt"))
        assert not os.path.exists(os.path.join(d, "rank0.npz"))
