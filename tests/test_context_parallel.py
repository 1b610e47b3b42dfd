"""Context-parallel prefill (tokens of every sequence split over ranks, one exchange step).

CPU: two and four `gloo` ranks run state_space_model_04_b200.context.prefill_context_parallel -- the
same orchestration the GPUs run over NCCL -- with the steps (local state, fold, prefill)
done by the fp64 oracle, so the exchange itself (what is gathered, in which order, which
earlier ranks each rank folds) is checked against one whole-sequence oracle run.
The kernels of the steps are checked on the GPU in test_prefill_gpu.py, with the ranks
emulated in one process.
"""
import json
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# rank r holds tokens [split[r], split[r + 1]): uneven shards, none a multiple of the chunk
SPLITS = {2: [0, 250, 600], 4: [0, 100, 250, 430, 600]}


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class _OracleOps:
    """The three steps on CPU float64 tensors through the oracle (test infrastructure)."""

    @staticmethod
    def local_state(x, dt, A, B):
        import oracle
        xn, dtn, An, Bn = (t.numpy() for t in (x, dt, A, B))
        zeros = np.zeros_like(Bn)
        _, h = oracle.ssd_recurrence(xn, dtn, An, Bn, zeros, np.zeros_like(An), None)
        return torch.from_numpy(h), torch.from_numpy((dtn * An).sum(axis=1))

    @staticmethod
    def context_scan(rank, h_all, ld_all, h0):
        run = np.zeros(h_all.shape[1:]) if h0 is None else h0.numpy().copy()
        for q in range(rank):
            run = np.exp(ld_all[q].numpy())[:, :, None, None] * run + h_all[q].numpy()
        return torch.from_numpy(run)

    @staticmethod
    def prefill(x, dt, A, B, C, D, chunk, h0):
        import oracle
        y, h = oracle.ssd_recurrence(*(t.numpy() for t in (x, dt, A, B, C, D)), None if h0 is None else h0.numpy())
        return torch.from_numpy(y), torch.from_numpy(h)


def _worker(rank, world, port, out_dir, split):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from datetime import timedelta
    from ssd_inputs import make_prefill
    from state_space_model_04_b200.context import prefill_context_parallel
    dist.init_process_group("gloo", timeout=timedelta(seconds=60))
    c = make_prefill(2, split[-1], 4, 64, 16, 2, 64, "f32", h0_std=0.1, seed=77)
    lo, hi = split[rank], split[rank + 1]
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float64))
    y, h = prefill_context_parallel(t(c.x[:, lo:hi]), t(c.dt[:, lo:hi]), t(c.A), t(c.B[:, lo:hi]),
                                    t(c.C[:, lo:hi]), t(c.D), h0=t(c.h0), ops=_OracleOps)
    dist.destroy_process_group()
    np.save(os.path.join(out_dir, "y%d.npy" % rank), y.numpy())
    np.save(os.path.join(out_dir, "h%d.npy" % rank), h.numpy())


@pytest.mark.parametrize("world", [2, 4])
def test_gloo_ranks_context_parallel_prefill(world, tmp_path):
    import oracle
    from ssd_inputs import make_prefill
    split, port = SPLITS[world], _free_port()
    mp.start_processes(_worker, args=(world, port, str(tmp_path), split), nprocs=world, join=True,
                       start_method="spawn")
    c = make_prefill(2, split[-1], 4, 64, 16, 2, 64, "f32", h0_std=0.1, seed=77)
    y_ref, h_ref = oracle.ssd_recurrence(c.x, c.dt, c.A, c.B, c.C, c.D, c.h0)
    y = np.concatenate([np.load(tmp_path / ("y%d.npy" % r)) for r in range(world)], axis=1)
    np.testing.assert_allclose(y, y_ref, rtol=1e-9, atol=1e-9 * np.abs(y_ref).max())
    # every rank's state is the state after its own last token, not the sequence's
    for r in range(world):
        hi = split[r + 1]
        _, h_r = oracle.ssd_recurrence(c.x[:, :hi], c.dt[:, :hi], c.A, c.B[:, :hi], c.C[:, :hi], c.D, c.h0)
        np.testing.assert_allclose(np.load(tmp_path / ("h%d.npy" % r)), h_r, rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(np.load(tmp_path / ("h%d.npy" % (world - 1))), h_ref, rtol=1e-9, atol=1e-12)


def test_single_process_is_a_plain_prefill():
    """Without a process group the orchestration is one prefill with the given h0."""
    from ssd_inputs import make_prefill
    from state_space_model_04_b200.context import prefill_context_parallel
    import oracle
    c = make_prefill(1, 100, 2, 64, 16, 1, 64, "f32", h0_std=0.1, seed=78)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float64))
    y, h = prefill_context_parallel(t(c.x), t(c.dt), t(c.A), t(c.B), t(c.C), t(c.D), h0=t(c.h0), ops=_OracleOps)
    y_ref, h_ref = oracle.ssd_recurrence(c.x, c.dt, c.A, c.B, c.C, c.D, c.h0)
    np.testing.assert_array_equal(y.numpy(), y_ref)
    np.testing.assert_array_equal(h.numpy(), h_ref)
