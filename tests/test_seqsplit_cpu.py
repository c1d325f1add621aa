"""The sequence-split exchange (structured_state_space_mamba_b200.seqsplit) as
2 and 3 gloo ranks on the CPU: each rank takes a contiguous slice of the
sequence, the oracle stands in for the per-rank scan, and the stitched outputs
and every rank's final state must equal the oracle's recurrence over the whole
sequence (fp64, 1e-12).  No GPU: this checks the exchange step itself."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from structured_state_space_mamba_b200.inputs import make_inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_scan(x, dt, A, B, C, D, chunk_len, h0):
    import oracle
    y, f = oracle.ssd_recurrent(x.numpy(), dt.numpy(), A.numpy(), B.numpy(), C.numpy(),
                                D=None if D is None else D.numpy(), h0=None if h0 is None else h0.numpy(),
                                nthreads=1)
    return torch.from_numpy(y), torch.from_numpy(f)


def _worker(rank, world, port, cuts, with_h0, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from structured_state_space_mamba_b200.seqsplit import forward_sequence_split
        inp = make_inputs(2, cuts[-1], 3, 4, 5, 1, cuts[-1], dtype="f32", seed=61, init_state=with_h0, h0_std=0.5)
        t0, t1 = cuts[rank], cuts[rank + 1]
        T = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(torch.float64)  # noqa: E731
        y, fin = forward_sequence_split(
            _oracle_scan, T(inp.x[:, t0:t1]), T(inp.dt[:, t0:t1]), T(inp.A), T(inp.B[:, t0:t1]),
            T(inp.C[:, t0:t1]), D=T(inp.D), chunk_len=16, h0=None if inp.h0 is None else T(inp.h0))
        out[rank] = (y.numpy(), fin.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("cuts, with_h0", [([0, 23, 48], True), ([0, 10, 11, 40], False), ([0, 17, 30, 45], True)])
def test_sequence_split_matches_the_recurrence(oracle, cuts, with_h0):
    world = len(cuts) - 1
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, cuts, with_h0, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    inp = make_inputs(2, cuts[-1], 3, 4, 5, 1, cuts[-1], dtype="f32", seed=61, init_state=with_h0, h0_std=0.5)
    y_ref, f_ref = oracle.ssd_recurrent(inp.x, inp.dt, inp.A, inp.B, inp.C, D=inp.D, h0=inp.h0)
    y = np.concatenate([out[r][0] for r in range(world)], axis=1)
    scale = np.max(np.abs(y_ref))
    assert np.max(np.abs(y - y_ref)) <= 1e-12 * scale
    # every rank's final state is the state after its last token
    for r in range(world):
        _, f_r = oracle.ssd_recurrent(inp.x[:, :cuts[r + 1]], inp.dt[:, :cuts[r + 1]], inp.A,
                                      inp.B[:, :cuts[r + 1]], inp.C[:, :cuts[r + 1]], h0=inp.h0)
        assert np.max(np.abs(out[r][1] - f_r)) <= 1e-12 * max(np.max(np.abs(f_r)), 1e-30)
    assert np.max(np.abs(out[world - 1][1] - f_ref)) <= 1e-12 * np.max(np.abs(f_ref))
