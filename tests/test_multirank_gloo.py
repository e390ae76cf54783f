"""Multi-rank host logic of bench.py on CPU with gloo, world size 2.

The hot path shards by independent (batch, head) units, so N GPUs run N
replicas with no collective on the data path; the only cross-rank steps are
the barrier around the timed region and the max-over-ranks time."""
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_rank_reduction_and_reference_arm():
    from tests import _dist_worker
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_dist_worker.run, args=(r, 2, port, results)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        for p in procs:
            if p.is_alive():
                p.kill()
                pytest.fail("gloo worker did not finish")
            assert p.exitcode == 0
        res = dict(results)
    assert res[0]["max"] == res[1]["max"] == 2.5
    assert res[0]["seed"] != res[1]["seed"]
    assert res[1]["ref_stdout"] == ""
