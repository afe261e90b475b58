"""Context-parallel prefill (gated_delta_rule_113_b200.context_parallel).

CPU: two and three gloo ranks run the real schedule and state exchange with
the fp64 oracle standing in for the per-segment compute; the concatenated
outputs and the last rank's state must equal the oracle on the whole
sequence.  GPU: the same schedule with the library's kernels, the ranks
emulated as threads of one process that hand states through queues (no
kernel waits on another), checked against the oracle.
"""
import math
import os
import queue
import sys
import threading

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _case(seed, T, H, Dk, Dv):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, H, Dk))
    k = rng.standard_normal((T, H, Dk))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H, Dv))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, H))))
    la = rng.uniform(math.log(0.8), 0.0, size=(T, H, Dk))
    S0 = 0.1 * rng.standard_normal((1, H, Dk, Dv))
    return q, k, v, la, beta, S0


def _oracle_forward(q, k, v, la, beta, S0, cu):
    """The fp64 oracle with the library forward's call shape (CPU tensors)."""
    sys.path.insert(0, ROOT)
    import oracle
    o, s = oracle.forward(q.numpy(), k.numpy(), v.numpy(), la.numpy(), beta.numpy(),
                          None if S0 is None else S0.numpy(), cu.numpy())
    return torch.from_numpy(o), torch.from_numpy(s)


def _rank_main(rank, world, port, bounds, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    from gated_delta_rule_113_b200.context_parallel import cp_prefill, torch_distributed_transport
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v, la, beta, S0 = (torch.from_numpy(x) for x in _case(7, bounds[-1], 5, 4, 3))
        a, b = bounds[rank], bounds[rank + 1]
        send, recv = torch_distributed_transport()
        out, sf = cp_prefill(q[a:b], k[a:b], v[a:b], la[a:b], beta[a:b],
                             S0 if rank == 0 else None, rank=rank, world=world, group_size=2,
                             send_state=send, recv_state=recv, forward=_oracle_forward,
                             state_dtype=torch.float64)
        results[rank] = (out.numpy(), None if sf is None else sf.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("bounds", [[0, 40, 97], [0, 30, 30, 71]])   # incl. an empty segment
def test_gloo_ranks_reproduce_the_whole_sequence(bounds):
    sys.path.insert(0, ROOT)
    import oracle
    world = len(bounds) - 1
    port = 29700 + os.getpid() % 500 + world
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        results = m.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, bounds, results))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=180)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        got = dict(results)
    q, k, v, la, beta, S0 = _case(7, bounds[-1], 5, 4, 3)
    o_ref, s_ref = oracle.forward(q, k, v, la, beta, S0=S0)
    out = np.concatenate([got[r][0] for r in range(world)])
    assert np.allclose(out, o_ref, rtol=1e-12, atol=1e-12)
    assert np.allclose(got[world - 1][1], s_ref, rtol=1e-12, atol=1e-12)


def test_head_groups_cover_every_head_once():
    sys.path.insert(0, ROOT)
    from gated_delta_rule_113_b200.context_parallel import head_groups
    assert head_groups(7, 3) == [(0, 3), (3, 6), (6, 7)]
    assert head_groups(4, 8) == [(0, 4)]
    with pytest.raises(ValueError):
        head_groups(4, 0)


@pytest.mark.gpu
def test_threaded_ranks_on_one_gpu_match_the_oracle():
    sys.path.insert(0, ROOT)
    import oracle
    from gated_delta_rule_113_b200.context_parallel import cp_prefill
    from gated_delta_rule_113_b200.inputs import WORKLOADS, forward_inputs
    from helpers import TOL_BF16, as_np, rel_fro
    inp = forward_inputs(WORKLOADS[1], lengths=[1500], H=6)
    bounds = [0, 512, 640, 1500]              # segment lengths 512, 128, 860
    world = len(bounds) - 1
    d = {n: inp[n].cuda() for n in ("q", "k", "v", "log_alpha", "beta")}
    S0 = inp["S0"].cuda()
    boxes = [queue.Queue() for _ in range(world)]   # boxes[r]: states sent to rank r

    def send(t, peer):
        boxes[peer].put(t.clone())

    def recv(t, peer):
        t.copy_(boxes[peer + 1].get(timeout=60))

    results, errors = {}, []

    def run(r):
        try:
            a, b = bounds[r], bounds[r + 1]
            results[r] = cp_prefill(*(d[n][a:b] for n in ("q", "k", "v", "log_alpha", "beta")),
                                    S0 if r == 0 else None, rank=r, world=world, group_size=4,
                                    send_state=send, recv_state=recv)
        except Exception as e:   # pragma: no cover - reported below
            errors.append(e)

    threads = [threading.Thread(target=run, args=(r,)) for r in range(world)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
    assert not errors, errors
    torch.cuda.synchronize()
    out = torch.cat([results[r][0] for r in range(world)])
    ro, rs = oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                            inp["S0"], inp["cu_seqlens"].numpy())
    assert rel_fro(as_np(out), ro) <= TOL_BF16
    assert rel_fro(as_np(results[world - 1][1]), rs) <= TOL_BF16


def test_group_size_rule():
    """Groups fill the GPU per call (about SMs / 4 heads at four chain CTAs per
    head) before the rank pipeline gets more of them; the busy fraction is
    G / (G + W - 1)."""
    from gated_delta_rule_113_b200.context_parallel import (busy_fraction, choose_group_size,
                                                            head_groups)
    # 32 heads (the long-context workloads) never fill 148 SMs: one group
    assert choose_group_size(32, 8) == 32
    assert busy_fraction(32, 32, 8) == 1 / 8
    # 128 heads on 148 SMs: four groups of 32 (each call 128 of 148 SMs)
    assert choose_group_size(128, 8) == 32
    assert busy_fraction(128, 32, 8) == 4 / 11
    # uneven head counts split into equal groups no larger than the fill size
    gs = choose_group_size(100, 4)
    assert gs <= 37 and len(head_groups(100, gs)) == 3
    assert choose_group_size(64, 1) == 64          # one rank: no pipeline to feed
    with pytest.raises(ValueError):
        choose_group_size(0, 2)
