"""The sequence-sharded prefill's rank logic as gloo processes on the CPU.

Each rank holds one consecutive token range and runs ``prefill_sequence_sharded`` with
CPU stand-ins for the library calls (the prefill and the state fold computed by the
oracle and numpy, since these processes have no GPU): the ranges, the all_gather of the
ranges' states, the order of the fold and the hand-over of the incoming state are the
code under test.  Every rank's output and final state must equal the oracle's on the
whole sequence.  The CUDA calls themselves are checked on the GPU
(``test_gpu_state_init.py``).
"""

from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from chunked_causal_linear_b200.seqshard import part_ranges


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem(decay):
    rng = np.random.default_rng(5)
    B, H, T, d = 1, 2, 300, 8
    q, k, v = (rng.standard_normal((B, H, T, d)).astype(np.float32) * 0.5 for _ in range(3))
    gamma = [0.9, 0.97] if decay else None
    return q, k, v, gamma


def _fake_prefill(oracle, fm):
    def prefill(q, k, v, out, *, gamma, normalize, states_only=False, S_init=None, Z_init=None,
                **kw):
        o, S, Z = oracle.forward(q.numpy(), k.numpy(), v.numpy(), feature_map=fm, gamma=gamma,
                                 normalize=normalize,
                                 S_init=None if S_init is None else S_init.numpy(),
                                 Z_init=None if Z_init is None else Z_init.numpy(),
                                 want_out=not states_only)
        to = lambda a: torch.from_numpy(np.ascontiguousarray(a))
        return (None if states_only else to(o)), to(S), (to(Z) if normalize else None)
    return prefill


def _fake_combine(S_parts, Z_parts, upto, part_tokens, *, gamma):
    # P <- gamma^(tokens of part j) P + S_j over the parts before `upto`.
    H = S_parts.shape[2]
    g = np.ones(H) if gamma is None else np.asarray(gamma, dtype=np.float64)
    def fold(parts, extra):
        P = np.zeros(parts.shape[1:], dtype=np.float64)
        for j in range(upto):
            a = (g ** part_tokens[j]).reshape((1, H) + (1,) * extra)
            P = a * P + parts[j].numpy()
        return torch.from_numpy(P)
    return fold(S_parts, 2), (None if Z_parts is None else fold(Z_parts, 1))


def _worker(rank, world, port, decay, q_out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from chunked_causal_linear_b200 import ranks
    from chunked_causal_linear_b200.seqshard import prefill_sequence_sharded
    from oracle.oracle import default_oracle
    info = ranks.init(backend="gloo", timeout_s=60)
    q, k, v, gamma = _problem(decay)
    fm, norm = ("identity", False) if decay else ("elu1", True)
    rng = part_ranges(q.shape[2], world, chunk=64)
    s0, n = rng[rank]
    sl = lambda a: torch.from_numpy(np.ascontiguousarray(a[:, :, s0:s0 + n]))
    out, S_fin, Z_fin, _, _ = prefill_sequence_sharded(
        sl(q), sl(k), sl(v), info=info, part_tokens=[t for _, t in rng], gamma=gamma,
        normalize=norm, prefill=_fake_prefill(default_oracle(), fm), combine=_fake_combine)
    ranks.finish(info)
    q_out.put((rank, s0, n, out.numpy(), S_fin.numpy(),
               None if Z_fin is None else Z_fin.numpy()))


@pytest.mark.parametrize("decay", [False, True])
@pytest.mark.parametrize("world", [2, 3])
def test_sequence_sharded_ranks_reproduce_the_whole_sequence(world, decay):
    from oracle.oracle import default_oracle
    ctx = mp.get_context("spawn")
    qu = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, decay, qu)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted((qu.get(timeout=180) for _ in procs), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    q, k, v, gamma = _problem(decay)
    fm, norm = ("identity", False) if decay else ("elu1", True)
    o_ref, S_ref, Z_ref = default_oracle().forward(q, k, v, feature_map=fm, gamma=gamma,
                                                   normalize=norm)
    # Each range's output equals the whole run's on that range; the state after each
    # range equals the whole run's state at that token (checked at the sequence end).
    for rank, s0, n, out, S_fin, Z_fin in results:
        np.testing.assert_allclose(out, o_ref[:, :, s0:s0 + n], rtol=1e-10, atol=1e-12)
    _, _, _, _, S_last, Z_last = results[-1]
    np.testing.assert_allclose(S_last, S_ref, rtol=1e-10, atol=1e-12)
    if norm:
        np.testing.assert_allclose(Z_last, Z_ref, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("T,world,C", [(300, 2, 64), (300, 3, 64), (64, 4, 64), (1, 2, 64),
                                       (0, 3, 64), (1000, 8, 32)])
def test_part_ranges_cover_the_sequence_in_whole_chunks(T, world, C):
    r = part_ranges(T, world, C)
    assert len(r) == world
    pos = 0
    for start, n in r:
        assert start == pos and n >= 0
        pos += n
        if pos < T:
            assert n % C == 0  # only the last non-empty range may be ragged
    assert pos == T
