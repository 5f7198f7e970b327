"""Sequence-parallel forward across ranks, its host logic on two gloo ranks (CPU).

Each rank holds one half of every sequence. The per-segment forward and the segment-state
scan are injected as fp64 CPU stand-ins (the oracle's forward; the scan S_{g+1} = A_g S_g
+ B_g written out), so the test checks what the library's orchestration does -- the zero
and identity inputs of the transition pass, the all-gather, the rank order, the entering
state each rank starts from -- against the oracle's forward over the whole sequence.
"""
import json
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from gated_delta_rule_wy_b200 import inputs as I
from gated_delta_rule_wy_b200.segments import gdr2_forward_sequence_parallel


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_forward(q, k, v, la, b, w, S0, final_state=True):
    """The fp64 oracle with the library forward's calling convention (scalar gates broadcast)."""
    n = lambda t: None if t is None else t.double().numpy()  # noqa: E731
    bb = n(b) if b.dim() == 4 else np.repeat(n(b)[..., None], q.shape[-1], axis=-1)
    ww = n(w) if w.dim() == 4 else np.repeat(n(w)[..., None], v.shape[-1], axis=-1)
    o, S_T = oracle.forward(n(q), n(k), n(v), n(la), bb, ww, S0=n(S0))
    return torch.from_numpy(o), (torch.from_numpy(S_T) if final_state else None), None


def _scan(A, Bst, S0):
    """S_starts[:, 0] = S0, S_starts[:, g + 1] = A_g S_starts[:, g] + B_g (fp64)."""
    A, Bst = A.double(), Bst.double()
    S = torch.zeros_like(Bst[:, 0]) if S0 is None else S0.double()
    starts = []
    for g in range(A.shape[1]):
        starts.append(S)
        S = A[:, g] @ S + Bst[:, g]
    return torch.stack(starts, 1), S


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x = I.make_forward_inputs(B=2, H=2, T=12, dk=4, dv=3, dtype=torch.float32, decay_shift=0.0, seed=131,
                                  with_S0=True)
        L = 12 // world
        part = lambda t: t[:, rank * L:(rank + 1) * L].contiguous()  # noqa: E731
        o, S_T = gdr2_forward_sequence_parallel(*(part(t) for t in (x.q, x.k, x.v, x.log_alpha, x.b, x.w)), x.S0,
                                                forward=_oracle_forward, segment_states=_scan)
        o_all, S_ref, _ = _oracle_forward(x.q, x.k, x.v, x.log_alpha, x.b, x.w, x.S0)
        res = {"o_err": float((o - part(o_all)).abs().max()), "S_err": float((S_T - S_ref).abs().max()),
               "o_scale": float(o_all.abs().max())}
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump(res, f)
    finally:
        dist.destroy_process_group()


def test_two_ranks_reproduce_the_whole_sequence(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_worker, args=(world, port, str(tmp_path)), nprocs=world, start_method="spawn")
    for r in range(world):
        res = json.loads((tmp_path / f"rank{r}.json").read_text())
        assert res["o_err"] <= 1e-12 * max(1.0, res["o_scale"]), res
        assert res["S_err"] <= 1e-12, res


def test_the_oracle_is_affine_in_the_entering_state():
    """What the segments rest on, checked on the fp64 oracle: the final state from any S0 is
    A S0 + B, A the final state from the identity with the write gate off, B from zero."""
    x = I.make_forward_inputs(B=1, H=2, T=9, dk=5, dv=3, dtype=torch.float32, decay_shift=0.0, seed=132)
    n = x.as_numpy64()
    _, B_ = oracle.forward(n["q"], n["k"], n["v"], n["log_alpha"], n["b"], n["w"])
    eye = np.broadcast_to(np.eye(5), (1, 2, 5, 5)).copy()
    _, A_ = oracle.forward(n["q"], n["k"], np.zeros(n["k"].shape), n["log_alpha"], n["b"], np.zeros(n["k"].shape),
                           S0=eye)
    S0 = np.random.default_rng(133).standard_normal((1, 2, 5, 3))
    _, S_T = oracle.forward(n["q"], n["k"], n["v"], n["log_alpha"], n["b"], n["w"], S0=S0)
    np.testing.assert_allclose(S_T, A_ @ S0 + B_, rtol=0, atol=1e-12)
