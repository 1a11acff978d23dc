"""Sequence sharding (seqshard.py) on CPU: gloo ranks each scan one segment of every
sequence, exchange the ShortConv history and the segment maps with all-gathers, and
rescan from their exact start state.  The two library operations (the scan and the
affine step S M + N) are supplied here by the fp64 oracle and numpy; the checks are
the host logic and the exchange: each rank's outputs and end state must equal the
oracle's scan of the whole, unsharded sequence to 1e-10."""
import datetime
import os
import socket
import sys

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


class OracleOps:
    """The library's two operations, restated by the oracle (fp64, CPU).  A ShortConv
    history (conv_state [B, H, W-1, d_v]) is fed to the oracle as W - 1 leading tokens
    that carry it in v and leave the state alone (gamma = 1; beta = alpha = 0; q, k, u,
    gain = 0); their outputs are dropped."""

    def scan(self, q, k, v, gamma, beta, u, alpha, gain, conv_w, L, S0, lengths, chain, chunk, conv_state=None):
        from oracle import prism_seq

        n = lambda t: None if t is None else t.double().numpy()
        h = 0 if conv_state is None else conv_state.shape[2]
        if h:
            def lead(x, fill):
                if x is None:
                    return None
                pad = torch.full((x.shape[0], h) + tuple(x.shape[2:]), fill, dtype=x.dtype)
                return torch.cat([pad, x], 1)
            q, k, u, gain = lead(q, 0.0), lead(k, 0.0), lead(u, 0.0), lead(gain, 0.0)
            gamma, beta, alpha = lead(gamma, 1.0), lead(beta, 0.0), lead(alpha, 0.0)
            v = torch.cat([conv_state.permute(0, 2, 1, 3).to(v.dtype), v], 1)
            lengths = None if lengths is None else lengths + h
        o, S = prism_seq(n(q), n(k), n(v), n(gamma), n(beta), n(u) if L > 1 else None, n(alpha) if L > 1 else None,
                         n(gain) if L > 1 else None, n(conv_w), S0=n(S0), lengths=n(lengths), chain=chain)
        return torch.from_numpy(o[:, h:]), torch.from_numpy(S)

    def affine(self, S, M, N):
        return torch.from_numpy(np.einsum("bhij,bhjk->bhik", S.double().numpy(), M.double().numpy())
                                + N.double().numpy())


def _problem(seed, B, T, H, dk, dv, L, W):
    g = torch.Generator().manual_seed(seed)
    r = lambda *s: torch.randn(*s, generator=g, dtype=torch.float64)
    k = r(B, T, H, dk)
    k = k / k.norm(dim=-1, keepdim=True)
    m = L - 1
    return dict(q=0.5 * r(B, T, H, dk), k=k, v=r(B, T, H, dv),
                gamma=torch.sigmoid(r(B, T, H) + 2.0), beta=torch.sigmoid(r(B, T, H)),
                u=0.3 * r(B, T, H, m, dk), alpha=torch.sigmoid(r(B, T, H, m)),
                gain=torch.sigmoid(r(B, T, H, m, dv)), conv_w=0.5 * r(H, dv, W), S0=0.3 * r(B, H, dv, dk))


def _worker(rank, world, port, out_dir, case):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from linear_attention_sequence_shortconv_b200 import seqshard
    from test_seqshard_cpu import OracleOps, _problem

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        p = _problem(**case["shape"])
        bounds = case["bounds"]  # segment starts, then T
        s, e = bounds[rank], bounds[rank + 1]
        seg = seqshard.Segment(**{n: p[n][:, s:e].contiguous() for n in ("q", "k", "v", "gamma", "beta", "u", "alpha",
                                                                         "gain")}, start=s)
        lengths = None if case["lengths"] is None else torch.tensor(case["lengths"], dtype=torch.int32)
        try:
            o, S_end = seqshard.scan_fwd_sequence_sharded(seg, p["conv_w"], case["shape"]["L"], S0=p["S0"],
                                                          lengths=lengths, chain=case["chain"], ops=OracleOps())
        except ValueError as e:  # a segment shorter than the history: every rank must see it
            np.save(os.path.join(out_dir, f"err_{rank}.npy"), np.array([1]))
            assert "W - 1" in str(e)
            dist.barrier()
            return
        np.save(os.path.join(out_dir, f"o_{rank}.npy"), o.numpy())
        np.save(os.path.join(out_dir, f"S_{rank}.npy"), S_end.numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


CASES = {
    # two ranks, equal segments, ragged lengths (one ends inside rank 0's segment)
    "two_ranks": dict(shape=dict(seed=1, B=3, T=24, H=2, dk=6, dv=5, L=3, W=4), bounds=[0, 12, 24],
                      lengths=[24, 17, 9], chain="linear"),
    # three uneven segments, the exact GELU chain, W = 3
    "three_ranks_gelu": dict(shape=dict(seed=2, B=2, T=23, H=1, dk=4, dv=4, L=4, W=3), bounds=[0, 7, 16, 23],
                             lengths=None, chain="gelu"),
    # W = 1 (no history to exchange), L = 1 (plain gated delta rule)
    "no_history_gdn": dict(shape=dict(seed=3, B=2, T=10, H=2, dk=4, dv=3, L=1, W=1), bounds=[0, 5, 10],
                           lengths=[10, 3], chain="linear"),
}


def test_short_segment_fails_on_every_rank(tmp_path):
    """Rank 1's segment (2 tokens) is shorter than the W - 1 = 3 history rows: both
    ranks raise together, none waits in a collective."""
    case = dict(shape=dict(seed=5, B=1, T=12, H=1, dk=4, dv=4, L=2, W=4), bounds=[0, 10, 12], lengths=None,
                chain="linear")
    mp.start_processes(_worker, args=(2, _free_port(), str(tmp_path), case), nprocs=2, join=True,
                       start_method="spawn")
    assert (tmp_path / "err_0.npy").exists() and (tmp_path / "err_1.npy").exists()


@pytest.mark.parametrize("name", list(CASES))
def test_sharded_scan_equals_whole_sequence(name, tmp_path):
    case = CASES[name]
    world = len(case["bounds"]) - 1
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path), case), nprocs=world, join=True,
                       start_method="spawn")
    sys.path.insert(0, ROOT)
    from oracle import prism_seq

    p = _problem(**case["shape"])
    L = case["shape"]["L"]
    n = lambda t: t.numpy()
    lengths = None if case["lengths"] is None else np.array(case["lengths"])
    o_ref, S_ref = prism_seq(n(p["q"]), n(p["k"]), n(p["v"]), n(p["gamma"]), n(p["beta"]),
                             n(p["u"]) if L > 1 else None, n(p["alpha"]) if L > 1 else None,
                             n(p["gain"]) if L > 1 else None, n(p["conv_w"]), S0=n(p["S0"]), lengths=lengths,
                             chain=case["chain"])
    o = np.concatenate([np.load(tmp_path / f"o_{r}.npy") for r in range(world)], axis=1)
    assert o.shape == o_ref.shape
    assert np.abs(o - o_ref).max() <= 1e-10 * max(1.0, np.abs(o_ref).max())
    S_last = np.load(tmp_path / f"S_{world - 1}.npy")
    assert np.abs(S_last - S_ref).max() <= 1e-10 * max(1.0, np.abs(S_ref).max())


def test_phases_without_collectives():
    """One process running every segment in turn (the gathers become lists): the same
    phases, the same answer; and a segment shorter than the history is rejected."""
    sys.path.insert(0, ROOT)
    from linear_attention_sequence_shortconv_b200 import seqshard
    from oracle import prism_seq

    ops = OracleOps()
    L, W, T = 3, 4, 20
    p = _problem(seed=4, B=2, T=T, H=1, dk=4, dv=4, L=L, W=W)
    bounds = [0, 6, 13, 20]
    segs = [seqshard.Segment(**{n: p[n][:, s:e].contiguous() for n in ("q", "k", "v", "gamma", "beta", "u", "alpha",
                                                                      "gain")}, start=s)
            for s, e in zip(bounds[:-1], bounds[1:])]
    halos = [seqshard.halo_rows(s.v, W) for s in segs]
    hists = [seqshard.conv_history(halos[i - 1]) if i else None for i in range(len(segs))]
    lens = [seqshard.local_lengths(None, s, s.v.shape[1]) for s in segs]
    maps = [seqshard.segment_map(s, p["conv_w"], L, ln, "linear", 64, ops, hs) for s, ln, hs in zip(segs, lens, hists)]
    outs = []
    for r, (sg, ln, hs) in enumerate(zip(segs, lens, hists)):
        S_start = seqshard.start_state(p["S0"], maps[:r], maps[0][1], ops)
        o, S_end = seqshard.scan_segment(sg, p["conv_w"], L, ln, "linear", 64, S_start, ops, hs)
        outs.append(o.numpy())
    n = lambda t: t.numpy()
    o_ref, S_ref = prism_seq(n(p["q"]), n(p["k"]), n(p["v"]), n(p["gamma"]), n(p["beta"]), n(p["u"]), n(p["alpha"]),
                             n(p["gain"]), n(p["conv_w"]), S0=n(p["S0"]))
    assert np.abs(np.concatenate(outs, 1) - o_ref).max() < 1e-10
    assert np.abs(S_end.numpy() - S_ref).max() < 1e-10
    with pytest.raises(ValueError):
        seqshard.halo_rows(p["v"][:, :2], W)


@pytest.mark.parametrize("P,T,W,L,chain,lengths", [
    (4, 26, 4, 3, "linear", [26, 11]),   # uneven: the last segment is padded
    (3, 18, 3, 4, "gelu", None),
    (2, 9, 1, 1, "linear", [9, 0]),      # no history, plain gated delta rule, an empty row
])
def test_segmented_single_device_equals_whole_sequence(P, T, W, L, chain, lengths):
    """scan_fwd_segmented: the segments of every sequence stacked along the batch axis
    in one process, against the oracle's scan of the whole sequence."""
    sys.path.insert(0, ROOT)
    from linear_attention_sequence_shortconv_b200 import seqshard
    from oracle import prism_seq

    p = _problem(seed=P * 10 + T, B=2, T=T, H=2, dk=4, dv=3, L=L, W=W)
    lens = None if lengths is None else torch.tensor(lengths, dtype=torch.int32)
    o, S = seqshard.scan_fwd_segmented(p["q"], p["k"], p["v"], p["gamma"], p["beta"], p["u"], p["alpha"],
                                       p["gain"], p["conv_w"], L, P, S0=p["S0"], lengths=lens, chain=chain,
                                       ops=OracleOps())
    n = lambda t: t.numpy()
    o_ref, S_ref = prism_seq(n(p["q"]), n(p["k"]), n(p["v"]), n(p["gamma"]), n(p["beta"]),
                             n(p["u"]) if L > 1 else None, n(p["alpha"]) if L > 1 else None,
                             n(p["gain"]) if L > 1 else None, n(p["conv_w"]), S0=n(p["S0"]),
                             lengths=None if lengths is None else np.array(lengths), chain=chain)
    assert o.shape == o_ref.shape
    assert np.abs(o.numpy() - o_ref).max() < 1e-10
    assert np.abs(S.numpy() - S_ref).max() < 1e-10
