"""Sequence sharding of the PRISM scan over ranks (one GPU per rank).

A long sequence is split into consecutive segments, one per rank.  The state
update (ICML 2026 PRISM write-up, 核心迭代形式 / 架构形式)

    S_t = S_{t-1} gamma_t (I - beta_t k_t k_t^T) + beta_t v_t k_t^T + sum_l alpha_l r_l u_l^T

is affine in the state, so a run over a segment maps its start state S to S M + N:
M (d_k x d_k) is the ordered product of the transitions and N the segment's end
state from a zero start.  Each rank

  0. all-gathers the segment lengths (a segment shorter than the W - 1 history rows
     makes every rank raise, not only its own);
  1. all-gathers the last W - 1 rows of v of every segment: the ShortConv history
     of the segment after it;
  2. scans its segment from a zero state (N) and, with the writes switched off, from
     the identity (M);
  3. all-gathers (M, N) and folds S0 through the maps of the segments before its own
     (prism_state_affine): its exact start state;
  4. scans its segment again from that state: its outputs and end state are exact.

The ShortConv history enters a segment as the scan's conv_state: the previous
segment's last W - 1 rows of v, which feed the segment's first anchors.

Every step runs in the library (prism_scan_fwd, prism_state_affine); the two
exchanges are torch.distributed all-gathers (NCCL over NVLink between GPUs).  The
phases are separate functions so that one process can also run all segments in
turn, with the gathers replaced by plain lists.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional, Tuple

import torch

from . import _lib


@dataclass
class Segment:
    """One rank's tokens of every sequence: tensors [B, Ts, H, ...] as for scan_fwd,
    and the global index of the first token."""
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    gamma: torch.Tensor
    beta: torch.Tensor
    u: Optional[torch.Tensor]
    alpha: Optional[torch.Tensor]
    gain: Optional[torch.Tensor]
    start: int


class LibraryOps:
    """The two operations the sharded scan needs, on the library."""

    def scan(self, q, k, v, gamma, beta, u, alpha, gain, conv_w, L, S0, lengths, chain, chunk, conv_state=None):
        return _lib.scan_fwd(q, k, v, gamma, beta, u, alpha, gain, conv_w, L=L, chunk=chunk, S0=S0,
                             lengths=lengths, chain=chain, conv_state=conv_state)

    def affine(self, S, M, N):
        return _lib.state_affine(S, M, N)


def halo_rows(v: torch.Tensor, W: int) -> torch.Tensor:
    """The last W - 1 token rows of a segment's v, [B, W-1, H, d_v]."""
    if v.shape[1] < W - 1:
        raise ValueError(f"a segment needs at least W - 1 = {W - 1} tokens, got {v.shape[1]}")
    return v[:, v.shape[1] - (W - 1):].contiguous()


def conv_history(halo: torch.Tensor) -> torch.Tensor:
    """Halo rows [B, W-1, H, d_v] as the scan's conv_state [B, H, W-1, d_v]."""
    return halo.permute(0, 2, 1, 3).contiguous()


def local_lengths(lengths: Optional[torch.Tensor], seg: Segment, n_tokens: int):
    """Valid tokens of the segment per sequence (None: all of them)."""
    if lengths is None:
        return None
    return (lengths.to(torch.int64) - seg.start).clamp(0, n_tokens).to(torch.int32).contiguous()


def segment_map(seg: Segment, conv_w, L: int, lens, chain: str, chunk: int, ops,
                conv_state=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """(M, N) of a segment: S_end = S_start M + N (conv_state: its ShortConv history)."""
    _, N = ops.scan(seg.q, seg.k, seg.v, seg.gamma, seg.beta, seg.u, seg.alpha, seg.gain, conv_w, L, None, lens,
                    chain, chunk, conv_state)
    # the transitions alone: no writes (v = 0, L = 1), start from the identity
    B, T, H, d_k = seg.k.shape
    zq = torch.zeros_like(seg.q)
    zv = torch.zeros((B, T, H, d_k), dtype=seg.v.dtype, device=seg.v.device)
    zw = torch.zeros((H, d_k, 1), dtype=torch.float32, device=seg.v.device)
    eye = torch.eye(d_k, dtype=torch.float32, device=seg.v.device).expand(B, H, d_k, d_k).contiguous()
    _, M = ops.scan(zq, seg.k, zv, seg.gamma, seg.beta, None, None, None, zw, 1, eye, lens, chain, chunk)
    return M, N


def start_state(S0, maps: List[Tuple[torch.Tensor, torch.Tensor]], like: torch.Tensor, ops) -> torch.Tensor:
    """S0 (or zeros shaped like `like`) carried through the maps of the earlier segments."""
    S = torch.zeros_like(like) if S0 is None else S0
    for M, N in maps:
        S = ops.affine(S.contiguous(), M, N)
    return S


def scan_segment(seg: Segment, conv_w, L: int, lens, chain: str, chunk: int, S_start, ops, conv_state=None):
    """The exact outputs and end state of a segment from its start state."""
    return ops.scan(seg.q, seg.k, seg.v, seg.gamma, seg.beta, seg.u, seg.alpha, seg.gain, conv_w, L,
                    S_start.contiguous(), lens, chain, chunk, conv_state)


def scan_fwd_sequence_sharded(seg: Segment, conv_w, L: int, S0=None, lengths=None, chain: str = "linear",
                              chunk: int = 64, group=None, ops=None):
    """This rank's outputs [B, Ts, H, d_v] and the state after its segment.  The
    segments are consecutive in rank order; `lengths` are the global sequence lengths
    and S0 the global initial state (read on every rank)."""
    import torch.distributed as dist

    ops = ops or LibraryOps()
    rank, P = dist.get_rank(group), dist.get_world_size(group)
    W = conv_w.shape[-1]
    n_tokens = seg.v.shape[1]
    # 0. every rank checks every segment's length, so that all of them raise together
    #    instead of some waiting in a collective that the others never reach
    sizes = [torch.zeros(1, dtype=torch.int64, device=seg.v.device) for _ in range(P)]
    dist.all_gather(sizes, torch.tensor([n_tokens], dtype=torch.int64, device=seg.v.device), group=group)
    if min(int(x.item()) for x in sizes) < W - 1:
        raise ValueError(f"every segment needs at least W - 1 = {W - 1} tokens; segment lengths "
                         f"{[int(x.item()) for x in sizes]}")
    # 1. ShortConv history of every segment
    mine = halo_rows(seg.v, W)
    halos = [torch.empty_like(mine) for _ in range(P)]
    if W > 1:
        dist.all_gather(halos, mine, group=group)
    hist = conv_history(halos[rank - 1]) if rank > 0 and W > 1 else None
    lens = local_lengths(lengths, seg, n_tokens)
    # 2. this segment's map
    M, N = segment_map(seg, conv_w, L, lens, chain, chunk, ops, hist)
    # 3. every segment's map; fold the earlier ones into this segment's start state
    Ms = [torch.empty_like(M) for _ in range(P)]
    Ns = [torch.empty_like(N) for _ in range(P)]
    dist.all_gather(Ms, M.contiguous(), group=group)
    dist.all_gather(Ns, N.contiguous(), group=group)
    S_start = start_state(S0, list(zip(Ms[:rank], Ns[:rank])), N, ops)
    # 4. the exact pass
    return scan_segment(seg, conv_w, L, lens, chain, chunk, S_start, ops, hist)


def scan_fwd_segmented(q, k, v, gamma, beta, u, alpha, gain, conv_w, L: int, P: int, S0=None, lengths=None,
                       chain: str = "linear", chunk: int = 64, ops=None):
    """The whole scan on one device with each sequence cut into P segments that run
    side by side: the segments are stacked along the batch axis (P x B sequences of
    ceil(T / P) tokens, each with the previous segment's last W - 1 rows of v as its
    conv_state), so each of the three scans has P times the parallelism at 1/P of the
    length; the maps are folded in P - 1 affine steps.  Returns (o [B, T, H, d_v],
    S_final) as scan_fwd."""
    ops = ops or LibraryOps()
    B, T, H, _ = q.shape
    W = conv_w.shape[-1]
    Ts = -(-T // P)
    if Ts < W - 1:
        raise ValueError(f"segments of {Ts} tokens are shorter than the W - 1 = {W - 1} history rows")
    pad = P * Ts - T

    def padded(x):  # [B, P*Ts, ...]: the tail past T is never a valid token
        if x is None or pad == 0:
            return x
        return torch.cat([x, torch.zeros((B, pad) + tuple(x.shape[2:]), dtype=x.dtype, device=x.device)], 1)

    full = {n: padded(x) for n, x in dict(q=q, k=k, v=v, gamma=gamma, beta=beta, u=u, alpha=alpha,
                                          gain=gain).items()}
    if lengths is None:
        lengths = torch.full((B,), T, dtype=torch.int32, device=q.device)
    segs, lens, hists = [], [], []
    for r in range(P):
        seg = Segment(**{n: None if x is None else x[:, r * Ts:(r + 1) * Ts] for n, x in full.items()},
                      start=r * Ts)
        halo = (full["v"][:, r * Ts - (W - 1):r * Ts] if r > 0 else
                torch.zeros((B, W - 1) + tuple(v.shape[2:]), dtype=v.dtype, device=v.device))
        segs.append(seg)
        lens.append(local_lengths(lengths, seg, Ts))
        hists.append(conv_history(halo))
    # every segment side by side: batch index r * B + b
    cat = lambda xs: None if xs[0] is None else torch.cat(xs, 0).contiguous()
    stacked = Segment(**{n: cat([getattr(e, n) for e in segs]) for n in full}, start=0)
    lens_all = torch.cat(lens, 0).contiguous()
    hist = cat(hists) if W > 1 else None
    M, N = segment_map(stacked, conv_w, L, lens_all, chain, chunk, ops, hist)
    Ms, Ns = M.view(P, B, *M.shape[1:]), N.view(P, B, *N.shape[1:])
    starts = [torch.zeros_like(Ns[0]) if S0 is None else S0]
    for r in range(1, P):
        starts.append(ops.affine(starts[-1].contiguous(), Ms[r - 1].contiguous(), Ns[r - 1].contiguous()))
    o, S_end = scan_segment(stacked, conv_w, L, lens_all, chain, chunk, torch.cat(starts, 0), ops, hist)
    o = o.reshape(P, B, Ts, *o.shape[2:]).permute(1, 0, 2, 3, 4).reshape(B, P * Ts, *o.shape[2:])
    return o[:, :T], S_end.view(P, B, *S_end.shape[1:])[P - 1]
