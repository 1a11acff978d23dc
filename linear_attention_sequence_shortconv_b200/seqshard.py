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

The ShortConv history enters a segment as W - 1 inert leading tokens (gamma = 1,
beta = alpha = 0, q = k = u = gain = 0) that carry the previous segment's last v
rows: they leave the state untouched and feed the first anchors.

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

    def scan(self, q, k, v, gamma, beta, u, alpha, gain, conv_w, L, S0, lengths, chain, chunk):
        return _lib.scan_fwd(q, k, v, gamma, beta, u, alpha, gain, conv_w, L=L, chunk=chunk, S0=S0,
                             lengths=lengths, chain=chain)

    def affine(self, S, M, N):
        return _lib.state_affine(S, M, N)


def halo_rows(v: torch.Tensor, W: int) -> torch.Tensor:
    """The last W - 1 token rows of a segment's v, [B, W-1, H, d_v]."""
    if v.shape[1] < W - 1:
        raise ValueError(f"a segment needs at least W - 1 = {W - 1} tokens, got {v.shape[1]}")
    return v[:, v.shape[1] - (W - 1):].contiguous()


def extend(seg: Segment, halo: torch.Tensor) -> Segment:
    """The segment with the inert history tokens in front (v = halo)."""
    n = halo.shape[1]
    if n == 0:
        return seg

    def lead(x, fill):
        if x is None:
            return None
        pad = torch.full((x.shape[0], n) + tuple(x.shape[2:]), fill, dtype=x.dtype, device=x.device)
        return torch.cat([pad, x], dim=1).contiguous()

    return Segment(q=lead(seg.q, 0.0), k=lead(seg.k, 0.0), v=torch.cat([halo.to(seg.v.dtype), seg.v], 1).contiguous(),
                   gamma=lead(seg.gamma, 1.0), beta=lead(seg.beta, 0.0), u=lead(seg.u, 0.0),
                   alpha=lead(seg.alpha, 0.0), gain=lead(seg.gain, 0.0), start=seg.start - n)


def local_lengths(lengths: Optional[torch.Tensor], seg: Segment, n_tokens: int, n_halo: int):
    """Valid tokens of the extended segment per sequence (None: all of them)."""
    if lengths is None:
        return None
    lo = seg.start + n_halo  # global index of the first real token
    return ((lengths.to(torch.int64) - lo).clamp(0, n_tokens) + n_halo).to(torch.int32).contiguous()


def segment_map(ext: Segment, conv_w, L: int, lens, chain: str, chunk: int, ops) -> Tuple[torch.Tensor, torch.Tensor]:
    """(M, N) of an extended segment: S_end = S_start M + N."""
    _, N = ops.scan(ext.q, ext.k, ext.v, ext.gamma, ext.beta, ext.u, ext.alpha, ext.gain, conv_w, L, None, lens,
                    chain, chunk)
    # the transitions alone: no writes (v = 0, L = 1), start from the identity
    B, T, H, d_k = ext.k.shape
    zq = torch.zeros_like(ext.q)
    zv = torch.zeros((B, T, H, d_k), dtype=ext.v.dtype, device=ext.v.device)
    zw = torch.zeros((H, d_k, 1), dtype=torch.float32, device=ext.v.device)
    eye = torch.eye(d_k, dtype=torch.float32, device=ext.v.device).expand(B, H, d_k, d_k).contiguous()
    _, M = ops.scan(zq, ext.k, zv, ext.gamma, ext.beta, None, None, None, zw, 1, eye, lens, chain, chunk)
    return M, N


def start_state(S0, maps: List[Tuple[torch.Tensor, torch.Tensor]], like: torch.Tensor, ops) -> torch.Tensor:
    """S0 (or zeros shaped like `like`) carried through the maps of the earlier segments."""
    S = torch.zeros_like(like) if S0 is None else S0
    for M, N in maps:
        S = ops.affine(S.contiguous(), M, N)
    return S


def scan_segment(ext: Segment, conv_w, L: int, lens, chain: str, chunk: int, S_start, n_halo: int, ops):
    """The exact outputs and end state of a segment from its start state."""
    o, S_end = ops.scan(ext.q, ext.k, ext.v, ext.gamma, ext.beta, ext.u, ext.alpha, ext.gain, conv_w, L,
                        S_start.contiguous(), lens, chain, chunk)
    return o[:, n_halo:], S_end


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
    halo = halos[rank - 1] if rank > 0 else torch.zeros_like(mine)
    ext = extend(seg, halo)
    lens = local_lengths(lengths, ext, n_tokens, W - 1)
    # 2. this segment's map
    M, N = segment_map(ext, conv_w, L, lens, chain, chunk, ops)
    # 3. every segment's map; fold the earlier ones into this segment's start state
    Ms = [torch.empty_like(M) for _ in range(P)]
    Ns = [torch.empty_like(N) for _ in range(P)]
    dist.all_gather(Ms, M.contiguous(), group=group)
    dist.all_gather(Ns, N.contiguous(), group=group)
    S_start = start_state(S0, list(zip(Ms[:rank], Ns[:rank])), N, ops)
    # 4. the exact pass
    return scan_segment(ext, conv_w, L, lens, chain, chunk, S_start, W - 1, ops)


def scan_fwd_segmented(q, k, v, gamma, beta, u, alpha, gain, conv_w, L: int, P: int, S0=None, lengths=None,
                       chain: str = "linear", chunk: int = 64, ops=None):
    """The whole scan on one device with each sequence cut into P segments that run
    side by side: the segments are stacked along the batch axis (P x B sequences of
    ceil(T / P) + W - 1 tokens), so each of the three scans has P times the
    parallelism at 1/P of the length; the maps are folded in P - 1 affine steps.
    Returns (o [B, T, H, d_v], S_final) as scan_fwd."""
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
    exts, lens = [], []
    for r in range(P):
        seg = Segment(**{n: None if x is None else x[:, r * Ts:(r + 1) * Ts] for n, x in full.items()},
                      start=r * Ts)
        halo = (full["v"][:, r * Ts - (W - 1):r * Ts] if r > 0 else
                torch.zeros((B, W - 1) + tuple(v.shape[2:]), dtype=v.dtype, device=v.device))
        ext = extend(seg, halo)
        exts.append(ext)
        lens.append(local_lengths(lengths, ext, Ts, W - 1))
    # every segment side by side: batch index r * B + b
    cat = lambda xs: None if xs[0] is None else torch.cat(xs, 0).contiguous()
    stacked = Segment(**{n: cat([getattr(e, n) for e in exts]) for n in full}, start=0)
    lens_all = torch.cat(lens, 0).contiguous()
    M, N = segment_map(stacked, conv_w, L, lens_all, chain, chunk, ops)
    Ms, Ns = M.view(P, B, *M.shape[1:]), N.view(P, B, *N.shape[1:])
    starts = [torch.zeros_like(Ns[0]) if S0 is None else S0]
    for r in range(1, P):
        starts.append(ops.affine(starts[-1].contiguous(), Ms[r - 1].contiguous(), Ns[r - 1].contiguous()))
    o, S_end = scan_segment(stacked, conv_w, L, lens_all, chain, chunk, torch.cat(starts, 0), W - 1, ops)
    o = o.reshape(P, B, Ts, *o.shape[2:]).permute(1, 0, 2, 3, 4).reshape(B, P * Ts, *o.shape[2:])
    return o[:, :T], S_end.view(P, B, *S_end.shape[1:])[P - 1]
