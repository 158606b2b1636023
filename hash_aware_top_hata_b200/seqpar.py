"""Sequence-parallel HATA decode step over torch.distributed ranks.

A head whose cache is too long for one GPU keeps a contiguous shard of its
tokens on every rank, in rank order (include/hata.h, "Sequence-parallel
decode step").  The histogram top-k of the HATA review page's Algorithm 3
(referee report, major comment 1) needs only the shards' histograms of the
r + 1 Hamming values, so one step is

    hata_sp_score   (local)   this shard's histogram per head
    all-gather                every rank's histograms, rank-major
    hata_sp_attend  (local)   this shard's part of the global selection and
                              its unnormalised attention partial (m, l, acc)
    all-gather                every rank's partials
    hata_sp_merge   (local)   the log-sum-exp merge into out

Both exchanges are a few KB per head (B*H_q*260 int32, then B*H_q*132
fp32), gathered over the process group's backend (NCCL over NVLink between
GPUs).  Every computation runs in libhata's kernels; this module only
allocates the exchange buffers and orders the calls.  Every rank takes the
same collective steps in the same order.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import hata


def _gather(t: torch.Tensor, world: int, group) -> torch.Tensor:
    """All-gather t from every rank into [world, *t.shape] (rank-major)."""
    out = torch.empty((world * t.shape[0],) + tuple(t.shape[1:]), dtype=t.dtype,
                      device=t.device)
    dist.all_gather_into_tensor(out, t.contiguous(), group=group)
    return out.view((world,) + tuple(t.shape))


def sp_decode_step(q: torch.Tensor, W_H: torch.Tensor, codes: torch.Tensor, K: torch.Tensor,
                   V: torch.Tensor, seq_len: torch.Tensor, max_seq_len: int, topk: int,
                   scale: float, workspace: torch.Tensor, out: torch.Tensor, *, group=None,
                   k_new: torch.Tensor | None = None, v_new: torch.Tensor | None = None,
                   sel_idx: torch.Tensor | None = None, ops=hata) -> None:
    """One sequence-parallel decode step of this rank (collective: every rank
    of `group` calls it with its own shard).

    q [B][H_q][128] (the same on every rank), W_H [H_kv][128][r]; codes, K, V
    and seq_len describe this rank's shard as an ordinary cache; k_new / v_new
    only on the rank that holds the newest token.  out [B][H_q][128] receives
    the step's output on every rank; sel_idx, if given, this shard's selected
    positions (shard-local).  `ops` supplies the three phases (libhata's
    binding by default)."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    B, H_q, _ = q.shape
    r = W_H.shape[2]
    hist = torch.empty((B, H_q, hata.HATA_SP_HIST_WORDS), dtype=torch.int32, device=q.device)
    ops.hata_sp_score(q, W_H, codes, K, V, seq_len, max_seq_len, topk, workspace, hist,
                      k_new=k_new, v_new=v_new)
    hist_all = _gather(hist, world, group)
    part = torch.empty((B, H_q, hata.HATA_SP_PART_WORDS), dtype=torch.float32, device=q.device)
    ops.hata_sp_attend(hist_all, rank, codes, K, V, seq_len, max_seq_len, H_q, r, topk, scale,
                       workspace, part, sel_idx=sel_idx)
    part_all = _gather(part, world, group)
    ops.hata_sp_merge(part_all, out)
