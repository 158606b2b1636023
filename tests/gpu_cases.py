"""Helpers shared by the GPU parity tests: run the CUDA path through the
C ABI and the CPU oracle on the same seeded inputs.

The oracle never sees a value produced by the CUDA path: its K/V caches are
built on the host from the generator's own tensors (the prompt cache plus
the keys/values each decode step appends), and it hashes every key itself.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

import oracle
from hash_aware_top_hata_b200 import hata as H
from hash_aware_top_hata_b200 import workloads as wl

SCALE = 1.0 / math.sqrt(128)
ATOL = 2e-3  # max abs error of the attention output (bf16 K/V, fp32 accumulation)


def to_np_codes(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().numpy().view(np.uint32)


@dataclass
class HostCache:
    """Host copy of one (b, h_kv) slab as the oracle must see it."""
    K: np.ndarray   # [n_cap][128] uint16 (bf16 bits) or float32
    V: np.ndarray


def host_slabs(w: wl.Workload, pairs) -> dict:
    """Copy the generator's prompt cache of the given (b, h_kv) pairs to the
    host before any kernel runs."""
    return {(b, h): HostCache(wl.to_numpy_kv(w.K[b, h]).copy(), wl.to_numpy_kv(w.V[b, h]).copy())
            for (b, h) in pairs}


def host_append(slabs: dict, w: wl.Workload, step: int, pos: list[int]) -> None:
    """Apply decode step `step`'s appended key/value rows to the host slabs."""
    kn = wl.to_numpy_kv(w.k_new[step])
    vn = wl.to_numpy_kv(w.v_new[step])
    for (b, h), s in slabs.items():
        s.K[pos[b]] = kn[b, h]
        s.V[pos[b]] = vn[b, h]


class GpuDecoder:
    """Owns the device code cache and workspace of one workload."""

    def __init__(self, w: wl.Workload, topk: int, max_seq_len: int | None = None,
                 prefill: int | None = None, r: int = 128):
        cfg = w.cfg
        self.w = w
        self.topk = topk
        self.r = r
        # r < 128: the leading r columns of the workload's projection;
        # r = 256: more columns from their own seeded stream
        self.W = wl.projection(w.W_H, r)
        self.max_seq_len = max_seq_len or w.n_cap
        self.codes = torch.full((cfg.B, cfg.H_kv, w.n_cap, r // 32), -1, dtype=torch.int32,
                                device="cuda")
        H.hata_hash_keys(w.K, self.W, self.codes, 0, cfg.N if prefill is None else prefill)
        self.ws = torch.empty(H.hata_decode_workspace_size(cfg.B, cfg.H_q, cfg.H_kv,
                                                           self.max_seq_len, topk),
                              dtype=torch.uint8, device="cuda")
        self.drow = H.hata_dist_row_bytes(self.max_seq_len)

    def step(self, q: torch.Tensor, seq_len: list[int], k_new=None, v_new=None):
        cfg = self.w.cfg
        B, Hq = cfg.B, cfg.H_q
        out = torch.full((B, Hq, 128), float("nan"), device="cuda")
        sel = torch.full((B, Hq, self.topk), -7, dtype=torch.int32, device="cuda")
        qc = torch.zeros((B, Hq, self.r // 32), dtype=torch.int32, device="cuda")
        dist = torch.full((B, Hq, self.drow), 77, dtype=torch.uint8, device="cuda")
        sl = torch.tensor(seq_len, dtype=torch.int32, device="cuda")
        H.hata_decode_step(q, self.W, self.codes, self.w.K, self.w.V, sl, self.max_seq_len,
                           self.topk, SCALE, self.ws, out, k_new=k_new, v_new=v_new,
                           sel_idx=sel, q_codes=qc, dist=dist)
        flags = H.hata_workspace_check(self.ws)
        assert flags == 0
        return out.cpu().numpy(), sel.cpu().numpy(), to_np_codes(qc), dist.cpu().numpy()


def oracle_head(slab: HostCache, W: np.ndarray, q: np.ndarray, n: int, topk: int,
                codes: np.ndarray | None = None):
    """Oracle decode of one query head over the first n tokens of its slab."""
    if codes is None:
        codes = oracle.hash_keys(slab.K[None, None, :n], W[None])[0, 0]
    qc, dist, idx, out, m = oracle.decode_head(q, W, codes[:n], slab.K[:n], slab.V[:n], n, topk,
                                               SCALE)
    return codes, qc, dist, idx, out


def compare_head(got, want, b, hq, n, drow, check_dist=True):
    """Bit-exact q code / distances / indices, toleranced output.  The
    byte-wide distance rows hold min(distance, 255) (256-bit codes reach 256)."""
    out, sel, qc, dist = got
    _, wqc, wdist, widx, wout = want
    assert np.array_equal(qc[b, hq], wqc), (b, hq, qc[b, hq], wqc)
    if check_dist:
        wdist = np.minimum(wdist, 255)
        d = dist[b, hq]
        bad = np.nonzero(d[:n] != wdist)[0]
        assert bad.size == 0, (b, hq, bad[:10], d[bad[:10]], wdist[bad[:10]])
        assert np.all(d[n:drow] == 255)
    np.testing.assert_array_equal(sel[b, hq], widx, err_msg=f"indices b={b} hq={hq}")
    err = np.max(np.abs(out[b, hq].astype(np.float64) - wout))
    assert err <= ATOL, (b, hq, err)
    return err
