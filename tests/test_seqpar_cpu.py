"""Sequence-parallel decode step on two `gloo` ranks (CPU): the exchange
plumbing of hash_aware_top_hata_b200.seqpar against the oracle.

Each rank holds a contiguous shard of one long sequence per (b, KV head) and
runs seqpar.sp_decode_step; the three local phases are supplied here from
the oracle's own primitives (hash, Hamming distance, top-k, fp64 attention)
plus a plain statement of the shard-quota reading of Algorithm 3 (the
HATA review page's referee report, major comment 1: a threshold on the
histogram of Hamming values, boundary ties to the lower token index), so
what runs on the ranks is the module's collective logic.  The union of the
ranks' selections must be the oracle's selection over the whole sequence,
bit for bit, and the merged output its output.  The CUDA phases are checked
against the same oracle in the GPU parity tests.
"""
import math
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LOG2E = 1.0 / math.log(2.0)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OraclePhases:
    """The three local phases of a sequence-parallel step, from the oracle."""

    def __init__(self):
        self.dist = {}

    def hata_sp_score(self, q, W_H, codes, K, V, seq_len, max_seq_len, topk, workspace, hist,
                      k_new=None, v_new=None):
        import oracle
        B, H_q, _ = q.shape
        G = H_q // K.shape[1]
        r = W_H.shape[2]
        hist.zero_()
        for b in range(B):
            n = int(seq_len[b])
            for hq in range(H_q):
                h = hq // G
                qc = oracle.hash_vec(q[b, hq].numpy(), W_H[h].numpy())
                d = oracle.hamming_all(qc, codes[b, h, :n].numpy().view(np.uint32))
                self.dist[b, hq] = d
                hist[b, hq, :r + 1] = torch_from(np.bincount(d, minlength=r + 1))
        self.q = q

    def hata_sp_attend(self, hist_all, rank, codes, K, V, seq_len, max_seq_len, H_q, r, topk,
                       scale, workspace, part, sel_idx=None):
        import oracle
        H = hist_all.numpy().astype(np.int64)[..., :r + 1]  # [world][B][H_q][r+1]
        B = H.shape[1]
        G = H_q // K.shape[1]
        part.zero_()
        for b in range(B):
            for hq in range(H_q):
                tot = H[:, b, hq].sum(0)
                k_eff = min(topk, int(tot.sum()))
                k_loc = 0
                if k_eff > 0:
                    cum = np.cumsum(tot)
                    T = int(np.argmax(cum >= k_eff))
                    n_less = int(cum[T] - tot[T])
                    ties_before = int(H[:rank, b, hq, T].sum())
                    take = min(max(k_eff - n_less - ties_before, 0), int(H[rank, b, hq, T]))
                    k_loc = int(H[rank, b, hq, :T].sum()) + take
                idx = oracle.topk(self.dist[b, hq], k_loc) if k_loc else np.zeros(0, np.int32)
                if sel_idx is not None:
                    sel_idx[b, hq].fill_(-1)
                    sel_idx[b, hq, :len(idx)] = torch_from(idx)
                h = hq // G
                if len(idx) == 0:
                    part[b, hq, 0] = float("-inf")
                    continue
                Ks = K[b, h].numpy()[idx].astype(np.float64)
                Vs = V[b, h].numpy()[idx].astype(np.float64)
                s = (Ks @ self.q[b, hq].numpy().astype(np.float64)) * scale * LOG2E
                m = s.max()
                w = np.exp2(s - m)
                part[b, hq, 0] = m
                part[b, hq, 1] = w.sum()
                part[b, hq, 4:] = torch_from(w @ Vs)

    def hata_sp_merge(self, part_all, out):
        P = part_all.numpy().astype(np.float64)
        M = P[..., 0].max(0)
        wt = np.where(P[..., 0] == -np.inf, 0.0, np.exp2(P[..., 0] - M[None]))
        L = (P[..., 1] * wt).sum(0)
        A = (P[..., 4:] * wt[..., None]).sum(0)
        res = np.where(L[..., None] > 0, A / np.where(L > 0, L, 1)[..., None], 0.0)
        out.copy_(torch_from(res.astype(np.float32)))


def torch_from(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a))


CASES = {
    # name: (B, H_q, H_kv, shard lengths per rank, topk, tie codes)
    "ragged_shards": (2, 4, 2, (700, 333), 64, False),
    "ties_across_the_boundary": (1, 2, 1, (300, 300), 450, True),
    "empty_first_shard": (1, 2, 2, (0, 257), 40, False),
    "k_above_n": (1, 2, 1, (50, 31), 200, False),
}


def _rank_main(rank, world, port, q_out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist

    import oracle
    from hash_aware_top_hata_b200 import seqpar
    res = {}
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world)
        for name, (B, H_q, H_kv, lens, topk, ties) in CASES.items():
            rng = np.random.default_rng(20260 + len(name))
            N = sum(lens)
            d, r = 128, 128
            W = (rng.standard_normal((H_kv, d, r)) / math.sqrt(d)).astype(np.float32)
            q = rng.standard_normal((B, H_q, d)).astype(np.float32)
            K = rng.standard_normal((B, H_kv, N, d)).astype(np.float32)
            V = rng.standard_normal((B, H_kv, N, d)).astype(np.float32)
            codes = oracle.hash_keys(K, W)
            if ties:
                codes[...] = 0
            o0 = sum(lens[:rank])
            n_loc = lens[rank]
            cap = max(n_loc, 1)
            Kl = np.zeros((B, H_kv, cap, d), np.float32)
            Vl = np.zeros_like(Kl)
            Cl = np.zeros((B, H_kv, cap, r // 32), np.uint32)
            Kl[:, :, :n_loc] = K[:, :, o0:o0 + n_loc]
            Vl[:, :, :n_loc] = V[:, :, o0:o0 + n_loc]
            Cl[:, :, :n_loc] = codes[:, :, o0:o0 + n_loc]
            scale = 1 / math.sqrt(d)
            out = torch.zeros(B, H_q, d)
            sel = torch.zeros(B, H_q, topk, dtype=torch.int32)
            seqpar.sp_decode_step(
                torch.from_numpy(q), torch.from_numpy(W), torch.from_numpy(Cl.view(np.int32)),
                torch.from_numpy(Kl), torch.from_numpy(Vl),
                torch.full((B,), n_loc, dtype=torch.int32), cap, topk, scale, None, out,
                sel_idx=sel, ops=OraclePhases())
            # gather the shard selections (global positions) to check the union
            glob = torch.where(sel >= 0, sel + o0, sel)
            allsel = [torch.zeros_like(glob) for _ in range(world)]
            dist.all_gather(allsel, glob)
            checks = []
            for b in range(B):
                for hq in range(H_q):
                    h = hq // (H_q // H_kv)
                    _, _, idx, ref, m = oracle.decode_head(q[b, hq], W[h], codes[b, h], K[b, h],
                                                           V[b, h], N, topk, scale)
                    union = sorted(int(x) for t in allsel for x in t[b, hq].tolist() if x >= 0)
                    checks.append((union == idx[:m].tolist(),
                                   float(np.abs(out[b, hq].numpy() - ref).max())))
            res[name] = checks
        dist.destroy_process_group()
    except Exception as e:  # reported to the parent, which fails the test
        import traceback
        res["error"] = traceback.format_exc()
    q_out.put((rank, res))


@pytest.mark.timeout(300)
def test_sequence_parallel_step_on_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=60)
    for rank, d in res.items():
        assert "error" not in d, d["error"]
        for name in CASES:
            for same_set, err in d[name]:
                assert same_set, (rank, name)
                assert err < 1e-5, (rank, name, err)
