"""Parity with the CPU oracle of the ablation's 256-bit codes at the top of
their distance range, and of the sequence-parallel step (one head's keys
sharded over ranks).

The sequence-parallel step is run here on one GPU: the shards of every rank
go through hata_sp_score / hata_sp_attend one after another and the two
exchanges are stacks of the ranks' buffers (what an all-gather delivers);
no kernel waits on another rank.  The union of the shards' selections must
be the oracle's selection over the whole sequence bit for bit, the merged
output its output within the attention tolerance."""
import math

import numpy as np
import pytest
import torch

import oracle
from hash_aware_top_hata_b200 import hata as H
from hash_aware_top_hata_b200 import workloads as wl
from tests.gpu_cases import (ATOL, SCALE, GpuDecoder, compare_head, host_slabs, oracle_head,
                             to_np_codes)

pytestmark = pytest.mark.gpu


# ------------------------------------------------ 256-bit codes, d = 255/256 --

@pytest.mark.parametrize("topk", [30, 300, 540, 2000, 80010])
def test_wide_codes_boundary_at_saturated_distances(topk):
    """Head 0's keys are coded as the complement of its query code (distance
    256), 500 of them with one bit flipped back (255), 40 close to the query:
    the boundary falls below 255 (k = 30), inside the 255 bucket (300),
    exactly at its end (540), inside the 256 bucket (2000) or past every key,
    over three selection tiles.  Head 1 (another query of the same KV head)
    sees ordinary distances."""
    N = 80000
    cfg = wl.Config("wide-top", 1, 2, 1, N, topk, "bf16", 0.0, 0.0, 0, 1)
    w = wl.make_workload(cfg, 61, device="cuda", steps=1)
    slabs = host_slabs(w, [(0, 0)])
    dec = GpuDecoder(w, topk, r=256)
    Wn = dec.W.cpu().numpy()
    q0 = w.q[0, 0, 0].cpu().numpy()
    qc = oracle.hash_vec(q0, Wn[0])
    rng = np.random.default_rng(5)
    codes = np.tile(~qc, (N, 1))
    pos = rng.choice(N, 540, replace=False)
    for i in pos[:500]:
        wd, bt = divmod(int(rng.integers(0, 256)), 32)
        codes[i, wd] ^= np.uint32(1 << bt)
    for i in pos[500:]:
        codes[i] = qc
        codes[i, 0] ^= np.uint32(7)  # distance 3
    host = to_np_codes(dec.codes).copy()
    host[0, 0, :N] = codes
    dec.codes.copy_(torch.from_numpy(host.view(np.int32)).cuda())
    got = dec.step(w.q[0], [N])
    for hq in (0, 1):
        want = oracle_head(slabs[(0, 0)], Wn[0], w.q[0, 0, hq].cpu().numpy(), N, topk, codes)
        compare_head(got, want, 0, hq, N, dec.drow)
    d0 = got[3][0, 0, :N]
    assert np.all(d0[pos[:500]] == 255) and np.all(d0[pos[500:]] == 3)


# ------------------------------------------------------ sequence-parallel --

def _shard(t: torch.Tensor, o: int, n: int) -> torch.Tensor:
    """Tokens o .. o+n-1 of a [B][H_kv][N][...] cache as its own cache (at
    least one position)."""
    out = torch.zeros((t.shape[0], t.shape[1], max(n, 1)) + tuple(t.shape[3:]), dtype=t.dtype,
                      device=t.device)
    out[:, :, :n] = t[:, :, o:o + n]
    return out


def run_sp(w: wl.Workload, lens, topk: int, r: int = 128, codes_np=None):
    """The sequence-parallel step over len(lens) emulated ranks; returns
    (out [B][H_q][128], selected global indices per head, phase outputs)."""
    cfg = w.cfg
    B, H_q, H_kv = cfg.B, cfg.H_q, cfg.H_kv
    W = wl.projection(w.W_H, r)
    q = w.q[0]
    world = len(lens)
    shards, hists = [], []
    o = 0
    for rank, n in enumerate(lens):
        K, V = _shard(w.K, o, n), _shard(w.V, o, n)
        codes = torch.full((B, H_kv, K.shape[2], r // 32), -1, dtype=torch.int32, device="cuda")
        if codes_np is not None:
            codes[:, :, :n] = torch.from_numpy(
                np.ascontiguousarray(codes_np[:, :, o:o + n]).view(np.int32)).cuda()
        elif n:
            H.hata_hash_keys(K, W, codes, 0, n)
        sl = torch.full((B,), n, dtype=torch.int32, device="cuda")
        max_len = K.shape[2]
        ws = torch.empty(H.hata_decode_workspace_size(B, H_q, H_kv, max_len, topk),
                         dtype=torch.uint8, device="cuda")
        hist = torch.full((B, H_q, H.HATA_SP_HIST_WORDS), -1, dtype=torch.int32, device="cuda")
        H.hata_sp_score(q, W, codes, K, V, sl, max_len, topk, ws, hist)
        shards.append((o, n, K, V, codes, sl, max_len, ws))
        hists.append(hist)
        o += n
    hist_all = torch.stack(hists)
    parts, sels = [], []
    for rank, (o, n, K, V, codes, sl, max_len, ws) in enumerate(shards):
        part = torch.full((B, H_q, H.HATA_SP_PART_WORDS), float("nan"), device="cuda")
        sel = torch.full((B, H_q, topk), -7, dtype=torch.int32, device="cuda")
        H.hata_sp_attend(hist_all, rank, codes, K, V, sl, max_len, H_q, r, topk, SCALE, ws,
                         part, sel_idx=sel)
        assert H.hata_workspace_check(ws) == 0
        parts.append(part)
        sels.append(torch.where(sel >= 0, sel + o, sel))
    out = torch.full((B, H_q, 128), float("nan"), device="cuda")
    H.hata_sp_merge(torch.stack(parts), out)
    torch.cuda.synchronize()
    sel_all = torch.stack(sels).cpu().numpy()  # [world][B][H_q][topk]
    union = {}
    for b in range(B):
        for hq in range(H_q):
            s = sel_all[:, b, hq]
            assert np.all((s >= 0) | (s == -1))
            union[b, hq] = np.sort(s[s >= 0])
    return out.cpu().numpy(), union, hist_all.cpu().numpy()


def check_sp(w, lens, topk, r=128, heads=None, codes_np=None):
    cfg = w.cfg
    N = sum(lens)
    pairs = sorted({(b, hq // cfg.G) for b in range(cfg.B) for hq in range(cfg.H_q)})
    slabs = host_slabs(w, pairs)
    out, union, hist_all = run_sp(w, lens, topk, r, codes_np)
    Wn = wl.projection(w.W_H, r).cpu().numpy()
    heads = heads or [(b, hq) for b in range(cfg.B) for hq in range(cfg.H_q)]
    cache = {}
    for b, hq in heads:
        h = hq // cfg.G
        codes = None if codes_np is None else codes_np[b, h]
        codes = cache.get((b, h), codes)
        want = oracle_head(slabs[(b, h)], Wn[h], w.q[0, b, hq].cpu().numpy(), N, topk, codes)
        cache[(b, h)] = want[0]
        _, _, wdist, widx, wout = want
        m = min(topk, N)
        np.testing.assert_array_equal(union[b, hq], widx[:m], err_msg=f"b={b} hq={hq}")
        err = np.max(np.abs(out[b, hq].astype(np.float64) - wout))
        assert err <= ATOL, (b, hq, err)
        # each shard's histogram is the oracle's distance histogram of its tokens
        o = 0
        for rank, n in enumerate(lens):
            want_h = np.bincount(wdist[o:o + n], minlength=r + 1)
            np.testing.assert_array_equal(hist_all[rank, b, hq, :r + 1], want_h)
            assert np.all(hist_all[rank, b, hq, r + 1:] == 0)
            o += n


SP_CASES = {
    # name: (config, shard lengths, topk, r)
    "gqa_three_ranks": (wl.Config("sp", 1, 8, 2, 50000, 2048, "bf16", 0.02, 0.3, 0, 1),
                        (20000, 17000, 13000), 2048, 128),
    "gqa_batch_two_ranks": (wl.Config("sp", 2, 4, 1, 30000, 500, "bf16", 0.02, 0.3, 0, 1),
                            (12288, 17712), 500, 128),
    "mha_fp32_empty_first_shard": (wl.Config("sp", 1, 3, 3, 9000, 300, "f32", 0.0, 0.0, 0, 1),
                                   (0, 5000, 4000), 300, 128),
    "wide_codes_four_ranks": (wl.Config("sp", 1, 4, 1, 40000, 1000, "bf16", 0.02, 0.3, 0, 1),
                              (10000, 10000, 10000, 10000), 1000, 256),
    "narrow_codes_many_ties": (wl.Config("sp", 1, 4, 2, 40000, 3000, "bf16", 0.0, 0.0, 0, 1),
                               (15000, 25000), 3000, 32),
    "k_above_n": (wl.Config("sp", 1, 2, 1, 700, 1000, "bf16", 0.0, 0.0, 0, 1),
                  (300, 400), 1000, 128),
}


@pytest.mark.parametrize("name", list(SP_CASES))
def test_sequence_parallel_step_matches_oracle(name):
    cfg, lens, topk, r = SP_CASES[name]
    w = wl.make_workload(cfg, 70 + len(name), device="cuda", steps=1)
    check_sp(w, lens, topk, r)


def test_sequence_parallel_ties_across_ranks():
    """Identical keys on every rank: all distances tie, so the selection is
    the k lowest global indices -- the whole first shard and the head of the
    second, more than one attention CTA's index capacity on one rank."""
    cfg = wl.Config("sp-ties", 1, 2, 1, 30000, 9000, "bf16", 0.0, 0.0, 0, 1)
    w = wl.make_workload(cfg, 81, device="cuda", steps=1)
    w.K[0, 0, :] = w.K[0, 0, 5].clone()
    lens = (6000, 14000, 10000)
    out, union, _ = run_sp(w, lens, cfg.topk)
    for hq in range(2):
        assert np.array_equal(union[0, hq], np.arange(9000))
    check_sp(w, lens, cfg.topk)


def test_sequence_parallel_matches_single_gpu_step():
    """The sharded step selects what the single-GPU step selects on the
    same sequence (both against the oracle above; here against each other
    at a size the oracle skips: a 262K-token head over four ranks)."""
    cfg = wl.Config("sp-big", 1, 8, 2, 262144, 4096, "bf16", 0.0, 0.0, 64, 1)
    w = wl.make_workload(cfg, 83, device="cuda", steps=1)
    dec = GpuDecoder(w, cfg.topk)
    out1, sel1, _, _ = dec.step(w.q[0], [cfg.N])
    out, union, _ = run_sp(w, (65536, 65536, 65536, 65536), cfg.topk)
    for b in range(cfg.B):
        for hq in range(cfg.H_q):
            assert np.array_equal(union[b, hq], sel1[b, hq]), hq
            assert np.max(np.abs(out[b, hq] - out1[b, hq])) <= 1e-4
