"""hata_decode_step_noalloc: the decode step for callers that cannot
allocate device memory (a plugin whose engine owns all device memory, or a
latency-critical path that must not hit cudaMalloc's implicit device
synchronisation).  It takes its scratch from a fixed array in the library's
device image.  Checked through the C ABI against hata_decode_step (which
uses a caller workspace) on the same inputs, on two calls in a row: the
second call reuses the shared scratch left by the first.

This file is named so that pytest collects it last."""
import math

import numpy as np
import pytest
import torch

from hash_aware_top_hata_b200 import hata as H
from hash_aware_top_hata_b200 import workloads as wl

ATOL = 2e-3
SCALE = 1.0 / math.sqrt(128)


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice():
    cfg = wl.Config("noalloc", 2, 8, 2, 9000, 150, "bf16", 0.02, 0.3, 0, 2)
    w = wl.make_workload(cfg, 91, device="cuda", steps=2)
    codes = torch.zeros((cfg.B, cfg.H_kv, w.n_cap, 4), dtype=torch.int32, device="cuda")
    H.hata_hash_keys(w.K, w.W_H, codes, 0, cfg.N)
    ws = torch.empty(H.hata_decode_workspace_size(cfg.B, cfg.H_q, cfg.H_kv, w.n_cap, cfg.topk),
                     dtype=torch.uint8, device="cuda")
    assert ws.numel() <= H.HATA_NOALLOC_WORKSPACE_BYTES
    for t in range(2):  # two calls in a row, the second on the first one's scratch
        sl = torch.full((cfg.B,), cfg.N - 100 * t, dtype=torch.int32, device="cuda")
        outs = []
        for noalloc in (False, True):
            out = torch.full((cfg.B, cfg.H_q, 128), float("nan"), device="cuda")
            sel = torch.full((cfg.B, cfg.H_q, cfg.topk), -7, dtype=torch.int32, device="cuda")
            if noalloc:
                H.hata_decode_step_noalloc(w.q[t], w.W_H, codes, w.K, w.V, sl, w.n_cap, cfg.topk,
                                           SCALE, out, sel_idx=sel)
            else:
                H.hata_decode_step(w.q[t], w.W_H, codes, w.K, w.V, sl, w.n_cap, cfg.topk, SCALE,
                                   ws, out, sel_idx=sel)
            torch.cuda.synchronize()
            outs.append((out.cpu().numpy(), sel.cpu().numpy()))
        (o_ref, s_ref), (o_na, s_na) = outs
        assert np.all(np.isfinite(o_na))
        assert np.max(np.abs(o_na - o_ref)) <= ATOL
        assert np.array_equal(s_na, s_ref)


@pytest.mark.gpu
def test_noalloc_rejects_sizes_beyond_its_buffer():
    q = torch.zeros((1, 1, 128), device="cuda")
    small = torch.zeros(16, dtype=torch.int32, device="cuda")
    big_len = 1 << 20
    need = H.hata_decode_workspace_size(32, 28, 4, big_len, 16384)
    assert need > H.HATA_NOALLOC_WORKSPACE_BYTES
    # rejected by the size check on the host, before anything is enqueued
    st = H.lib().hata_decode_step_noalloc(
        q.data_ptr(), q.data_ptr(), small.data_ptr(), small.data_ptr(), small.data_ptr(),
        H.HATA_DT_BF16, big_len, small.data_ptr(), big_len, None, None, 32, 28, 4, 128, 128,
        16384, SCALE, q.data_ptr(), None, None, None, 0, None,
        torch.cuda.current_stream().cuda_stream)
    assert st == H.HATA_ERR_INVALID_ARG
    assert "no-alloc buffer" in H.lib().hata_last_error().decode()
