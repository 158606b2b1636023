"""Parity with the CPU oracle of the cluster step (one kernel per decode step:
a thread-block cluster per (batch row, KV head), its CTAs meeting through
distributed shared memory), forced with HATA_MODE_CLUSTER on shapes it
serves -- each case first checks that the step is one launch, i.e. that the
cluster step, not the multi-kernel fallback, is what runs.

Bar as everywhere: codes, distances and indices bit-exact, outputs within
2e-3 of the fp64 oracle."""
import numpy as np
import pytest
import torch

from hash_aware_top_hata_b200 import hata as H
from hash_aware_top_hata_b200 import workloads as wl
from tests.gpu_cases import GpuDecoder, compare_head, host_slabs, oracle_head, to_np_codes
from tests.test_parity_gpu import run_and_check

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def cluster_mode():
    H.hata_set_decode_mode(H.HATA_MODE_CLUSTER)
    yield
    H.hata_set_decode_mode(H.HATA_MODE_AUTO)


def _launches(cfg, n_cap):
    dt = torch.bfloat16 if cfg.kv_dtype == "bf16" else torch.float32
    return H.hata_decode_kernel_launches(cfg.B, cfg.H_q, cfg.H_kv, n_cap, cfg.topk, dt)


CASES = {
    # name: Config(name, B, H_q, H_kv, N, topk, dtype, planted, scale, needles, steps)
    "one_cta_mha": wl.Config("c", 2, 4, 4, 5000, 300, "bf16", 0.02, 0.3, 0, 2),
    "four_ctas_mha": wl.Config("c", 1, 8, 8, 30000, 512, "bf16", 0.02, 0.3, 0, 2),
    "two_heads_per_kv": wl.Config("c", 1, 8, 4, 20000, 700, "bf16", 0.02, 0.3, 0, 2),
    "eight_ctas_gqa4": wl.Config("c", 1, 8, 2, 65000, 2048, "bf16", 0.02, 0.3, 0, 2),
    "16k_ctas_gqa4": wl.Config("c", 4, 32, 8, 40000, 1500, "bf16", 0.02, 0.3, 0, 2),
    "llama2_shape": wl.Config("c", 1, 32, 32, 32768, 512, "bf16", 0.02, 0.3, 0, 2),
    "k_above_n": wl.Config("c", 2, 4, 2, 3000, 5000, "bf16", 0.0, 0.0, 0, 2),
    "fp32_mha": wl.Config("c", 1, 4, 4, 6000, 200, "f32", 0.02, 0.3, 0, 2),
    "fp32_gqa2_three_ctas": wl.Config("c", 2, 8, 4, 40000, 700, "f32", 0.02, 0.3, 0, 2),
    "tiny_shape": wl.Config("c", 1, 1, 1, 4096, 64, "f32", 0.0, 0.0, 0, 2),
}


@pytest.mark.parametrize("name", list(CASES))
def test_cluster_step_matches_oracle(name):
    cfg = CASES[name]
    n_cap = cfg.N + cfg.steps
    assert _launches(cfg, n_cap) == 1, "the cluster step should serve this shape"
    run_and_check(cfg, seed=90 + len(name), steps=2)


def test_cluster_ties_across_cta_boundaries():
    """Identical keys: every distance ties, so the selection is the k lowest
    indices, crossing the ranges of several CTAs of a cluster."""
    cfg = wl.Config("c-ties", 1, 4, 2, 30000, 20000, "bf16", 0.0, 0.0, 0, 1)
    w = wl.make_workload(cfg, 95, device="cuda", steps=1)
    w.K[0, :, :] = w.K[0, :, 3:4].clone()
    dec = GpuDecoder(w, cfg.topk)
    assert _launches(cfg, dec.max_seq_len) == 1
    out, sel, qc, dist = dec.step(w.q[0], [cfg.N])
    assert np.all(sel[0] == np.arange(cfg.topk)[None, :])
    slabs = host_slabs(w, [(0, 0), (0, 1)])
    Wn = w.W_H.cpu().numpy()
    for hq in range(4):
        want = oracle_head(slabs[(0, hq // 2)], Wn[hq // 2], w.q[0, 0, hq].cpu().numpy(), cfg.N,
                           cfg.topk)
        compare_head((out, sel, qc, dist), want, 0, hq, cfg.N, dec.drow)


def test_cluster_ragged_lengths_and_boundary_ties():
    """Lengths that end inside, at and before CTA ranges (and an empty row),
    with a run of identical keys across a range boundary forming the
    boundary bucket."""
    cfg = wl.Config("c-rag", 4, 8, 4, 40000, 1200, "bf16", 0.0, 0.0, 0, 1)
    w = wl.make_workload(cfg, 96, device="cuda", steps=1)
    w.K[:, :, 7000:12000] = w.K[:, :, 1:2].clone()  # crosses the range boundary at 8000
    dec = GpuDecoder(w, cfg.topk, max_seq_len=40000)
    assert _launches(cfg, 40000) == 1
    lens = [40000, 10001, 0, 9001]
    got = dec.step(w.q[0], lens)
    pairs = [(b, h) for b in range(4) for h in range(4)]
    slabs = host_slabs(w, pairs)
    Wn = w.W_H.cpu().numpy()
    for b in range(4):
        for hq in range(8):
            n = lens[b]
            if n == 0:
                assert np.all(got[0][b, hq] == 0) and np.all(got[1][b, hq] == -1)
                assert np.all(got[3][b, hq] == 255)
                continue
            want = oracle_head(slabs[(b, hq // 2)], Wn[hq // 2], w.q[0, b, hq].cpu().numpy(), n,
                               cfg.topk)
            compare_head(got, want, b, hq, n, dec.drow)


def test_cluster_step_is_bitwise_repeatable_and_matches_multi_kernel():
    cfg = wl.Config("c-rep", 2, 16, 4, 30000, 900, "bf16", 0.02, 0.3, 0, 1)
    w = wl.make_workload(cfg, 97, device="cuda", steps=1)
    dec = GpuDecoder(w, cfg.topk)
    a = dec.step(w.q[0], [cfg.N, cfg.N - 77])
    b = dec.step(w.q[0], [cfg.N, cfg.N - 77])
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    H.hata_set_decode_mode(H.HATA_MODE_MULTI_KERNEL)
    c = dec.step(w.q[0], [cfg.N, cfg.N - 77])
    assert np.array_equal(a[1], c[1]) and np.array_equal(a[2], c[2]) and np.array_equal(a[3], c[3])
    assert np.max(np.abs(a[0] - c[0])) <= 1e-4


def test_cluster_append_lands_in_first_and_middle_ctas():
    """The new token's code and K/V rows are written by the CTA whose range
    holds position seq_len - 1: here the first CTA of one row's cluster and
    a middle CTA of another's (max_seq_len 40000: three CTAs of ~13.3K)."""
    cfg = wl.Config("c-app", 2, 8, 4, 40000, 300, "bf16", 0.02, 0.3, 0, 1)
    w = wl.make_workload(cfg, 98, device="cuda", steps=1)
    dec = GpuDecoder(w, cfg.topk, max_seq_len=40000)
    assert _launches(cfg, 40000) == 1
    lens = [100, 20000]  # appends at 99 (CTA 0) and 19999 (CTA 1)
    pairs = [(b, h) for b in range(2) for h in range(4)]
    slabs = host_slabs(w, pairs)
    kn, vn = wl.to_numpy_kv(w.k_new[0]), wl.to_numpy_kv(w.v_new[0])
    for (b, h), sl in slabs.items():
        sl.K[lens[b] - 1] = kn[b, h]
        sl.V[lens[b] - 1] = vn[b, h]
    got = dec.step(w.q[0], lens, k_new=w.k_new[0], v_new=w.v_new[0])
    Wn = w.W_H.cpu().numpy()
    gcodes = to_np_codes(dec.codes)
    for b in range(2):
        for hq in range(8):
            h = hq // 2
            n = lens[b]
            want = oracle_head(slabs[(b, h)], Wn[h], w.q[0, b, hq].cpu().numpy(), n, cfg.topk)
            assert np.array_equal(gcodes[b, h, :n], want[0]), ("key codes", b, h)
            compare_head(got, want, b, hq, n, dec.drow)
    for (b, h), sl in slabs.items():  # the appended rows reached the caches
        p = lens[b] - 1
        assert np.array_equal(wl.to_numpy_kv(w.K[b, h, p]), sl.K[p])
        assert np.array_equal(wl.to_numpy_kv(w.V[b, h, p]), sl.V[p])
