"""Seeded synthetic decode workloads.

This module only draws random inputs; it holds none of the method's
arithmetic.  Tests, the oracle checks, ``smoke()`` and ``bench.py`` all take
their inputs from here, so the CUDA path and the CPU oracle see the same
tensors.

The shapes follow the decode workloads of the HATA review page (Llama-2-7B
MHA, Llama-3.1-8B GQA, Qwen2.5 GQA, long-context needle tests; head_dim 128,
rbit 128, a 1.56% token budget).  The page's own evaluation suites (LongBench,
RULER, InfiniteBench, NIAH) and trained hash weights are not available, so:

* q, K, V are i.i.d. N(0, 1); W_H is N(0, 1/128) per KV head (random-hyperplane
  hashing stands in for the trained hash);
* a fraction of keys per KV head is "planted": key = a * u + N(0, 1), where u
  is the direction of the group's first query head scaled to the norm of an
  N(0, I_128) draw, u = q / |q| * sqrt(128);
* the million-token case instead plants 64 "needles" per KV head,
  key = 0.8 * u + 0.2 * N(0, 1), at random positions;
* queries of later decode steps are q_t = q_0 + 0.25 * eps_t, and each step
  appends one fresh N(0, 1) key and value per sequence and KV head;
* the other code widths of the page's ablation use the leading r columns of
  W_H (r = 32, 64), or W_H followed by r - 128 more N(0, 1/128) columns drawn
  from their own seeded stream (r = 256): see ``projection``.
"""
from __future__ import annotations

import dataclasses
import math

import torch

D = 128
RBIT = 128


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    B: int
    H_q: int
    H_kv: int
    N: int
    topk: int
    kv_dtype: str          # "bf16" | "f32"
    planted_frac: float    # fraction of planted relevant keys per KV head
    planted_scale: float   # a in key = a * u + noise
    needles: int           # needles per KV head (0 = none)
    steps: int             # decode steps the workload describes

    @property
    def G(self) -> int:
        return self.H_q // self.H_kv


CONFIGS = {
    "tiny_mha_4k": Config("tiny_mha_4k", 1, 1, 1, 4096, 64, "f32", 0.0, 0.0, 0, 1),
    "llama2_7b_mha_32k": Config("llama2_7b_mha_32k", 1, 32, 32, 32768, 512, "bf16",
                                0.02, 0.3, 0, 1),
    "llama31_8b_gqa_128k": Config("llama31_8b_gqa_128k", 4, 32, 8, 131072, 2048, "bf16",
                                  0.02, 0.3, 0, 1),
    "qwen_gqa_b32_32k": Config("qwen_gqa_b32_32k", 32, 28, 4, 32768, 512, "bf16",
                               0.01, 0.5, 0, 16),
    "needle_gqa_1m": Config("needle_gqa_1m", 1, 32, 8, 1048576, 16384, "bf16",
                            0.0, 0.0, 64, 1),
}
CONFIG_ORDER = list(CONFIGS)
SEED_BASE = 20260000


def scaled(cfg: Config, N: int, topk: int | None = None, B: int | None = None,
           name: str | None = None) -> Config:
    """The same workload at a smaller context (for tests the oracle finishes)."""
    return dataclasses.replace(cfg, N=N, topk=cfg.topk if topk is None else topk,
                               B=cfg.B if B is None else B,
                               name=name or f"{cfg.name}@N{N}")


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn(shape, g, device, dtype=torch.float32):
    return torch.randn(shape, generator=g, device=device, dtype=dtype)


@dataclasses.dataclass
class Workload:
    cfg: Config
    n_cap: int
    q: torch.Tensor          # [steps][B][H_q][D] f32 (q for every decode step)
    W_H: torch.Tensor        # [H_kv][D][RBIT] f32
    K: torch.Tensor          # [B][H_kv][n_cap][D] bf16/f32; rows >= N are zero
    V: torch.Tensor          # same
    k_new: torch.Tensor      # [steps][B][H_kv][D] keys appended by each step
    v_new: torch.Tensor      # [steps][B][H_kv][D]
    planted: torch.Tensor    # [B][H_kv][P] int64 planted/needle positions (P may be 0)

    @property
    def kv_torch_dtype(self):
        return self.K.dtype


def make_workload(cfg: Config, seed: int, device="cpu", steps: int | None = None,
                  n_cap: int | None = None) -> Workload:
    """Draw one workload.  Separate generator streams feed q, K, V, W_H, the
    planted positions and the appended tokens, so changing one size does not
    shift the others' random numbers more than it must."""
    steps = cfg.steps if steps is None else steps
    B, Hq, Hkv, N = cfg.B, cfg.H_q, cfg.H_kv, cfg.N
    G = Hq // Hkv
    n_cap = N + steps if n_cap is None else n_cap
    assert n_cap >= N + max(steps - 1, 0)
    kv_dtype = torch.bfloat16 if cfg.kv_dtype == "bf16" else torch.float32

    g_q = _gen(device, seed * 16 + 1)
    g_k = _gen(device, seed * 16 + 2)
    g_v = _gen(device, seed * 16 + 3)
    g_w = _gen(device, seed * 16 + 4)
    g_p = _gen("cpu", seed * 16 + 5)
    g_s = _gen(device, seed * 16 + 6)

    q0 = _randn((B, Hq, D), g_q, device)
    q = [q0]
    for _ in range(1, max(steps, 1)):
        q.append(q0 + 0.25 * _randn((B, Hq, D), g_s, device))
    q = torch.stack(q)

    W_H = _randn((Hkv, D, RBIT), g_w, device) * (1.0 / math.sqrt(D))

    K = torch.zeros((B, Hkv, n_cap, D), dtype=kv_dtype, device=device)
    V = torch.zeros((B, Hkv, n_cap, D), dtype=kv_dtype, device=device)
    # Draw per (b, h) slab to bound peak memory for million-token contexts.
    planted_all = []
    for b in range(B):
        row = []
        for h in range(Hkv):
            kf = _randn((N, D), g_k, device)
            u = q0[b, h * G]
            u = u / u.norm() * math.sqrt(D)
            if cfg.needles > 0:
                pos = torch.randperm(N, generator=g_p)[:cfg.needles].sort().values
                noise = kf[pos.to(device)]
                kf[pos.to(device)] = 0.8 * u + 0.2 * noise
            elif cfg.planted_frac > 0:
                cnt = int(round(cfg.planted_frac * N))
                pos = torch.randperm(N, generator=g_p)[:cnt].sort().values
                kf[pos.to(device)] += cfg.planted_scale * u
            else:
                pos = torch.zeros(0, dtype=torch.int64)
            row.append(pos)
            K[b, h, :N] = kf.to(kv_dtype)
            del kf
            V[b, h, :N] = _randn((N, D), g_v, device).to(kv_dtype)
        planted_all.append(row)
    P = max((p.numel() for r in planted_all for p in r), default=0)
    planted = torch.full((B, Hkv, P), -1, dtype=torch.int64)
    for b in range(B):
        for h in range(Hkv):
            p = planted_all[b][h]
            planted[b, h, :p.numel()] = p

    k_new = _randn((max(steps, 1), B, Hkv, D), g_s, device).to(kv_dtype)
    v_new = _randn((max(steps, 1), B, Hkv, D), g_s, device).to(kv_dtype)
    return Workload(cfg, n_cap, q, W_H, K, V, k_new, v_new, planted)


def projection(W_H: torch.Tensor, r: int, seed: int = 20260256) -> torch.Tensor:
    """The [H_kv][D][r] projection of an r-bit code from a workload's
    [H_kv][D][128] W_H: its leading r columns for r <= 128, else W_H with
    r - 128 further N(0, 1/D) columns appended (their own generator, seeded
    `seed`, on W_H's device)."""
    if r <= RBIT:
        return W_H if r == RBIT else W_H[:, :, :r].contiguous()
    g = _gen(W_H.device, seed)
    extra = _randn((W_H.shape[0], D, r - RBIT), g, W_H.device) * (1.0 / math.sqrt(D))
    return torch.cat([W_H, extra], dim=2).contiguous()


def bf16_bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (the oracle's bf16 format)."""
    import numpy as np
    if t.dtype == torch.bfloat16:
        return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    return t.detach().cpu().contiguous().numpy()


def to_numpy_kv(t: torch.Tensor):
    """K/V in the oracle's storage format: uint16 bits for bf16, float32 else."""
    return bf16_bits(t)
