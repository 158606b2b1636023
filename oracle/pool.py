"""The CPU oracle's decode step spread over the host cores -- TEST AND BENCH
INFRASTRUCTURE ONLY (bench.py's CPU-baseline leg and reference arm).

A whole decode step of a workload runs as one task per query head on a
process pool started with the "spawn" method (safe next to a CUDA context).
The K/V caches, the key codes, W_H and the queries live in memory-mapped
files under a temporary directory, so the workers share them without copies.
Every task calls the oracle exactly as it stands (``oracle.decode_head``,
``oracle.hash_keys``); nothing here computes any step of the method itself.
"""
from __future__ import annotations

import multiprocessing as mp
import os
import shutil
import tempfile
import time

import numpy as np

_maps: dict = {}


def _open(spec):
    """(path, dtype, shape) -> a memory map of the file, cached per process."""
    path, dtype, shape = spec
    m = _maps.get(path)
    if m is None:
        m = np.memmap(path, dtype=np.dtype(dtype), mode="r+", shape=tuple(shape))
        _maps[path] = m
    return m


def _hash_slab(args):
    import oracle
    Ks, Ws, Cs, b, h, n = args
    K, W, C = _open(Ks), _open(Ws), _open(Cs)
    C[b, h, :n] = oracle.hash_keys(np.ascontiguousarray(K[b, h, :n])[None, None],
                                   np.ascontiguousarray(W[h])[None])[0, 0]
    return b, h


def _decode(args):
    import oracle
    Ks, Vs, Ws, Cs, Qs, b, hq, G, n, k, scale = args
    K, V, W, C, Q = _open(Ks), _open(Vs), _open(Ws), _open(Cs), _open(Qs)
    h = hq // G
    _, _, idx, out, _ = oracle.decode_head(np.ascontiguousarray(Q[b, hq]), np.ascontiguousarray(W[h]),
                                           np.ascontiguousarray(C[b, h, :n]),
                                           np.ascontiguousarray(K[b, h, :n]),
                                           np.ascontiguousarray(V[b, h, :n]), n, k, scale)
    return b, hq, idx, out


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


class OracleStep:
    """A workload's caches on the host and a pool of oracle workers.

    K, V: [B][H_kv][n_cap][d] (uint16 bf16 bits or float32); W: [H_kv][d][r];
    the key codes are hashed by the pool (``hash_prefix``)."""

    def __init__(self, K: np.ndarray, V: np.ndarray, W: np.ndarray, H_q: int,
                 workers: int | None = None):
        self.dir = tempfile.mkdtemp(prefix="hata_oracle_")
        self.B, self.H_kv, self.n_cap, self.d = K.shape
        self.H_q, self.G = H_q, H_q // self.H_kv
        self.r = W.shape[2]
        self.K = self._store("K", K)
        self.V = self._store("V", V)
        self.W = self._store("W", W.astype(np.float32))
        self.C = self._alloc("C", np.uint32, (self.B, self.H_kv, self.n_cap, self.r // 32))
        self.Q = self._alloc("Q", np.float32, (self.B, self.H_q, self.d))
        self.workers = workers or host_cores()
        self.pool = mp.get_context("spawn").Pool(self.workers)

    def _alloc(self, name, dtype, shape):
        path = os.path.join(self.dir, name)
        m = np.memmap(path, dtype=dtype, mode="w+", shape=shape)
        return (path, np.dtype(dtype).str, shape), m

    def _store(self, name, arr):
        spec, m = self._alloc(name, arr.dtype, arr.shape)
        m[...] = arr
        m.flush()
        return spec, m

    def hash_prefix(self, n: int) -> float:
        """Key codes of positions 0 .. n-1 of every slab (one task per slab);
        returns the wall seconds."""
        t0 = time.perf_counter()
        tasks = [(self.K[0], self.W[0], self.C[0], b, h, n)
                 for b in range(self.B) for h in range(self.H_kv)]
        self.pool.map(_hash_slab, tasks)
        return time.perf_counter() - t0

    def append(self, k_new: np.ndarray, v_new: np.ndarray, pos: int) -> None:
        """The decode step's append: K/V rows at pos, and their codes hashed by
        the oracle."""
        import oracle
        self.K[1][:, :, pos] = k_new
        self.V[1][:, :, pos] = v_new
        W = self.W[1]
        for b in range(self.B):
            for h in range(self.H_kv):
                self.C[1][b, h, pos] = oracle.hash_vec(np.ascontiguousarray(k_new[b, h]),
                                                       np.ascontiguousarray(W[h]))
        for m in (self.K[1], self.V[1], self.C[1]):
            m.flush()

    def step(self, q: np.ndarray, n: int, topk: int, scale: float,
             heads: list | None = None):
        """The oracle's decode of every (or the given) query head over keys
        0 .. n-1, one task per head; returns (wall seconds, {(b, hq): (idx, out)})."""
        self.Q[1][...] = q
        self.Q[1].flush()
        heads = heads or [(b, hq) for b in range(self.B) for hq in range(self.H_q)]
        tasks = [(self.K[0], self.V[0], self.W[0], self.C[0], self.Q[0], b, hq, self.G, n, topk,
                  scale) for b, hq in heads]
        t0 = time.perf_counter()
        res = self.pool.map(_decode, tasks, chunksize=1)
        dt = time.perf_counter() - t0
        return dt, {(b, hq): (idx, out) for b, hq, idx, out in res}

    def one_core_seconds_per_head(self, q: np.ndarray, n: int, topk: int, scale: float,
                                  heads: list) -> float:
        """Whole heads decoded one after another in this process (one core)."""
        self.Q[1][...] = q
        self.Q[1].flush()
        t0 = time.perf_counter()
        for b, hq in heads:
            _decode((self.K[0], self.V[0], self.W[0], self.C[0], self.Q[0], b, hq, self.G, n,
                     topk, scale))
        return (time.perf_counter() - t0) / len(heads)

    def close(self) -> None:
        self.pool.terminate()
        self.pool.join()
        _maps.clear()
        shutil.rmtree(self.dir, ignore_errors=True)
