"""CPU oracle for the HATA decode-step path -- TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously-correct C (``hata_oracle.c``) behind a ctypes shim that
takes and returns numpy arrays.  Only ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU-baseline / reference legs may import this package; the
CUDA library never does, and this package imports nothing from it.

Every function follows the HATA review page (arXiv 2506.02572, Pith review):
"What carries the argument" (hash, XOR + popcount Hamming score, top-k,
attention over the selected keys), "Assumptions & free parameters"
(h(x) = sign(x W_H), rbit = 128), Figure 2 / Algorithm 1 (key code cache of
rbit/32 words per token) and major comment 1 (Algorithm 3's top-k over 129
Hamming values, ties in the boundary bucket).  The readings taken where the
page is silent are stated in ``hata_oracle.c``'s header.

Parity pins (the tests in ``tests/test_oracle_pins.py``) tie each function to
something other than itself: brute force, closed forms, invariants and
library routines.  No function here is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hata_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

DT_BF16 = 0
DT_F32 = 1


def _cpu_has_fma() -> bool:
    try:
        with open("/proc/cpuinfo") as f:
            return any(line.startswith("flags") and " fma" in line for line in f)
    except OSError:
        return False


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(src)):
        return out
    cmd = ["gcc", "-O3", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
           "-fPIC", "-shared", "-o", out + ".tmp", src, "-lm"]
    if _cpu_has_fma():
        cmd.insert(1, "-mfma")
    subprocess.check_call(cmd)
    os.replace(out + ".tmp", out)
    return out


_lib = None


def use_library(path: str | None) -> None:
    """Load the oracle from another build of hata_oracle.c (the mutation
    tests load deliberately broken copies); None returns to the default."""
    global _lib
    _lib = None if path is None else _bind(ctypes.CDLL(path))


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        _lib = _bind(ctypes.CDLL(_LIB))
    return _lib


def _bind(L: ctypes.CDLL) -> ctypes.CDLL:
    P, I, I64, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
    L.oracle_hash_f32.argtypes = [P, P, I, I, P]
    L.oracle_hash_vec.argtypes = [P, I, P, I, I, P]
    L.oracle_hash_keys.argtypes = [P, I, P, P, I64, I, I, I64, I64, I, I]
    L.oracle_hamming.argtypes = [P, P, I]
    L.oracle_hamming.restype = I
    L.oracle_hamming_all.argtypes = [P, P, I64, I, P]
    L.oracle_topk.argtypes = [P, I64, I64, P]
    L.oracle_topk.restype = I64
    L.oracle_attend.argtypes = [P, P, P, I, I, P, I64, D, P]
    L.oracle_dense.argtypes = [P, P, P, I, I, I64, D, P]
    L.oracle_decode_head.argtypes = [P, P, P, P, P, I, I64, I, I, I64, D, P, P, P, P]
    L.oracle_decode_head.restype = I64
    return L


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a: np.ndarray) -> int:
    return a.ctypes.data


def _kv_dtype(a: np.ndarray) -> int:
    """bf16 arrays travel as uint16 bit patterns; fp32 as float32."""
    if a.dtype == np.uint16:
        return DT_BF16
    if a.dtype == np.float32:
        return DT_F32
    raise TypeError(f"K/V must be uint16 (bf16 bits) or float32, got {a.dtype}")


def hash_vec(x: np.ndarray, W: np.ndarray) -> np.ndarray:
    """Code of one vector x [d] with one head's W [d][r] -> uint32 [r/32]."""
    d, r = W.shape
    x = np.ascontiguousarray(x)
    dt = _kv_dtype(x)
    W = _c(W, np.float32)
    out = np.zeros(r // 32, np.uint32)
    lib().oracle_hash_vec(_p(x), dt, _p(W), d, r, _p(out))
    return out


def hash_rows(X: np.ndarray, W: np.ndarray) -> np.ndarray:
    """Codes of every row of X [..., d] with one head's W -> [..., r/32]."""
    d, r = W.shape
    X = np.ascontiguousarray(X)
    flat = X.reshape(-1, d)
    out = np.zeros((flat.shape[0], r // 32), np.uint32)
    for i in range(flat.shape[0]):
        out[i] = hash_vec(flat[i], W)
    return out.reshape(X.shape[:-1] + (r // 32,))


def hash_keys(K: np.ndarray, W_H: np.ndarray, pos0: int = 0, n: int | None = None,
              codes: np.ndarray | None = None) -> np.ndarray:
    """Algorithm 1's HashEncode over a [B][H][n_cap][d] key cache."""
    B, H, n_cap, d = K.shape
    r = W_H.shape[2]
    if n is None:
        n = n_cap - pos0
    K = np.ascontiguousarray(K)
    W_H = _c(W_H, np.float32)
    if codes is None:
        codes = np.zeros((B, H, n_cap, r // 32), np.uint32)
    lib().oracle_hash_keys(_p(K), _kv_dtype(K), _p(W_H), _p(codes), n_cap, B, H, pos0, n, d, r)
    return codes


def hamming(a: np.ndarray, b: np.ndarray) -> int:
    a = _c(a, np.uint32)
    b = _c(b, np.uint32)
    return int(lib().oracle_hamming(_p(a), _p(b), a.shape[-1] * 32))


def hamming_all(qcode: np.ndarray, codes: np.ndarray) -> np.ndarray:
    """Distances of one query code to codes [n][r/32] -> int32 [n]."""
    qcode = _c(qcode, np.uint32)
    codes = _c(codes, np.uint32)
    n = codes.shape[0]
    out = np.zeros(n, np.int32)
    lib().oracle_hamming_all(_p(qcode), _p(codes), n, qcode.shape[0] * 32, _p(out))
    return out


def topk(dist: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k smallest distances (ties: lower index), ascending,
    padded with -1 to length k."""
    dist = _c(dist, np.int32)
    out = np.full(max(k, 1), -1, np.int32)
    lib().oracle_topk(_p(dist), dist.shape[0], k, _p(out))
    return out[:k]


def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, idx: np.ndarray,
           scale: float) -> np.ndarray:
    """fp64 softmax attention of q over rows idx of K, V [n][d]."""
    q = _c(q, np.float32)
    K = np.ascontiguousarray(K)
    V = np.ascontiguousarray(V)
    dt = _kv_dtype(K)
    assert _kv_dtype(V) == dt
    idx = _c(idx[idx >= 0], np.int32)
    out = np.zeros(q.shape[0], np.float64)
    lib().oracle_attend(_p(q), _p(K), _p(V), dt, q.shape[0], _p(idx), idx.shape[0],
                        float(scale), _p(out))
    return out


def dense(q: np.ndarray, K: np.ndarray, V: np.ndarray, n: int, scale: float) -> np.ndarray:
    q = _c(q, np.float32)
    K = np.ascontiguousarray(K)
    V = np.ascontiguousarray(V)
    out = np.zeros(q.shape[0], np.float64)
    lib().oracle_dense(_p(q), _p(K), _p(V), _kv_dtype(K), q.shape[0], n, float(scale), _p(out))
    return out


def decode_head(q: np.ndarray, W: np.ndarray, codes: np.ndarray, K: np.ndarray,
                V: np.ndarray, n: int, k: int, scale: float):
    """One query head's decode step over its KV head's first n cached tokens.

    Returns (qcode uint32 [r/32], dist int32 [n], idx int32 [k] ascending
    with -1 pad, out float64 [d], number selected)."""
    d, r = W.shape
    q = _c(q, np.float32)
    W = _c(W, np.float32)
    codes = _c(codes, np.uint32)
    K = np.ascontiguousarray(K)
    V = np.ascontiguousarray(V)
    qcode = np.zeros(r // 32, np.uint32)
    dist = np.zeros(max(n, 1), np.int32)
    idx = np.full(max(k, 1), -1, np.int32)
    out = np.zeros(d, np.float64)
    m = lib().oracle_decode_head(_p(q), _p(W), _p(codes), _p(K), _p(V), _kv_dtype(K), n, d, r,
                                 k, float(scale), _p(qcode), _p(dist), _p(idx), _p(out))
    return qcode, dist[:n], idx[:k], out, int(m)
