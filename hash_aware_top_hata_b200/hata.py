"""ctypes binding of libhata (include/hata.h).

Argument marshalling only: every function takes torch tensors that already
live on the GPU, checks dtype / shape / device, and passes raw pointers and
sizes to the C entry point of the same name on the current torch stream
(or the one given).  Nothing here computes any step of the method, and
there is no fallback: if libhata.so is missing the first call raises.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhata.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "hata.h")

HATA_OK = 0
HATA_ERR_INVALID_ARG = 1
HATA_ERR_UNSUPPORTED = 2
HATA_ERR_CUDA = 3
HATA_ERR_DEVICE_CHECK = 4
HATA_DT_BF16 = 0
HATA_DT_F32 = 1
HATA_FLAG_SEQ_LEN_RANGE = 1
HATA_FLAG_POS_RANGE = 2
HATA_FLAG_TIMEOUT = 4
HATA_NOALLOC_WORKSPACE_BYTES = 64 << 20
HATA_MODE_AUTO = 0
HATA_MODE_MULTI_KERNEL = 1
HATA_MODE_FUSED = 2
HATA_MODE_CLUSTER = 3
HATA_SP_HIST_WORDS = 260
HATA_SP_PART_WORDS = 132
D = 128
RBIT = 128


class HataError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        self.status = status
        super().__init__(f"{where}: {status_name(status)}: {detail}")


_lib = None
P, I, I64, U64, F = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t,
                     ctypes.c_float)
_SIGS = {
    "hata_abi_version": ([], I),
    "hata_status_string": ([I], ctypes.c_char_p),
    "hata_last_error": ([], ctypes.c_char_p),
    "hata_hash_keys": ([P, I, I64, I64, I64, P, P, I64, I, I, I64, I64, I, I, P], I),
    "hata_append_code": ([P, I, P, P, I64, P, I, I, I, I, P, P], I),
    "hata_decode_workspace_size": ([I, I, I, I64, I], U64),
    "hata_dist_row_bytes": ([I64], I64),
    "hata_decode_kernel_launches": ([I, I, I, I64, I, I, I], I),
    "hata_decode_step": ([P, P, P, P, P, I, I64, P, I64, P, P, I, I, I, I, I, I, F, P, U64, P,
                          P, P, P, I64, P, P], I),
    "hata_decode_step_noalloc": ([P, P, P, P, P, I, I64, P, I64, P, P, I, I, I, I, I, I, F, P,
                                  P, P, P, I64, P, P], I),
    "hata_workspace_check": ([P, U64, P, P], I),
    "hata_dense_workspace_size": ([I, I, I, I64], U64),
    "hata_dense_decode": ([P, P, P, I, I64, P, I64, I, I, I, I, F, P, U64, P, P], I),
    "hata_set_decode_mode": ([I], I),
    "hata_get_decode_mode": ([], I),
    "hata_set_wait_limit_ns": ([ctypes.c_uint64], I),
    "hata_sp_score": ([P, P, P, P, P, I, I64, P, I64, P, P, I, I, I, I, I, I, P, U64, P, P], I),
    "hata_sp_attend": ([P, I, I, P, P, P, I, I64, P, I64, I, I, I, I, I, I, F, P, U64, P, P, P],
                       I),
    "hata_sp_merge": ([P, I, I, I, P, P], I),
}


def lib() -> ctypes.CDLL:
    """Load libhata.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m hash_aware_top_hata_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def header_functions() -> list[str]:
    """Names of every function include/hata.h declares."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^[A-Za-z_][\w \*]*?\b(hata_\w+)\s*\(", text, re.M)))


def status_name(status: int) -> str:
    return lib().hata_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != HATA_OK:
        raise HataError(status, where, lib().hata_last_error().decode())


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _kv_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return HATA_DT_BF16
    if t.dtype == torch.float32:
        return HATA_DT_F32
    raise TypeError(f"K/V must be bfloat16 or float32, got {t.dtype}")


def _need(t: torch.Tensor, name: str, dtype=None, ndim=None, cuda=True, host_ok=False) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got shape {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if cuda and not t.is_cuda and not (host_ok and t.is_pinned()):
        raise ValueError(f"{name} must be a CUDA tensor" +
                         (" or a pinned host tensor" if host_ok else ""))


def _need_code_words(codes: torch.Tensor, W_H: torch.Tensor) -> None:
    """codes [..][r/32] must match W_H [H_kv][d][r]."""
    if W_H.dim() != 3 or codes.shape[-1] * 32 != W_H.shape[2]:
        raise ValueError(f"codes {tuple(codes.shape)} hold {codes.shape[-1]} words per token; "
                         f"W_H {tuple(W_H.shape)} gives r/32 words")


# ------------------------------------------------------------------ API --

def hata_abi_version() -> int:
    return int(lib().hata_abi_version())


def hata_status_string(status: int) -> str:
    return status_name(status)


def hata_hash_keys(K: torch.Tensor, W_H: torch.Tensor, codes: torch.Tensor, pos0: int = 0,
                   n: int | None = None, stream=None) -> None:
    """Prefill: codes[b, h, pos0:pos0+n] = hash(K[b, h, pos0:pos0+n]).
    K [B][H_kv][n_cap][128] bf16/fp32, any strides with the last dimension
    contiguous (a strided view of a larger cache is hashed in place),
    W_H [H_kv][128][r] fp32 (r = 32, 64 or 128), codes [B][H_kv][n_cap][r/32]
    int32 (uint32 bit patterns).  K may be a pinned host tensor (a cache kept
    in host memory)."""
    if not isinstance(K, torch.Tensor) or K.dim() != 4:
        raise ValueError("K must be a 4-dim tensor [B][H_kv][n_cap][d]")
    if K.stride(3) != 1:
        raise ValueError("K's last dimension must be contiguous")
    if not K.is_cuda and not K.is_pinned():
        raise ValueError("K must be a CUDA tensor or a pinned host tensor")
    _need(W_H, "W_H", torch.float32, 3)
    _need(codes, "codes", torch.int32, 4)
    _need_code_words(codes, W_H)
    B, H, n_cap, d = K.shape
    if codes.shape[:3] != (B, H, n_cap):
        raise ValueError(f"codes {tuple(codes.shape)} must be [B][H_kv][n_cap][r/32] of K "
                         f"{tuple(K.shape)}")
    n = n_cap - pos0 if n is None else n
    sb, sh, sn, _ = K.stride()
    _check(lib().hata_hash_keys(_ptr(K), _kv_code(K), sb, sh, sn, _ptr(W_H), _ptr(codes), n_cap,
                                B, H, pos0, n, d, W_H.shape[2], _stream(stream)),
           "hata_hash_keys")


def hata_append_code(k_new: torch.Tensor, W_H: torch.Tensor, codes: torch.Tensor,
                     pos: torch.Tensor, err_flags: torch.Tensor | None = None,
                     stream=None) -> None:
    """codes[b, h, pos[b]] = hash(k_new[b, h]).  k_new [B][H_kv][128]."""
    _need(k_new, "k_new", ndim=3)
    _need(W_H, "W_H", torch.float32, 3)
    _need(codes, "codes", torch.int32, 4)
    _need_code_words(codes, W_H)
    _need(pos, "pos", torch.int32, 1)
    if err_flags is not None:
        _need(err_flags, "err_flags", torch.int32)
    B, H, d = k_new.shape
    _check(lib().hata_append_code(_ptr(k_new), _kv_code(k_new), _ptr(W_H), _ptr(codes),
                                  codes.shape[2], _ptr(pos), B, H, d, W_H.shape[2],
                                  _ptr(err_flags), _stream(stream)), "hata_append_code")


def hata_decode_workspace_size(B: int, H_q: int, H_kv: int, max_seq_len: int, topk: int) -> int:
    return int(lib().hata_decode_workspace_size(B, H_q, H_kv, max_seq_len, topk))


def hata_dist_row_bytes(max_seq_len: int) -> int:
    return int(lib().hata_dist_row_bytes(max_seq_len))


def hata_decode_kernel_launches(B: int, H_q: int, H_kv: int, max_seq_len: int, topk: int,
                                kv_dtype: torch.dtype, r: int = RBIT) -> int:
    """Kernels one decode step with these sizes launches on the current device."""
    code = HATA_DT_BF16 if kv_dtype == torch.bfloat16 else HATA_DT_F32
    n = int(lib().hata_decode_kernel_launches(B, H_q, H_kv, max_seq_len, topk, code, r))
    if n < 0:
        raise HataError(HATA_ERR_INVALID_ARG, "hata_decode_kernel_launches",
                        lib().hata_last_error().decode())
    return n


def hata_decode_step(q: torch.Tensor, W_H: torch.Tensor, codes: torch.Tensor, K: torch.Tensor,
                     V: torch.Tensor, seq_len: torch.Tensor, max_seq_len: int, topk: int,
                     scale: float, workspace: torch.Tensor, out: torch.Tensor,
                     k_new: torch.Tensor | None = None, v_new: torch.Tensor | None = None,
                     sel_idx: torch.Tensor | None = None, q_codes: torch.Tensor | None = None,
                     dist: torch.Tensor | None = None, events=None, stream=None) -> None:
    """One HATA decode step for every (b, h_q); see include/hata.h.
    q [B][H_q][128] fp32, K/V [B][H_kv][n_cap][128], seq_len [B] int32,
    workspace uint8 of hata_decode_workspace_size bytes, out [B][H_q][128] fp32.
    Optional: k_new/v_new [B][H_kv][128], sel_idx [B][H_q][topk] int32,
    q_codes [B][H_q][r/32] int32, dist [B][H_q][row] uint8, events: 6 torch.cuda.Event.
    q, k_new, v_new and out may also be pinned host tensors: the kernels read
    and write them over the bus once per step (no separate copies)."""
    _need(q, "q", torch.float32, 3, host_ok=True)
    _need(W_H, "W_H", torch.float32, 3)
    _need(codes, "codes", torch.int32, 4)
    _need_code_words(codes, W_H)
    _need(K, "K", ndim=4, host_ok=True)
    _need(V, "V", ndim=4, host_ok=True)
    _need(seq_len, "seq_len", torch.int32, 1)
    _need(workspace, "workspace", torch.uint8)
    _need(out, "out", torch.float32, 3, host_ok=True)
    for t, name in ((k_new, "k_new"), (v_new, "v_new")):
        if t is not None:
            _need(t, name, K.dtype, 3, host_ok=True)
    if sel_idx is not None:
        _need(sel_idx, "sel_idx", torch.int32, 3)
    if q_codes is not None:
        _need(q_codes, "q_codes", torch.int32, 3)
    drow = 0
    if dist is not None:
        _need(dist, "dist", torch.uint8, 3)
        drow = dist.shape[2]
    B, H_q, d = q.shape
    H_kv, n_cap = K.shape[1], K.shape[2]
    ev = None
    if events is not None:
        if len(events) != 6:
            raise ValueError("events: give 6 torch.cuda.Event (recorded around the 5 kernels)")
        ev = (ctypes.c_void_p * 6)(*[e.cuda_event for e in events])
    _check(lib().hata_decode_step(
        _ptr(q), _ptr(W_H), _ptr(codes), _ptr(K), _ptr(V), _kv_code(K), n_cap, _ptr(seq_len),
        max_seq_len, _ptr(k_new), _ptr(v_new), B, H_q, H_kv, d, W_H.shape[2], topk,
        float(scale), _ptr(workspace), workspace.numel(), _ptr(out), _ptr(sel_idx),
        _ptr(q_codes), _ptr(dist), drow, ev, _stream(stream)), "hata_decode_step")


def hata_sp_score(q: torch.Tensor, W_H: torch.Tensor, codes: torch.Tensor, K: torch.Tensor,
                  V: torch.Tensor, seq_len: torch.Tensor, max_seq_len: int, topk: int,
                  workspace: torch.Tensor, hist_out: torch.Tensor,
                  k_new: torch.Tensor | None = None, v_new: torch.Tensor | None = None,
                  stream=None) -> None:
    """Phase 1 of a sequence-parallel step on this rank's token shard (see
    include/hata.h): hist_out [B][H_q][HATA_SP_HIST_WORDS] int32 receives the
    shard's per-head histogram of Hamming distances."""
    _need(q, "q", torch.float32, 3)
    _need(W_H, "W_H", torch.float32, 3)
    _need(codes, "codes", torch.int32, 4)
    _need_code_words(codes, W_H)
    _need(K, "K", ndim=4)
    _need(V, "V", ndim=4)
    _need(seq_len, "seq_len", torch.int32, 1)
    _need(workspace, "workspace", torch.uint8)
    _need(hist_out, "hist_out", torch.int32, 3)
    for t, name in ((k_new, "k_new"), (v_new, "v_new")):
        if t is not None:
            _need(t, name, K.dtype, 3)
    B, H_q, d = q.shape
    if tuple(hist_out.shape) != (B, H_q, HATA_SP_HIST_WORDS):
        raise ValueError(f"hist_out must be [{B}][{H_q}][{HATA_SP_HIST_WORDS}]")
    H_kv, n_cap = K.shape[1], K.shape[2]
    _check(lib().hata_sp_score(
        _ptr(q), _ptr(W_H), _ptr(codes), _ptr(K), _ptr(V), _kv_code(K), n_cap, _ptr(seq_len),
        max_seq_len, _ptr(k_new), _ptr(v_new), B, H_q, H_kv, d, W_H.shape[2], topk,
        _ptr(workspace), workspace.numel(), _ptr(hist_out), _stream(stream)), "hata_sp_score")


def hata_sp_attend(hist_all: torch.Tensor, rank: int, codes: torch.Tensor, K: torch.Tensor,
                   V: torch.Tensor, seq_len: torch.Tensor, max_seq_len: int, H_q: int, r: int,
                   topk: int, scale: float, workspace: torch.Tensor, part_out: torch.Tensor,
                   sel_idx: torch.Tensor | None = None, stream=None) -> None:
    """Phase 2 of a sequence-parallel step: hist_all [world][B][H_q][HATA_SP_HIST_WORDS]
    int32 (every rank's histograms, rank-major) -> part_out [B][H_q][HATA_SP_PART_WORDS]
    fp32, this shard's unnormalised partial; sel_idx [B][H_q][topk] int32
    optionally receives the shard-local selected positions."""
    _need(hist_all, "hist_all", torch.int32, 4)
    _need(codes, "codes", torch.int32, 4)
    _need(K, "K", ndim=4)
    _need(V, "V", ndim=4)
    _need(seq_len, "seq_len", torch.int32, 1)
    _need(workspace, "workspace", torch.uint8)
    _need(part_out, "part_out", torch.float32, 3)
    if sel_idx is not None:
        _need(sel_idx, "sel_idx", torch.int32, 3)
    world, B = hist_all.shape[0], hist_all.shape[1]
    H_kv, n_cap, d = K.shape[1], K.shape[2], K.shape[3]
    if tuple(part_out.shape) != (B, H_q, HATA_SP_PART_WORDS):
        raise ValueError(f"part_out must be [{B}][{H_q}][{HATA_SP_PART_WORDS}]")
    _check(lib().hata_sp_attend(
        _ptr(hist_all), world, rank, _ptr(codes), _ptr(K), _ptr(V), _kv_code(K), n_cap,
        _ptr(seq_len), max_seq_len, B, H_q, H_kv, d, r, topk, float(scale), _ptr(workspace),
        workspace.numel(), _ptr(part_out), _ptr(sel_idx), _stream(stream)), "hata_sp_attend")


def hata_sp_merge(part_all: torch.Tensor, out: torch.Tensor, stream=None) -> None:
    """Phase 3: part_all [world][B][H_q][HATA_SP_PART_WORDS] fp32 -> out [B][H_q][128]."""
    _need(part_all, "part_all", torch.float32, 4)
    _need(out, "out", torch.float32, 3)
    world, B, H_q = part_all.shape[:3]
    _check(lib().hata_sp_merge(_ptr(part_all), world, B, H_q, _ptr(out), _stream(stream)),
           "hata_sp_merge")


def hata_decode_step_noalloc(q: torch.Tensor, W_H: torch.Tensor, codes: torch.Tensor,
                             K: torch.Tensor, V: torch.Tensor, seq_len: torch.Tensor,
                             max_seq_len: int, topk: int, scale: float, out: torch.Tensor,
                             k_new: torch.Tensor | None = None, v_new: torch.Tensor | None = None,
                             sel_idx: torch.Tensor | None = None,
                             q_codes: torch.Tensor | None = None,
                             dist: torch.Tensor | None = None, events=None, stream=None) -> None:
    """hata_decode_step with the library's fixed device scratch instead of a
    caller workspace, for callers that cannot allocate device memory (see
    include/hata.h).  Calls on one device share that scratch: keep them
    ordered on one stream."""
    _need(q, "q", torch.float32, 3, host_ok=True)
    _need(W_H, "W_H", torch.float32, 3)
    _need(codes, "codes", torch.int32, 4)
    _need_code_words(codes, W_H)
    _need(K, "K", ndim=4, host_ok=True)
    _need(V, "V", ndim=4, host_ok=True)
    _need(seq_len, "seq_len", torch.int32, 1)
    _need(out, "out", torch.float32, 3, host_ok=True)
    for t, name in ((k_new, "k_new"), (v_new, "v_new")):
        if t is not None:
            _need(t, name, K.dtype, 3, host_ok=True)
    if sel_idx is not None:
        _need(sel_idx, "sel_idx", torch.int32, 3)
    if q_codes is not None:
        _need(q_codes, "q_codes", torch.int32, 3)
    drow = 0
    if dist is not None:
        _need(dist, "dist", torch.uint8, 3)
        drow = dist.shape[2]
    B, H_q, d = q.shape
    H_kv, n_cap = K.shape[1], K.shape[2]
    ev = None
    if events is not None:
        if len(events) != 6:
            raise ValueError("events: give 6 torch.cuda.Event (recorded around the 5 kernels)")
        ev = (ctypes.c_void_p * 6)(*[e.cuda_event for e in events])
    _check(lib().hata_decode_step_noalloc(
        _ptr(q), _ptr(W_H), _ptr(codes), _ptr(K), _ptr(V), _kv_code(K), n_cap, _ptr(seq_len),
        max_seq_len, _ptr(k_new), _ptr(v_new), B, H_q, H_kv, d, W_H.shape[2], topk,
        float(scale), _ptr(out), _ptr(sel_idx), _ptr(q_codes), _ptr(dist), drow, ev,
        _stream(stream)), "hata_decode_step_noalloc")


def hata_set_decode_mode(mode: int) -> None:
    """HATA_MODE_AUTO (the library's choice), HATA_MODE_MULTI_KERNEL or
    HATA_MODE_FUSED (the fused step for bf16 caches); process-wide."""
    _check(lib().hata_set_decode_mode(int(mode)), "hata_set_decode_mode")


def hata_get_decode_mode() -> int:
    return int(lib().hata_get_decode_mode())


def hata_set_wait_limit_ns(ns: int) -> None:
    """Bound of every wait of the fused step (default 1 s); process-wide."""
    _check(lib().hata_set_wait_limit_ns(int(ns)), "hata_set_wait_limit_ns")


def hata_workspace_check(workspace: torch.Tensor, stream=None) -> int:
    """Synchronise, then return (and clear) the device-side check flags;
    raises HataError(HATA_ERR_DEVICE_CHECK) if any is set."""
    flags = ctypes.c_uint32(0)
    st = lib().hata_workspace_check(_ptr(workspace), workspace.numel(), ctypes.byref(flags),
                                    _stream(stream))
    if st not in (HATA_OK, HATA_ERR_DEVICE_CHECK):
        _check(st, "hata_workspace_check")
    if st == HATA_ERR_DEVICE_CHECK:
        raise HataError(st, "hata_workspace_check", lib().hata_last_error().decode())
    return int(flags.value)


def hata_dense_workspace_size(B: int, H_q: int, H_kv: int, max_seq_len: int) -> int:
    return int(lib().hata_dense_workspace_size(B, H_q, H_kv, max_seq_len))


def hata_dense_decode(q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, seq_len: torch.Tensor,
                      max_seq_len: int, scale: float, workspace: torch.Tensor,
                      out: torch.Tensor, stream=None) -> None:
    """Dense decode attention over keys 0..seq_len[b]-1 (the full-attention
    baseline)."""
    _need(q, "q", torch.float32, 3)
    _need(K, "K", ndim=4, host_ok=True)
    _need(V, "V", ndim=4, host_ok=True)
    _need(seq_len, "seq_len", torch.int32, 1)
    _need(workspace, "workspace", torch.uint8)
    _need(out, "out", torch.float32, 3)
    B, H_q, d = q.shape
    H_kv, n_cap = K.shape[1], K.shape[2]
    _check(lib().hata_dense_decode(_ptr(q), _ptr(K), _ptr(V), _kv_code(K), n_cap, _ptr(seq_len),
                                   max_seq_len, B, H_q, H_kv, d, float(scale), _ptr(workspace),
                                   workspace.numel(), _ptr(out), _stream(stream)),
           "hata_dense_decode")
