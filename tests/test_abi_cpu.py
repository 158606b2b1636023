"""The C-ABI library without a GPU: it loads, exports every function that
include/hata.h declares, sizes workspaces, and rejects bad arguments on the
host before anything is enqueued (so no call here reaches the GPU)."""
import ctypes

import pytest
import torch

from hash_aware_top_hata_b200 import hata as H

pytestmark = pytest.mark.skipif(
    torch.cuda.is_available(),
    reason="uses fake device addresses; the GPU suite checks the same cases with real tensors")

FAKE = 1 << 20          # 256-byte aligned fake device address (never dereferenced)
NULL = None


def test_library_exports_every_header_function():
    names = H.header_functions()
    assert len(names) >= 10
    lib = H.lib()
    for n in names:
        assert hasattr(lib, n), n
    assert H.hata_abi_version() == 4


def test_status_strings():
    assert H.hata_status_string(0) == "HATA_OK"
    assert H.hata_status_string(1) == "HATA_ERR_INVALID_ARG"
    assert H.hata_status_string(4) == "HATA_ERR_DEVICE_CHECK"
    assert H.hata_status_string(99) == "HATA_ERR_UNKNOWN"


def test_workspace_sizes():
    s = H.hata_decode_workspace_size(4, 32, 8, 131072, 2048)
    assert s > 4 * 32 * 131072  # holds the u8 distance rows at least
    assert H.hata_decode_workspace_size(1, 1, 1, 4096, 64) > 0
    assert H.hata_decode_workspace_size(0, 1, 1, 4096, 64) == 0
    assert H.hata_decode_workspace_size(1, 3, 2, 4096, 64) == 0     # H_q % H_kv
    assert H.hata_decode_workspace_size(1, 1, 1, 0, 64) == 0
    assert H.hata_decode_workspace_size(1, 1, 1, 4096, 0) == 0
    assert H.hata_dist_row_bytes(1) == 4096
    assert H.hata_dist_row_bytes(4096) == 4096
    assert H.hata_dist_row_bytes(4097) == 8192
    assert H.hata_dense_workspace_size(1, 32, 8, 1 << 20) > 0


def decode(**over):
    """hata_decode_step through raw ctypes with fake (never touched) pointers."""
    args = dict(q=FAKE, W=FAKE, codes=FAKE, K=FAKE, V=FAKE, dt=0, n_cap=8192, seq_len=FAKE,
                max_len=4096, k_new=NULL, v_new=NULL, B=1, H_q=4, H_kv=2, d=128, r=128, topk=64,
                scale=0.088, ws=FAKE, ws_bytes=1 << 40, out=FAKE, sel=NULL, qc=NULL, dist=NULL,
                drow=0, ev=NULL, stream=NULL)
    args.update(over)
    return H.lib().hata_decode_step(*args.values())


@pytest.mark.parametrize("over,status", [
    (dict(q=NULL), H.HATA_ERR_INVALID_ARG),
    (dict(codes=NULL), H.HATA_ERR_INVALID_ARG),
    (dict(seq_len=NULL), H.HATA_ERR_INVALID_ARG),
    (dict(ws=NULL), H.HATA_ERR_INVALID_ARG),
    (dict(d=64), H.HATA_ERR_UNSUPPORTED),
    (dict(r=96), H.HATA_ERR_UNSUPPORTED),
    (dict(r=512), H.HATA_ERR_UNSUPPORTED),
    (dict(r=0), H.HATA_ERR_UNSUPPORTED),
    (dict(H_q=3), H.HATA_ERR_UNSUPPORTED),
    (dict(B=0), H.HATA_ERR_INVALID_ARG),
    (dict(topk=0), H.HATA_ERR_INVALID_ARG),
    (dict(max_len=0), H.HATA_ERR_INVALID_ARG),
    (dict(max_len=8193), H.HATA_ERR_INVALID_ARG),
    (dict(n_cap=1 << 31), H.HATA_ERR_INVALID_ARG),
    (dict(dt=7), H.HATA_ERR_INVALID_ARG),
    (dict(v_new=FAKE), H.HATA_ERR_INVALID_ARG),
    (dict(q=FAKE + 4), H.HATA_ERR_INVALID_ARG),
    (dict(codes=FAKE + 8), H.HATA_ERR_INVALID_ARG),
    (dict(K=FAKE + 2), H.HATA_ERR_INVALID_ARG),
    (dict(ws=FAKE + 16), H.HATA_ERR_INVALID_ARG),
    (dict(ws_bytes=1024), H.HATA_ERR_INVALID_ARG),
    (dict(dist=FAKE, drow=100), H.HATA_ERR_INVALID_ARG),
    (dict(dist=FAKE, drow=4080), H.HATA_ERR_INVALID_ARG),
    (dict(B=4096, H_q=32, H_kv=8), H.HATA_ERR_UNSUPPORTED),
    (dict(scale=float("nan")), H.HATA_ERR_INVALID_ARG),
])
def test_decode_step_rejects_on_host(over, status):
    assert decode(**over) == status
    assert H.lib().hata_last_error().decode() != ""


def sp_score(**over):
    """hata_sp_score through raw ctypes with fake pointers."""
    args = dict(q=FAKE, W=FAKE, codes=FAKE, K=FAKE, V=FAKE, dt=0, n_cap=8192, seq_len=FAKE,
                max_len=4096, k_new=NULL, v_new=NULL, B=1, H_q=4, H_kv=2, d=128, r=256, topk=64,
                ws=FAKE, ws_bytes=1 << 40, hist=FAKE, stream=NULL)
    args.update(over)
    return H.lib().hata_sp_score(*args.values())


def sp_attend(**over):
    args = dict(hist_all=FAKE, world=2, rank=1, codes=FAKE, K=FAKE, V=FAKE, dt=0, n_cap=8192,
                seq_len=FAKE, max_len=4096, B=1, H_q=4, H_kv=2, d=128, r=128, topk=64,
                scale=0.088, ws=FAKE, ws_bytes=1 << 40, part=FAKE, sel=NULL, stream=NULL)
    args.update(over)
    return H.lib().hata_sp_attend(*args.values())


@pytest.mark.parametrize("over,status", [
    (dict(q=NULL), H.HATA_ERR_INVALID_ARG),
    (dict(hist=NULL), H.HATA_ERR_INVALID_ARG),
    (dict(hist=FAKE + 2), H.HATA_ERR_INVALID_ARG),
    (dict(r=96), H.HATA_ERR_UNSUPPORTED),
    (dict(topk=0), H.HATA_ERR_INVALID_ARG),
    (dict(v_new=FAKE), H.HATA_ERR_INVALID_ARG),
    (dict(ws_bytes=1024), H.HATA_ERR_INVALID_ARG),
    (dict(max_len=8193), H.HATA_ERR_INVALID_ARG),
])
def test_sp_score_rejects_on_host(over, status):
    assert sp_score(**over) == status
    assert H.lib().hata_last_error().decode() != ""


@pytest.mark.parametrize("over,status", [
    (dict(hist_all=NULL), H.HATA_ERR_INVALID_ARG),
    (dict(part=NULL), H.HATA_ERR_INVALID_ARG),
    (dict(part=FAKE + 4), H.HATA_ERR_INVALID_ARG),
    (dict(world=0), H.HATA_ERR_INVALID_ARG),
    (dict(rank=2), H.HATA_ERR_INVALID_ARG),
    (dict(rank=-1), H.HATA_ERR_INVALID_ARG),
    (dict(scale=float("inf")), H.HATA_ERR_INVALID_ARG),
    (dict(H_q=3), H.HATA_ERR_UNSUPPORTED),
    (dict(ws=FAKE + 16), H.HATA_ERR_INVALID_ARG),
])
def test_sp_attend_rejects_on_host(over, status):
    assert sp_attend(**over) == status


def test_sp_merge_rejects_on_host():
    L = H.lib()
    assert L.hata_sp_merge(NULL, 2, 1, 4, FAKE, NULL) == H.HATA_ERR_INVALID_ARG
    assert L.hata_sp_merge(FAKE, 0, 1, 4, FAKE, NULL) == H.HATA_ERR_INVALID_ARG
    assert L.hata_sp_merge(FAKE, 2, 1, 4, FAKE + 4, NULL) == H.HATA_ERR_INVALID_ARG
    assert L.hata_sp_merge(FAKE, 2, 4096, 32, FAKE, NULL) == H.HATA_ERR_INVALID_ARG


def test_wide_codes_need_wider_histogram_rows():
    """The workspace reserves 257-bin tile histogram rows, whatever r."""
    import math
    B, H_q, n = 1, 4, 100_000
    tiles = math.ceil(math.ceil(n / 4096) * 4096 / 36864)
    assert H.hata_decode_workspace_size(B, H_q, 1, n, 64) >= 4 * B * H_q * tiles * 260


def test_hash_and_append_reject_on_host():
    L = H.lib()
    # K, dtype, strides (b, h, n), W_H, codes, n_cap, B, H_kv, pos0, n, d, r, stream
    dense = [4096 * 2 * 128, 4096 * 128, 128]
    ok_args = [FAKE, 0, *dense, FAKE, FAKE, 4096, 1, 2, 0, 4096, 128, 128, NULL]
    bad = list(ok_args); bad[13] = 96
    assert L.hata_hash_keys(*bad) == H.HATA_ERR_UNSUPPORTED
    bad = list(ok_args); bad[11] = 4097
    assert L.hata_hash_keys(*bad) == H.HATA_ERR_INVALID_ARG
    bad = list(ok_args); bad[10] = -1
    assert L.hata_hash_keys(*bad) == H.HATA_ERR_INVALID_ARG
    bad = list(ok_args); bad[6] = FAKE + 4
    assert L.hata_hash_keys(*bad) == H.HATA_ERR_INVALID_ARG
    bad = list(ok_args); bad[5] = FAKE + 4   # W_H is copied in 16-byte pieces
    assert L.hata_hash_keys(*bad) == H.HATA_ERR_INVALID_ARG
    bad = list(ok_args); bad[0] = NULL
    assert L.hata_hash_keys(*bad) == H.HATA_ERR_INVALID_ARG
    # strides: rows may not overlap, none negative; K aligned to its element
    bad = list(ok_args); bad[4] = 64
    assert L.hata_hash_keys(*bad) == H.HATA_ERR_INVALID_ARG
    bad = list(ok_args); bad[2] = -1
    assert L.hata_hash_keys(*bad) == H.HATA_ERR_INVALID_ARG
    bad = list(ok_args); bad[0] = FAKE + 1
    assert L.hata_hash_keys(*bad) == H.HATA_ERR_INVALID_ARG
    # a strided view (rows of a wider cache, an odd element offset) is fine
    view = [FAKE + 2, 0, 9000 * 2 * 256, 9000 * 256, 256, FAKE, FAKE, 4096, 1, 2, 0, 0, 128,
            128, NULL]
    assert L.hata_hash_keys(*view) == H.HATA_OK
    # n == 0 is a valid no-op that enqueues nothing
    zero = list(ok_args); zero[11] = 0
    assert L.hata_hash_keys(*zero) == H.HATA_OK
    app = [FAKE, 0, FAKE, FAKE, 4096, FAKE, 1, 2, 128, 128, NULL, NULL]
    bad = list(app); bad[5] = NULL
    assert L.hata_append_code(*bad) == H.HATA_ERR_INVALID_ARG
    bad = list(app); bad[8] = 64
    assert L.hata_append_code(*bad) == H.HATA_ERR_UNSUPPORTED


def test_binding_rejects_hash_keys_views_it_cannot_pass():
    K = torch.zeros((1, 2, 64, 128), dtype=torch.bfloat16)
    W = torch.zeros((2, 128, 128))
    codes = torch.zeros((1, 2, 64, 4), dtype=torch.int32)
    with pytest.raises(ValueError):                      # last dim not contiguous
        H.hata_hash_keys(K.transpose(2, 3), W, codes)
    with pytest.raises(ValueError):                      # host memory, not pinned
        H.hata_hash_keys(K, W, codes)


def test_decode_modes():
    assert H.hata_get_decode_mode() == H.HATA_MODE_AUTO
    assert H.lib().hata_set_decode_mode(7) == H.HATA_ERR_INVALID_ARG
    assert H.lib().hata_set_decode_mode(4) == H.HATA_ERR_INVALID_ARG
    for m in (H.HATA_MODE_MULTI_KERNEL, H.HATA_MODE_FUSED, H.HATA_MODE_CLUSTER):
        H.hata_set_decode_mode(m)
        try:
            assert H.hata_get_decode_mode() == m
        finally:
            H.hata_set_decode_mode(H.HATA_MODE_AUTO)
    assert H.hata_get_decode_mode() == H.HATA_MODE_AUTO
    assert H.lib().hata_set_wait_limit_ns(10**9) == H.HATA_OK


def test_dense_rejects_on_host():
    L = H.lib()
    args = [FAKE, FAKE, FAKE, 0, 8192, FAKE, 4096, 1, 4, 2, 128, 0.1, FAKE, 1 << 40, FAKE, NULL]
    bad = list(args); bad[10] = 64
    assert L.hata_dense_decode(*bad) == H.HATA_ERR_UNSUPPORTED
    bad = list(args); bad[13] = 16
    assert L.hata_dense_decode(*bad) == H.HATA_ERR_INVALID_ARG
    bad = list(args); bad[6] = 9000
    assert L.hata_dense_decode(*bad) == H.HATA_ERR_INVALID_ARG


def test_workspace_check_rejects_bad_workspace():
    flags = ctypes.c_uint32(7)
    assert H.lib().hata_workspace_check(NULL, 4096, ctypes.byref(flags), NULL) == \
        H.HATA_ERR_INVALID_ARG
    assert flags.value == 0


def test_decode_kernel_launches_host_logic():
    L = H.lib()
    # fp32 caches beyond the cluster step's reach (more than 8 x 16384 keys)
    # take the SIMT attention kernel, always followed by the combine
    assert H.hata_decode_kernel_launches(4, 32, 8, 200000, 2048, torch.float32) == 5
    # bf16 caches in the fused step: prep, score, the selection + attention kernel
    H.hata_set_decode_mode(H.HATA_MODE_FUSED)
    try:
        assert H.hata_decode_kernel_launches(4, 32, 8, 131072, 2048, torch.bfloat16) == 3
        # 256-bit codes never take the fused step
        assert H.hata_decode_kernel_launches(4, 32, 8, 131072, 2048, torch.float32, 256) == 5
    finally:
        H.hata_set_decode_mode(H.HATA_MODE_AUTO)
    # B, H_q, H_kv, max_seq_len, topk, dtype, r
    for bad in ((0, 32, 8, 4096, 2048, H.HATA_DT_BF16, 128), (4, 0, 8, 4096, 2048, H.HATA_DT_BF16, 128),
                (4, 32, 0, 4096, 2048, H.HATA_DT_BF16, 128), (4, 32, 5, 4096, 2048, H.HATA_DT_BF16, 128),
                (4, 32, 8, 0, 2048, H.HATA_DT_BF16, 128), (4, 32, 8, 4096, 0, H.HATA_DT_BF16, 128),
                (4, 32, 8, 4096, 2048, 9, 128), (4, 32, 8, 4096, 2048, H.HATA_DT_BF16, 96)):
        assert L.hata_decode_kernel_launches(*bad) == -1
    with pytest.raises(H.HataError):
        H.hata_decode_kernel_launches(4, 32, 8, 4096, -1, torch.bfloat16)


def test_library_build_record_matches_sources():
    """libhata.so carries a stamp of the sources it was built from; the
    library under test is the one these sources make."""
    from hash_aware_top_hata_b200 import build as hb
    rec = hb.build_record()
    assert rec.get("sources_sha256") and rec["matches_sources"], rec
