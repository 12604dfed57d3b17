"""The C-ABI library loads and exports every symbol include/kda.h declares;
host-side validation rejects bad calls before any launch (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    src = open(os.path.join(ROOT, "include", "kda.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_documented_entry_points():
    names = header_functions()
    for n in ("kda_chunk_fwd", "kda_decode_step", "kda_layer_fwd", "kda_chunk_fwd_workspace"):
        assert n in names


def test_library_exports_every_declared_symbol(kda):
    lib = ctypes.CDLL(kda.LIB_PATH)
    for name in header_functions():
        assert hasattr(lib, name), name
    assert set(kda.SYMBOLS) == set(header_functions())


def test_status_strings_and_head_dim(kda):
    lib = kda.lib()
    assert lib.kda_head_dim() == 128
    assert lib.kda_status_string(0) == b"KDA_OK"
    assert lib.kda_status_string(5) == b"KDA_ERR_TIMEOUT"
    assert lib.kda_status_string(99) == b"KDA_ERR_UNKNOWN"


def test_workspace_queries(kda):
    assert kda.chunk_fwd_workspace_bytes(1, 65536, 16) > 0
    # the segment scan needs per-segment states only when few (sequence, head) pairs
    few = kda.chunk_fwd_workspace_bytes(1, 65536, 16)
    many = kda.chunk_fwd_workspace_bytes(64, 1024, 16)
    assert few > 16 * 128 * 128 * 4 and many < few
    assert kda.chunk_fwd_workspace_bytes(1, 256, 2, 0, kda.KDA_FP32) >= 3 * 256 * 2 * 128 * 2
    assert kda.layer_fwd_workspace_bytes(65536, 2048, 16, 128, 8) > 65536 * 6416 * 2


def test_segment_plan_on_148_sms(kda):
    """Host-side plan (no device here: the library assumes a B200's 148 SMs).  With
    P = sequences x heads <= 148/3 pairs, each sequence is cut into G = 148 // P equal
    segments of L = ceil((chunks + 1) / G) chunks (the last holds the rest): one CTA per
    segment and pair in each phase.  With more pairs every (sequence, head) of a dense
    call runs whole; packed calls of at most 64 sequences longer than 16 chunks in all
    are cut on the device (the balanced plan), which the query reports as -1."""
    # B=1 H=16 T=65536: 1024 chunks, G = 9, L = ceil(1025 / 9) = 114 chunks
    assert kda.chunk_fwd_segments(1, 65536, 16) == (114 * 64, 114 * 64)
    # T=16384: 256 chunks, L = ceil(257 / 9) = 29
    assert kda.chunk_fwd_segments(1, 16384, 16) == (29 * 64, 29 * 64)
    # H=32, one sequence: G = 4, L = ceil(1025 / 4) = 257
    assert kda.chunk_fwd_segments(1, 65536, 32) == (257 * 64, 257 * 64)
    # 256 or 50 pairs (> 148 / 3): no segment scan
    assert kda.chunk_fwd_segments(16, 4096, 16) == (0, 0)
    assert kda.chunk_fwd_segments(1, 65536, 50) == (0, 0)
    # packed sequences count as separate pairs: 8 sequences x 16 heads = 128 pairs, so
    # the plan is made on the device from the lengths (balanced)
    assert kda.chunk_fwd_segments(1, 65536, 16, 8) == (-1, -1)
    # ... unless they are too many (> 64) or too short (16 chunks in all) to cut
    assert kda.chunk_fwd_segments(1, 65536, 16, 65) == (0, 0)
    assert kda.chunk_fwd_segments(1, 1024, 16, 8) == (0, 0)
    assert kda.chunk_fwd_segments(1, 1025, 16, 8) == (-1, -1)
    # its workspace holds one product image per chunk of the call and head, and the
    # per-segment states of at most N + ceil((chunks + N) / 16) segments; the minimal
    # workspace (the call then runs unsegmented) holds neither
    full = kda.lib().kda_chunk_fwd_workspace(1, 65536, 16, 8, 0, 0)
    small = kda.lib().kda_chunk_fwd_workspace_min(1, 65536, 16, 8, 0, 0)
    assert full - small >= (1024 + 8) * 16 * 67584 + 3 * (8 + 65) * 16 * 128 * 128 * 4
    assert small < 4096
    # too short to pay for the map pass: fewer than 3 segments' worth of chunks
    assert kda.chunk_fwd_segments(1, 64, 49) == (0, 0)
    # the product images only fit the full workspace; the minimal one runs the same plan
    lib = kda.lib()
    full = lib.kda_chunk_fwd_workspace(1, 65536, 16, 0, 0, 0)
    small = lib.kda_chunk_fwd_workspace_min(1, 65536, 16, 0, 0, 0)
    assert full - small >= 1024 * 16 * 67584 and small > 3 * 10 * 16 * 128 * 128 * 4
    assert lib.kda_chunk_fwd_workspace(16, 4096, 16, 0, 0, 0) == lib.kda_chunk_fwd_workspace_min(16, 4096, 16, 0, 0, 0)


def _bad_chunk(kda, **over):
    lib = kda.lib()
    a = dict(q=1 << 20, k=1 << 20, v=1 << 20, g=1 << 20, beta=1 << 20, init=None, fin=None, o=2 << 20,
             cu=None, nseq=0, B=1, T=64, H=2, dtype=0, scale=1.0, l2=0, ws=None, wsb=0, stream=None)
    a.update(over)
    return lib.kda_chunk_fwd(a["q"], a["k"], a["v"], a["g"], a["beta"], a["init"], a["fin"], a["o"], a["cu"],
                             a["nseq"], a["B"], a["T"], a["H"], a["dtype"], a["scale"], a["l2"], a["ws"], a["wsb"],
                             a["stream"])


def test_chunk_validation_rejects_before_launch(kda):
    assert _bad_chunk(kda, dtype=7) == kda.KDA_ERR_INVALID_ARG
    assert _bad_chunk(kda, B=-1) == kda.KDA_ERR_INVALID_ARG
    assert _bad_chunk(kda, q=None) == kda.KDA_ERR_INVALID_ARG
    assert _bad_chunk(kda, q=(1 << 20) + 4) == kda.KDA_ERR_INVALID_ARG        # misaligned
    assert _bad_chunk(kda, o=1 << 20) == kda.KDA_ERR_INVALID_ARG              # o aliases q
    assert _bad_chunk(kda, cu=1 << 21, nseq=2, B=2) == kda.KDA_ERR_INVALID_ARG  # varlen needs B == 1
    assert _bad_chunk(kda, nseq=3) == kda.KDA_ERR_INVALID_ARG                 # dense needs num_seqs == 0
    assert _bad_chunk(kda, ws=(1 << 22) + 16, wsb=1 << 20) == kda.KDA_ERR_INVALID_ARG  # workspace alignment
    assert b"aligned" in kda.lib().kda_last_error()


def test_decode_validation_rejects_before_launch(kda):
    lib = kda.lib()
    p = 1 << 20
    assert lib.kda_decode_step(p, p, p, p, p, None, p, 2, 2, 0, 1.0, 0, None) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_decode_step(p, p, p, p, p, p + 8, p, 2, 2, 0, 1.0, 0, None) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_decode_step(p, p, p, p, p, p, p, 2, 2, 9, 1.0, 0, None) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_decode_step(p, p, p, p, p, p, p, 0, 2, 0, 1.0, 0, None) == kda.KDA_OK  # empty: no launch


def test_layer_validation_rejects_before_launch(kda):
    lib = kda.lib()
    w = kda.LayerWeights(1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20, 2048, 16, 128)
    p, y = 1 << 20, 1 << 22
    assert lib.kda_layer_fwd(p, None, 1 << 21, 8, 64, None, None, None, None, y, None, 0, None) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_layer_fwd(p, ctypes.byref(w), None, 8, 64, None, None, None, None, y, None, 0, None) == \
        kda.KDA_ERR_INVALID_ARG
    # misaligned conv cache
    assert lib.kda_layer_fwd(p, ctypes.byref(w), 1 << 21, 8, 64, None, None, p + 2, None, y, None, 0, None) == \
        kda.KDA_ERR_INVALID_ARG
    w.d_model = 2047
    assert lib.kda_layer_fwd(p, ctypes.byref(w), 1 << 21, 8, 64, None, None, None, None, y, None, 0, None) == \
        kda.KDA_ERR_UNSUPPORTED


def test_layer_decode_validation_rejects_before_launch(kda):
    lib = kda.lib()
    w = kda.LayerWeights(1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20, 2048, 16, 128)
    p = 1 << 20
    assert lib.kda_layer_decode(p, None, p, p, p, 4, 1, None, 0, None) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_layer_decode(p, ctypes.byref(w), None, p, p, 4, 1, None, 0, None) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_layer_decode(p, ctypes.byref(w), p, p + 4, p, 4, 1, None, 0, None) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_layer_decode(p, ctypes.byref(w), p, p, p, -1, 1, None, 0, None) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_layer_decode(p, ctypes.byref(w), p, p, p, 0, 1, None, 0, None) == kda.KDA_OK  # nothing to do
    assert kda.layer_decode_workspace_bytes(4, 1, 2048, 16, 128) > 0


def test_recurrent_validation_rejects_before_launch(kda):
    lib = kda.lib()
    p = 1 << 20
    assert lib.kda_recurrent_fwd(p, p, p, p, p, None, p + 256, 2, 3, 2, 0, 1.0, 0, None) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_recurrent_fwd(p, p, p, p, p, p, p, 2, 3, 2, 0, 1.0, 0, None) == kda.KDA_ERR_INVALID_ARG  # o aliases q
    assert lib.kda_recurrent_fwd(p, p, p, p, p, p, p + 256, 2, 3, 2, 7, 1.0, 0, None) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_recurrent_fwd(p, p, p, p, p, p, p + 256, 2, 0, 2, 0, 1.0, 0, None) == kda.KDA_OK  # T = 0


def test_gdn_validation_rejects_before_launch(kda):
    lib = kda.lib()
    p = 1 << 20
    assert lib.kda_gdn_chunk_fwd(p, p, p, p, p, None, None, p + 256, None, 3, 1, 64, 2, 0, 1.0, 0, None, 0,
                                 None) == kda.KDA_ERR_INVALID_ARG  # num_seqs without cu_seqlens
    assert lib.kda_gdn_chunk_fwd(p, p, p, p, p, None, None, p, None, 0, 1, 64, 2, 0, 1.0, 0, None, 0,
                                 None) == kda.KDA_ERR_INVALID_ARG  # o aliases q
