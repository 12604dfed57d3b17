"""Kimi Delta Attention (KDA) on B200 -- thin Python binding of libkda.so.

Every function here only marshals arguments (device pointers, sizes, the
current CUDA stream) into the C ABI declared in ``include/kda.h``; every step
of the computation runs in the library's CUDA kernels.  PyTorch is used for
device memory and streams only.  There is no CPU fallback: if the compiled
library is missing or fails to load, importing this package raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# KDA_LIB may point at another build of the same library (e.g. an instrumented one).
LIB_PATH = os.environ.get("KDA_LIB") or os.path.join(_HERE, "libkda.so")

KDA_OK, KDA_ERR_INVALID_ARG, KDA_ERR_UNSUPPORTED, KDA_ERR_WORKSPACE, KDA_ERR_CUDA, KDA_ERR_TIMEOUT = range(6)
KDA_BF16, KDA_FP32 = 0, 1
HEAD_DIM = 128

# Exported symbols of include/kda.h (checked by the ABI tests).
SYMBOLS = (
    "kda_status_string", "kda_head_dim", "kda_last_error", "kda_device_status",
    "kda_chunk_fwd_workspace", "kda_chunk_fwd", "kda_decode_step",
    "kda_layer_fwd_workspace", "kda_layer_fwd", "kda_set_trace_events", "kda_chunk_fwd_noalloc",
    "kda_gdn_chunk_fwd", "kda_recurrent_fwd", "kda_layer_decode_workspace", "kda_layer_decode",
    "kda_dplr_chunk_fwd_workspace", "kda_dplr_chunk_fwd", "kda_recurrent_bwd_workspace", "kda_recurrent_bwd",
    "kda_chunk_fwd_segment_tokens", "kda_chunk_fwd_workspace_min", "kda_debug_fault_injection",
    "kda_linear_bf16", "kda_chunk_fwd_plan_items",
)


class KDAError(RuntimeError):
    def __init__(self, code: int, where: str, detail: str):
        self.code = code
        super().__init__(f"{where}: {_lib.kda_status_string(code).decode()} ({detail})")


class LayerWeights(ctypes.Structure):
    _fields_ = [("W_in", ctypes.c_void_p), ("W_aup", ctypes.c_void_p), ("W_gup", ctypes.c_void_p),
                ("conv_w", ctypes.c_void_p), ("norm_w", ctypes.c_void_p), ("W_o", ctypes.c_void_p),
                ("d_model", ctypes.c_int), ("H", ctypes.c_int), ("rank", ctypes.c_int)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libkda.so not built ({LIB_PATH}); run __graft_entry__.build()")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.kda_status_string.argtypes = [i]
    lib.kda_status_string.restype = ctypes.c_char_p
    lib.kda_head_dim.restype = i
    lib.kda_last_error.restype = ctypes.c_char_p
    lib.kda_device_status.argtypes = [vp]
    lib.kda_device_status.restype = i
    lib.kda_chunk_fwd_workspace.argtypes = [i, i, i, i, i, i]
    lib.kda_chunk_fwd_workspace.restype = sz
    lib.kda_chunk_fwd_workspace_min.argtypes = [i, i, i, i, i, i]
    lib.kda_chunk_fwd_workspace_min.restype = sz
    lib.kda_chunk_fwd_segment_tokens.argtypes = [i, i, i, i, ctypes.POINTER(ctypes.c_int)]
    lib.kda_chunk_fwd_segment_tokens.restype = i
    lib.kda_chunk_fwd_plan_items.argtypes = [vp, i, i, i, i, ctypes.POINTER(ctypes.c_int), i]
    lib.kda_chunk_fwd_plan_items.restype = i
    lib.kda_chunk_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp, sz, vp]
    lib.kda_chunk_fwd.restype = i
    lib.kda_gdn_chunk_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp, sz, vp]
    lib.kda_gdn_chunk_fwd.restype = i
    lib.kda_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, f, i, vp]
    lib.kda_decode_step.restype = i
    lib.kda_recurrent_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, vp]
    lib.kda_recurrent_fwd.restype = i
    lib.kda_dplr_chunk_fwd_workspace.argtypes = [i, i, i, i, i]
    lib.kda_dplr_chunk_fwd_workspace.restype = sz
    lib.kda_dplr_chunk_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, vp, sz, vp]
    lib.kda_dplr_chunk_fwd.restype = i
    lib.kda_recurrent_bwd_workspace.argtypes = [i, i, i]
    lib.kda_recurrent_bwd_workspace.restype = sz
    lib.kda_recurrent_bwd.argtypes = [vp] * 14 + [i, i, i, i, f, vp, sz, vp]
    lib.kda_recurrent_bwd.restype = i
    lib.kda_layer_fwd_workspace.argtypes = [i, i, i, i, i]
    lib.kda_layer_fwd_workspace.restype = sz
    lib.kda_layer_fwd.argtypes = [vp, ctypes.POINTER(LayerWeights), vp, i, i, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.kda_layer_fwd.restype = i
    lib.kda_layer_decode_workspace.argtypes = [i, i, i, i, i]
    lib.kda_layer_decode_workspace.restype = sz
    lib.kda_layer_decode.argtypes = [vp, ctypes.POINTER(LayerWeights), vp, vp, vp, i, i, vp, sz, vp]
    lib.kda_layer_decode.restype = i
    lib.kda_linear_bf16.argtypes = [vp, i, vp, i, vp, i, i, i, i, vp]
    lib.kda_linear_bf16.restype = i
    lib.kda_debug_fault_injection.argtypes = [ctypes.c_longlong, i]
    lib.kda_debug_fault_injection.restype = i
    lib.kda_set_trace_events.argtypes = [vp, i]
    lib.kda_set_trace_events.restype = i
    return lib


_lib = _load()


def lib():
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _check(rc: int, where: str):
    if rc != KDA_OK:
        raise KDAError(rc, where, _lib.kda_last_error().decode())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return KDA_BF16
    if t.dtype == torch.float32:
        return KDA_FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


def device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    s = ctypes.c_void_p(stream if stream is not None else torch.cuda.current_stream().cuda_stream)
    return _lib.kda_device_status(s)


def debug_fault_injection(wait_limit_cycles=0, skip_chunk=-1):
    """Failure-test hook (``kda_debug_fault_injection``): bound of every device-side
    wait in SM cycles (0 = the default) and a chunk whose input load the chunk
    kernels skip (-1 = none).  Device-global; for tests only."""
    _check(_lib.kda_debug_fault_injection(int(wait_limit_cycles), int(skip_chunk)), "kda_debug_fault_injection")


def set_trace_events(events):
    """Record 5 caller-owned torch.cuda.Event around the kernels of later
    chunk_fwd calls (see kda_set_trace_events); None stops."""
    global _trace_keep
    if events is None:
        _trace_keep = None
        _check(_lib.kda_set_trace_events(None, 0), "kda_set_trace_events")
        return
    for e in events:  # torch creates the CUDA event lazily, on its first record
        if e.cuda_event == 0:
            e.record()
    arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    _trace_keep = (arr, events)
    _check(_lib.kda_set_trace_events(arr, len(events)), "kda_set_trace_events")


_trace_keep = None


def chunk_fwd_segments(B, T, H, num_seqs=0):
    """(first segment tokens, following segment tokens) of a kda_chunk_fwd call; (0, 0) if unsegmented,
    (-1, -1) if the device plans the cuts from cu_seqlens (see chunk_fwd_plan)."""
    mid = ctypes.c_int(0)
    first = int(_lib.kda_chunk_fwd_segment_tokens(B, T, H, num_seqs, ctypes.byref(mid)))
    return first, mid.value


def chunk_fwd_plan(workspace, B, T, H, num_seqs=0):
    """The segments the last chunk_fwd call with this workspace and these sizes
    ran: a list of (sequence, first token, end token, g, G).  Waits for the device."""
    cap = 4096
    rows = (ctypes.c_int * (5 * cap))()
    n = int(_lib.kda_chunk_fwd_plan_items(ctypes.c_void_p(workspace.data_ptr()), B, T, H, num_seqs, rows, cap))
    if n < 0:
        raise KDAError(KDA_ERR_CUDA, "kda_chunk_fwd_plan_items", "copy failed")
    return [tuple(rows[5 * i: 5 * i + 5]) for i in range(min(n, cap))]


def chunk_fwd_workspace_bytes(B, T, H, num_seqs=0, dtype=KDA_BF16, l2norm_qk=False) -> int:
    return int(_lib.kda_chunk_fwd_workspace(B, T, H, num_seqs, dtype, int(l2norm_qk)))


def chunk_fwd(q, k, v, g, beta, initial_state=None, cu_seqlens=None, scale=1.0, l2norm_qk=False,
              output_final_state=True, out=None, final_state=None, workspace=None):
    """Chunkwise KDA prefill (``kda_chunk_fwd``).

    q, k, v, g: [B,T,H,128] (or [1,Ttot,H,128] with cu_seqlens); beta: [B,T,H].
    Returns (o, final_state or None)."""
    return _chunk_call(_lib.kda_chunk_fwd, "kda_chunk_fwd", q, k, v, g, beta, initial_state, cu_seqlens, scale,
                       l2norm_qk, output_final_state, out, final_state, workspace)


def gdn_chunk_fwd(q, k, v, g, beta, initial_state=None, cu_seqlens=None, scale=1.0, l2norm_qk=False,
                  output_final_state=True, out=None, final_state=None, workspace=None):
    """Chunkwise prefill with a per-head scalar decay (``kda_gdn_chunk_fwd``).

    q, k, v: [B,T,H,128]; g, beta: [B,T,H] (or [1,Ttot,...] with cu_seqlens).
    Returns (o, final_state or None)."""
    return _chunk_call(_lib.kda_gdn_chunk_fwd, "kda_gdn_chunk_fwd", q, k, v, g, beta, initial_state, cu_seqlens,
                       scale, l2norm_qk, output_final_state, out, final_state, workspace)


def _chunk_call(fn, name, q, k, v, g, beta, initial_state, cu_seqlens, scale, l2norm_qk, output_final_state, out,
                final_state, workspace):
    B, T, H, D = q.shape
    if D != HEAD_DIM:
        raise ValueError("head dim must be 128")
    dt = _dtype_code(q)
    nseq = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    N = B if cu_seqlens is None else nseq
    o = out if out is not None else torch.empty_like(q)
    fs = final_state
    if fs is None and output_final_state:
        fs = torch.empty((N, H, D, D), device=q.device, dtype=torch.float32)
    # a caller's workspace is used as is if it has at least the minimal size (the library
    # then picks the schedule that fits); otherwise one of the full size is allocated
    wmin = int(_lib.kda_chunk_fwd_workspace_min(B, T, H, nseq, dt, int(l2norm_qk)))
    if workspace is None or workspace.numel() < wmin:
        workspace = torch.empty(max(chunk_fwd_workspace_bytes(B, T, H, nseq, dt, l2norm_qk), 1), device=q.device,
                                dtype=torch.uint8)
    wsz = workspace.numel()
    rc = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(initial_state), _ptr(fs), _ptr(o),
            _ptr(cu_seqlens), nseq, B, T, H, dt, float(scale), int(l2norm_qk), _ptr(workspace), wsz,
            _stream(q.device))
    _check(rc, name)
    return o, fs


def decode_step(q, k, v, g, beta, state, scale=1.0, l2norm_qk=False, out=None):
    """One recurrent KDA step (``kda_decode_step``); ``state`` [B,H,128,128] fp32 is updated in place."""
    B, H, D = q.shape
    if D != HEAD_DIM:
        raise ValueError("head dim must be 128")
    o = out if out is not None else torch.empty_like(q)
    rc = _lib.kda_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state), _ptr(o), B, H,
                              _dtype_code(q), float(scale), int(l2norm_qk), _stream(q.device))
    _check(rc, "kda_decode_step")
    return o


def dplr_chunk_fwd(q, k, v, a, b, g, beta, initial_state=None, cu_seqlens=None, scale=1.0,
                   output_final_state=True, out=None, final_state=None, workspace=None):
    """Untied DPLR chunked prefill (``kda_dplr_chunk_fwd``): S = (I - a b^T) Diag(e^g) S + beta k v^T.

    q, k, v, a, b, g: [B,T,H,128] (or [1,Ttot,H,128] with cu_seqlens); beta: [B,T,H].
    Returns (o, final_state or None)."""
    B, T, H, D = q.shape
    if D != HEAD_DIM:
        raise ValueError("head dim must be 128")
    dt = _dtype_code(q)
    nseq = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    N = B if cu_seqlens is None else nseq
    o = out if out is not None else torch.empty_like(q)
    fs = final_state
    if fs is None and output_final_state:
        fs = torch.empty((N, H, D, D), device=q.device, dtype=torch.float32)
    wsz = int(_lib.kda_dplr_chunk_fwd_workspace(B, T, H, nseq, dt))
    if workspace is None or workspace.numel() < wsz:
        workspace = torch.empty(max(wsz, 1), device=q.device, dtype=torch.uint8)
    rc = _lib.kda_dplr_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(g), _ptr(beta),
                                 _ptr(initial_state), _ptr(fs), _ptr(o), _ptr(cu_seqlens), nseq, B, T, H, dt,
                                 float(scale), _ptr(workspace), wsz, _stream(q.device))
    _check(rc, "kda_dplr_chunk_fwd")
    return o, fs


def recurrent_bwd(q, k, v, g, beta, d_o, initial_state=None, d_final_state=None, scale=1.0, workspace=None):
    """Gradients of the recurrence (``kda_recurrent_bwd``).  Returns (dq, dk, dv, dg, dbeta, d_initial_state),
    all fp32; q, k, v, d_o [B,T,H,128] (bf16 or fp32), g [B,T,H,128], beta [B,T,H]."""
    B, T, H, D = q.shape
    if D != HEAD_DIM:
        raise ValueError("head dim must be 128")
    dev = q.device
    dq, dk, dv, dg = (torch.empty((B, T, H, D), device=dev, dtype=torch.float32) for _ in range(4))
    db = torch.empty((B, T, H), device=dev, dtype=torch.float32)
    ds0 = torch.empty((B, H, D, D), device=dev, dtype=torch.float32)
    wsz = int(_lib.kda_recurrent_bwd_workspace(B, T, H))
    if workspace is None or workspace.numel() < wsz:
        workspace = torch.empty(max(wsz, 1), device=dev, dtype=torch.uint8)
    rc = _lib.kda_recurrent_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(initial_state), _ptr(d_o),
                                _ptr(d_final_state), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dg), _ptr(db), _ptr(ds0),
                                B, T, H, _dtype_code(q), float(scale), _ptr(workspace), wsz, _stream(dev))
    _check(rc, "kda_recurrent_bwd")
    return dq, dk, dv, dg, db, ds0


def recurrent_fwd(q, k, v, g, beta, state, scale=1.0, l2norm_qk=False, out=None):
    """Fused recurrent segment (``kda_recurrent_fwd``): q, k, v, g [B,T,H,128], beta [B,T,H];
    ``state`` [B,H,128,128] fp32 is updated in place.  Returns o [B,T,H,128]."""
    B, T, H, D = q.shape
    if D != HEAD_DIM:
        raise ValueError("head dim must be 128")
    o = out if out is not None else torch.empty_like(q)
    rc = _lib.kda_recurrent_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state), _ptr(o), B, T, H,
                                _dtype_code(q), float(scale), int(l2norm_qk), _stream(q.device))
    _check(rc, "kda_recurrent_fwd")
    return o


def linear(x, W, out=None):
    """y = x W^T (``kda_linear_bf16``): x [M, K] and W [N, K] bf16 with contiguous rows.
    Returns y [M, N] bf16 (a view with a row stride padded to 8 elements when N is not
    a multiple of 8)."""
    M, K = x.shape
    N = W.shape[0]
    if W.shape[1] != K or x.dtype != torch.bfloat16 or W.dtype != torch.bfloat16:
        raise ValueError("linear: x [M, K] and W [N, K] must be bf16")
    y = out if out is not None else torch.empty((M, (N + 7) // 8 * 8), device=x.device, dtype=torch.bfloat16)[:, :N]
    rc = _lib.kda_linear_bf16(_ptr(x), x.stride(0), _ptr(W), W.stride(0), _ptr(y), y.stride(0), M, N, K,
                              _stream(x.device))
    _check(rc, "kda_linear_bf16")
    return y


def pack_layer_weights(W: dict) -> dict:
    """Lay the layer weights out as the C ABI expects (W_in rows: q, k, v,
    a_down, g_down, b; conv taps for q, k, v stacked)."""
    W_in = torch.cat([W["W_q"], W["W_k"], W["W_v"], W["W_adown"], W["W_gdown"], W["W_b"]], dim=0).contiguous()
    conv = torch.cat([W["conv_q"], W["conv_k"], W["conv_v"]], dim=0).contiguous()
    return dict(W_in=W_in, W_aup=W["W_aup"].contiguous(), W_gup=W["W_gup"].contiguous(), conv_w=conv,
                norm_w=W["norm_w"].float().contiguous(), W_o=W["W_o"].contiguous(),
                d_model=W["W_q"].shape[1], H=W["W_q"].shape[0] // HEAD_DIM, rank=W["W_adown"].shape[0])


def layer_fwd_workspace_bytes(total_tokens, d_model, H, rank, num_seqs) -> int:
    return int(_lib.kda_layer_fwd_workspace(total_tokens, d_model, H, rank, num_seqs))


def _layer_weights(packed: dict, d_model: int) -> LayerWeights:
    return LayerWeights(packed["W_in"].data_ptr(), packed["W_aup"].data_ptr(), packed["W_gup"].data_ptr(),
                        packed["conv_w"].data_ptr(), packed["norm_w"].data_ptr(), packed["W_o"].data_ptr(),
                        d_model, packed["H"], packed["rank"])


def layer_fwd(x, packed: dict, cu_seqlens, initial_state=None, output_final_state=True, out=None,
              final_state=None, workspace=None, conv_state_in=None, output_conv_state=False, conv_state_out=None):
    """KDA layer forward (``kda_layer_fwd``).  x: [Ttot, d_model] bf16.

    Returns (y, final_state or None, conv_state or None); the conv state is
    [num_seqs, 3, 3*H*128] bf16 (the ShortConv cache)."""
    Ttot, d_model = x.shape
    H, rank = packed["H"], packed["rank"]
    nseq = cu_seqlens.numel() - 1
    y = out if out is not None else torch.empty_like(x)
    fs = final_state
    if fs is None and output_final_state:
        fs = torch.empty((nseq, H, HEAD_DIM, HEAD_DIM), device=x.device, dtype=torch.float32)
    cs = conv_state_out
    if cs is None and output_conv_state:
        cs = torch.empty((nseq, 3, 3 * H * HEAD_DIM), device=x.device, dtype=torch.bfloat16)
    lw = _layer_weights(packed, d_model)
    wsz = layer_fwd_workspace_bytes(Ttot, d_model, H, rank, nseq)
    if workspace is None or workspace.numel() < wsz:
        workspace = torch.empty(max(wsz, 1), device=x.device, dtype=torch.uint8)
    rc = _lib.kda_layer_fwd(_ptr(x), ctypes.byref(lw), _ptr(cu_seqlens), nseq, Ttot, _ptr(initial_state), _ptr(fs),
                            _ptr(conv_state_in), _ptr(cs), _ptr(y), _ptr(workspace), wsz, _stream(x.device))
    _check(rc, "kda_layer_fwd")
    return y, fs, cs


def layer_decode_workspace_bytes(B, T, d_model, H, rank) -> int:
    return int(_lib.kda_layer_decode_workspace(B, T, d_model, H, rank))


def layer_decode(x, packed: dict, conv_state, state, out=None, workspace=None):
    """KDA layer on T new tokens per sequence (``kda_layer_decode``).  x: [B, T, d_model] bf16;
    conv_state [B, 3, 3*H*128] bf16 and state [B, H, 128, 128] fp32 are updated in place."""
    B, T, d_model = x.shape
    H, rank = packed["H"], packed["rank"]
    y = out if out is not None else torch.empty_like(x)
    lw = _layer_weights(packed, d_model)
    wsz = layer_decode_workspace_bytes(B, T, d_model, H, rank)
    if workspace is None or workspace.numel() < wsz:
        workspace = torch.empty(max(wsz, 1), device=x.device, dtype=torch.uint8)
    rc = _lib.kda_layer_decode(_ptr(x), ctypes.byref(lw), _ptr(conv_state), _ptr(state), _ptr(y), B, T,
                               _ptr(workspace), wsz, _stream(x.device))
    _check(rc, "kda_layer_decode")
    return y
