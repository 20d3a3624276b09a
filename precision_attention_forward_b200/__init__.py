"""Python binding of liblpfa: MXFP8 varlen quantization and block-scaled attention forward.

Argument marshalling only: every step of the path runs in the library's CUDA kernels
(``liblpfa.so``, built in-tree for sm_100a). PyTorch provides device memory and streams.
Importing this package fails if the library has not been built; there is no CPU fallback.

The functions carry the C ABI's names (``include/lpfa.h``); the LP-FA4 README names
(``Mxfp8VarlenMeta.from_lengths``, ``quantize_mxfp8_varlen``,
``mxfp8_flash_attn_varlen_forward``) are provided as aliases.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np
import torch

_PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG_DIR, "liblpfa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        "liblpfa.so is not built; run `python precision_attention_forward_b200/build.py` "
        "(the library has no CPU fallback)")

_lib = ctypes.CDLL(LIB_PATH)

LPFA_OK, LPFA_ERR_INVALID_ARG, LPFA_ERR_UNSUPPORTED, LPFA_ERR_CUDA, LPFA_ERR_TIMEOUT = 0, 1, 2, 3, 4
_STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "CUDA", 4: "TIMEOUT"}
IN_DTYPES = {"bf16": 0, "fp32": 1}
SCALING_MODES = {"rceil": 0, "floor": 1}
PV_MODES = {"bf16": 0, "fp8": 1, "bf16v": 2, "mxfp8": 3}  # bf16v: BF16 V input, bf16 PV; mxfp8: block-scaled PV

# Symbols the header declares; the tests check that each one is exported.
EXPORTED_SYMBOLS = (
    "lpfa_meta_dev_ints", "lpfa_varlen_meta_fill_host", "lpfa_varlen_meta_from_lengths",
    "lpfa_scale_bytes", "lpfa_quantize_mxfp8_varlen", "lpfa_cast_e4m3", "lpfa_attn_fwd_varlen",
    "lpfa_device_status", "lpfa_last_error_message", "lpfa_version", "lpfa_attn_fwd_varlen_debug",
    "lpfa_attn_fwd_varlen_descaled", "lpfa_quantize_mxfp8_varlen_tokens", "lpfa_attn_bwd_varlen",
    "lpfa_attn_bwd_varlen_debug", "lpfa_attn_fwd_shared_q", "lpfa_dequantize_mxfp8_varlen",
    "lpfa_attn_fwd_workspace_bytes", "lpfa_attn_fwd_varlen_ws", "lpfa_attn_fwd_shared_q_ws",
    "lpfa_attn_fwd_varlen_noalloc",
)


class LpfaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"lpfa status {_STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class _Descale(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("seq_stride", ctypes.c_int64), ("head_stride", ctypes.c_int64)]


class _Meta(ctypes.Structure):
    _fields_ = [("num_seqs", ctypes.c_int32), ("total_tokens", ctypes.c_int32),
                ("total_scale_blocks", ctypes.c_int32), ("max_seqlen", ctypes.c_int32),
                ("dev", ctypes.c_void_p)]


_vp, _i32, _i64, _f32p = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p
_lib.lpfa_meta_dev_ints.argtypes = [_i32]
_lib.lpfa_meta_dev_ints.restype = ctypes.c_size_t
_lib.lpfa_varlen_meta_fill_host.argtypes = [_vp, _i32, _vp, ctypes.POINTER(_Meta)]
_lib.lpfa_varlen_meta_fill_host.restype = ctypes.c_int
_lib.lpfa_varlen_meta_from_lengths.argtypes = [_vp, _i32, ctypes.POINTER(_Meta), _vp]
_lib.lpfa_varlen_meta_from_lengths.restype = ctypes.c_int
_lib.lpfa_scale_bytes.argtypes = [ctypes.POINTER(_Meta), _i32]
_lib.lpfa_scale_bytes.restype = ctypes.c_size_t
_lib.lpfa_quantize_mxfp8_varlen.argtypes = [_vp, ctypes.c_int, _i64, _i64, _i32, _i32, ctypes.POINTER(_Meta),
                                            ctypes.c_int, _vp, _vp, _vp]
_lib.lpfa_quantize_mxfp8_varlen.restype = ctypes.c_int
_lib.lpfa_quantize_mxfp8_varlen_tokens.argtypes = _lib.lpfa_quantize_mxfp8_varlen.argtypes
_lib.lpfa_quantize_mxfp8_varlen_tokens.restype = ctypes.c_int
_lib.lpfa_attn_bwd_varlen.argtypes = ([_vp] * 9 + [ctypes.POINTER(_Meta), ctypes.POINTER(_Meta), _i32, _i32] +
                                      [ctypes.POINTER(_Descale)] * 3 + [_vp] * 5 + [_i32, _vp])
_lib.lpfa_attn_bwd_varlen.restype = ctypes.c_int
_lib.lpfa_attn_bwd_varlen_debug.argtypes = list(_lib.lpfa_attn_bwd_varlen.argtypes) + [_i32]
_lib.lpfa_attn_bwd_varlen_debug.restype = ctypes.c_int
_lib.lpfa_cast_e4m3.argtypes = [_vp, _i64, _i64, _i64, _i32, _i32, _vp, _vp]
_lib.lpfa_cast_e4m3.restype = ctypes.c_int
_lib.lpfa_attn_fwd_varlen.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(_Meta), ctypes.POINTER(_Meta),
                                      _i32, _i32, ctypes.c_int, _f32p, _f32p, _f32p, _vp, _vp, _vp]
_lib.lpfa_attn_fwd_varlen.restype = ctypes.c_int
_lib.lpfa_attn_fwd_varlen_debug.argtypes = list(_lib.lpfa_attn_fwd_varlen.argtypes) + [_i32]
_lib.lpfa_attn_fwd_varlen_descaled.argtypes = (list(_lib.lpfa_attn_fwd_varlen.argtypes[:11]) +
                                               [ctypes.POINTER(_Descale)] * 3 + [_vp, _vp, _vp])
_lib.lpfa_attn_fwd_varlen_descaled.restype = ctypes.c_int
_lib.lpfa_attn_fwd_shared_q.argtypes = _lib.lpfa_attn_fwd_varlen_descaled.argtypes
_lib.lpfa_attn_fwd_shared_q.restype = ctypes.c_int
_lib.lpfa_attn_fwd_varlen_debug.restype = ctypes.c_int
_lib.lpfa_attn_fwd_varlen_ws.argtypes = (list(_lib.lpfa_attn_fwd_varlen_descaled.argtypes[:16]) +
                                         [_vp, ctypes.c_size_t, _vp])
_lib.lpfa_attn_fwd_varlen_ws.restype = ctypes.c_int
_lib.lpfa_attn_fwd_shared_q_ws.argtypes = _lib.lpfa_attn_fwd_varlen_ws.argtypes
_lib.lpfa_attn_fwd_shared_q_ws.restype = ctypes.c_int
_lib.lpfa_attn_fwd_varlen_noalloc.argtypes = _lib.lpfa_attn_fwd_varlen_descaled.argtypes
_lib.lpfa_attn_fwd_varlen_noalloc.restype = ctypes.c_int
_lib.lpfa_attn_fwd_workspace_bytes.argtypes = [ctypes.POINTER(_Meta), _i32, ctypes.c_int]
_lib.lpfa_attn_fwd_workspace_bytes.restype = ctypes.c_size_t
_lib.lpfa_dequantize_mxfp8_varlen.argtypes = [_vp, _vp, ctypes.POINTER(_Meta), _i32, _i32, _vp, _vp]
_lib.lpfa_dequantize_mxfp8_varlen.restype = ctypes.c_int
_lib.lpfa_device_status.argtypes = [_vp, ctypes.POINTER(_i32)]
_lib.lpfa_device_status.restype = ctypes.c_int
_lib.lpfa_last_error_message.argtypes = []
_lib.lpfa_last_error_message.restype = ctypes.c_char_p
_lib.lpfa_version.argtypes = []
_lib.lpfa_version.restype = ctypes.c_char_p


def _check(status: int) -> None:
    if status != LPFA_OK:
        raise LpfaError(status, _lib.lpfa_last_error_message().decode(errors="replace"))


def _stream_ptr(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def lpfa_version() -> str:
    return _lib.lpfa_version().decode()


class VarlenMeta:
    """Packed varlen metadata: host scalars plus a device int32 buffer (cu_seqlens | scale_off)."""

    def __init__(self, lengths, c_meta: _Meta, dev: Optional[torch.Tensor], host_ints: np.ndarray):
        self.lengths = np.asarray(lengths, dtype=np.int32)
        self._c = c_meta
        self.dev = dev
        self.host_ints = host_ints

    num_seqs = property(lambda self: self._c.num_seqs)
    total_tokens = property(lambda self: self._c.total_tokens)
    total_scale_blocks = property(lambda self: self._c.total_scale_blocks)
    max_seqlen = property(lambda self: self._c.max_seqlen)

    @property
    def cu_seqlens(self) -> np.ndarray:
        return self.host_ints[: self.num_seqs + 1]

    @property
    def scale_off(self) -> np.ndarray:
        return self.host_ints[self.num_seqs + 1:]

    def scale_bytes(self, heads: int) -> int:
        return int(_lib.lpfa_scale_bytes(ctypes.byref(self._c), heads))

    @classmethod
    def from_lengths(cls, lengths: Sequence[int], device="cuda", stream=None) -> "VarlenMeta":
        return lpfa_varlen_meta_from_lengths(lengths, device=device, stream=stream)


def lpfa_varlen_meta_fill_host(lengths: Sequence[int]) -> VarlenMeta:
    """Host-only metadata (no device buffer); usable without a GPU."""
    lens = np.ascontiguousarray(np.asarray(lengths, dtype=np.int32))
    n = int(lens.size)
    host = np.zeros(max(int(_lib.lpfa_meta_dev_ints(n)), 1), dtype=np.int32)
    m = _Meta()
    _check(_lib.lpfa_varlen_meta_fill_host(lens.ctypes.data if n else None, n, host.ctypes.data, ctypes.byref(m)))
    return VarlenMeta(lens, m, None, host)


def lpfa_varlen_meta_from_lengths(lengths: Sequence[int], device="cuda", stream=None) -> VarlenMeta:
    lens = np.ascontiguousarray(np.asarray(lengths, dtype=np.int32))
    n = int(lens.size)
    host_meta = lpfa_varlen_meta_fill_host(lens)
    dev = torch.empty(int(_lib.lpfa_meta_dev_ints(n)), dtype=torch.int32, device=device)
    m = _Meta()
    m.dev = dev.data_ptr()
    with torch.cuda.device(dev.device):
        _check(_lib.lpfa_varlen_meta_from_lengths(lens.ctypes.data, n, ctypes.byref(m), _stream_ptr(stream)))
    return VarlenMeta(lens, m, dev, host_meta.host_ints)


def _strides(x: torch.Tensor):
    if x.dim() != 3 or x.shape[2] != 128 or x.stride(2) != 1:
        raise ValueError("expected a (tokens, heads, 128) tensor with a contiguous last dimension")
    return x.stride(0), x.stride(1)


def lpfa_quantize_mxfp8_varlen(x: torch.Tensor, meta: VarlenMeta, scaling_mode: str = "rceil",
                               payload: Optional[torch.Tensor] = None, scales: Optional[torch.Tensor] = None,
                               stream=None, orientation: str = "head_dim"):
    """Quantize packed (T, H, 128) bf16/fp32 to (payload uint8 (T,H,128), scales uint8 (blocks*H*512,)).

    orientation "head_dim": one scale per 32 elements along head_dim (Q and K, and V in bf16 PV
    mode); "tokens": one scale per 32 tokens of a channel (V in mxfp8 PV mode).
    """
    if orientation not in ("head_dim", "tokens"):
        raise ValueError("orientation must be 'head_dim' or 'tokens'")
    dt = {torch.bfloat16: "bf16", torch.float32: "fp32"}.get(x.dtype)
    if dt is None:
        raise ValueError("x must be bf16 or fp32")
    if scaling_mode not in SCALING_MODES:
        raise ValueError("scaling_mode must be 'rceil' or 'floor'")
    ts, hs = _strides(x)
    T, H = x.shape[0], x.shape[1]
    if T != meta.total_tokens:
        raise ValueError("x has %d tokens but the metadata describes %d" % (T, meta.total_tokens))
    if payload is None:
        payload = torch.empty((T, H, 128), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(meta.scale_bytes(H), dtype=torch.uint8, device=x.device)
    with torch.cuda.device(x.device):
        fn = _lib.lpfa_quantize_mxfp8_varlen if orientation == "head_dim" else _lib.lpfa_quantize_mxfp8_varlen_tokens
        _check(fn(x.data_ptr(), IN_DTYPES[dt], ts, hs, H, 128, ctypes.byref(meta._c),
                  SCALING_MODES[scaling_mode], payload.data_ptr(), scales.data_ptr(), _stream_ptr(stream)))
    return payload, scales


def lpfa_cast_e4m3(v: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Unscaled E4M3 cast of a bf16 (T, H, 128) tensor (fp8 PV mode V)."""
    if v.dtype != torch.bfloat16:
        raise ValueError("v must be bf16")
    ts, hs = _strides(v)
    T, H = v.shape[0], v.shape[1]
    if out is None:
        out = torch.empty((T, H, 128), dtype=torch.uint8, device=v.device)
    with torch.cuda.device(v.device):
        _check(_lib.lpfa_cast_e4m3(v.data_ptr(), ts, hs, T, H, 128, out.data_ptr(), _stream_ptr(stream)))
    return out


def descale_strides(t: torch.Tensor, num_seqs: int, heads: int):
    """(seq_stride, head_stride) in elements of a descale tensor indexed by (sequence, head).

    Accepted shapes (vLLM #63232: per-tensor and per-head scales keep their descale tensors;
    FA4's descale views are (batch, kv_heads)): one element (per tensor), (heads,) (per head),
    and (S, Hd) with S in {1, num_seqs}, Hd in {1, heads}; size-1 axes broadcast (stride 0).
    """
    if t.dtype != torch.float32:
        raise ValueError("a descale must be a float32 tensor")
    if t.numel() == 1:
        return 0, 0
    if t.dim() == 1 and t.shape[0] == heads:
        return 0, t.stride(0)
    if t.dim() == 2 and t.shape[0] in (1, num_seqs) and t.shape[1] in (1, heads):
        return (t.stride(0) if t.shape[0] > 1 else 0), (t.stride(1) if t.shape[1] > 1 else 0)
    raise ValueError("a descale has one element, shape (heads,) or (num_seqs or 1, heads or 1); got %s"
                     % (tuple(t.shape),))


def lpfa_attn_fwd_varlen(q: torch.Tensor, q_sf: torch.Tensor, k: torch.Tensor, k_sf: torch.Tensor,
                         v: torch.Tensor, v_sf: Optional[torch.Tensor], meta_q: VarlenMeta, meta_k: VarlenMeta,
                         pv_mode: str = "bf16", q_descale: Optional[torch.Tensor] = None,
                         k_descale: Optional[torch.Tensor] = None, v_descale: Optional[torch.Tensor] = None,
                         out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None, stream=None,
                         debug_flags: int = 0, workspace=True):
    """Block-scaled attention forward; returns (out bf16 (Tq,H,128), lse fp32 (H,Tq)).

    q/k/v_descale: None (exactly 1.0), a one-element tensor (per tensor), (H,) (per head) or
    (S, H) (per sequence and head), float32 on the device; see descale_strides.
    workspace: where the bf16 PV mode converts V to BF16 once (lpfa_attn_fwd_varlen_ws): True
    allocates it, a uint8 device tensor of at least lpfa_attn_fwd_workspace_bytes bytes is used as
    is, False converts V tiles inside the attention kernel instead (same bits). Other modes ignore it.
    (An allocated workspace is recorded on `stream` when that is a torch.cuda.Stream; with a raw
    stream handle other than the current stream, pass a workspace tensor that outlives the work.)
    debug_flags != 0 goes through lpfa_attn_fwd_varlen_debug (test hook, see include/lpfa.h),
    which takes per-tensor descales only and no workspace.
    """
    if pv_mode not in PV_MODES:
        raise ValueError("pv_mode must be 'bf16', 'fp8', 'bf16v' or 'mxfp8'")
    for name, t in (("q", q), ("k", k), ("v", v)):
        want = torch.bfloat16 if (name == "v" and pv_mode == "bf16v") else torch.uint8
        if t.dtype != want or t.dim() != 3 or not t.is_contiguous():
            raise ValueError("%s must be a contiguous %s (tokens, heads, 128) tensor" % (name, want))
    Tq, H = q.shape[0], q.shape[1]
    descs = []
    for name, t in (("q_descale", q_descale), ("k_descale", k_descale), ("v_descale", v_descale)):
        if t is None:
            descs.append(_Descale(None, 0, 0))
            continue
        ss, hs = descale_strides(t, meta_q.num_seqs, H)
        if debug_flags and (ss or hs):
            raise ValueError("the debug entry point takes per-tensor descales only")
        if t.device != q.device:
            raise ValueError("%s must be on the device of q" % name)
        descs.append(_Descale(t.data_ptr(), ss, hs))
    if out is None:
        out = torch.empty((Tq, H, 128), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((H, Tq), dtype=torch.float32, device=q.device)
    args = (q.data_ptr(), q_sf.data_ptr(), k.data_ptr(), k_sf.data_ptr(), v.data_ptr(), _ptr(v_sf),
            ctypes.byref(meta_q._c), ctypes.byref(meta_k._c), H, 128, PV_MODES[pv_mode],
            _ptr(q_descale), _ptr(k_descale), _ptr(v_descale), out.data_ptr(), lse.data_ptr(),
            _stream_ptr(stream))
    ws = None if debug_flags else _workspace(workspace, meta_k, H, pv_mode, q.device, stream)
    with torch.cuda.device(q.device):
        if debug_flags:
            _check(_lib.lpfa_attn_fwd_varlen_debug(*args, debug_flags))
        elif ws is not None:
            _check(_lib.lpfa_attn_fwd_varlen_ws(*args[:11], ctypes.byref(descs[0]), ctypes.byref(descs[1]),
                                                ctypes.byref(descs[2]), out.data_ptr(), lse.data_ptr(),
                                                ws.data_ptr(), ctypes.c_size_t(ws.numel()), _stream_ptr(stream)))
        else:
            _check(_lib.lpfa_attn_fwd_varlen_descaled(*args[:11], ctypes.byref(descs[0]), ctypes.byref(descs[1]),
                                                      ctypes.byref(descs[2]), *args[14:]))
    return out, lse


def lpfa_attn_fwd_workspace_bytes(meta_k: VarlenMeta, heads: int, pv_mode: str) -> int:
    """Workspace bytes the bf16 PV mode needs (Tk * H * 256); 0 for the other modes."""
    return int(_lib.lpfa_attn_fwd_workspace_bytes(ctypes.byref(meta_k._c), heads, PV_MODES[pv_mode]))


def _workspace(workspace, meta_k: VarlenMeta, heads: int, pv_mode: str, device, stream=None):
    """The workspace tensor for a forward call, or None (in-kernel V conversion / not needed)."""
    need = lpfa_attn_fwd_workspace_bytes(meta_k, heads, pv_mode)
    if need == 0 or workspace is False or workspace is None:
        return None
    if workspace is True:
        ws = torch.empty(need, dtype=torch.uint8, device=device)
        if isinstance(stream, torch.cuda.Stream):
            ws.record_stream(stream)  # the kernels read it on that stream after this call returns
        return ws
    if not isinstance(workspace, torch.Tensor) or workspace.dtype != torch.uint8 or not workspace.is_contiguous():
        raise ValueError("workspace must be True, False or a contiguous uint8 device tensor")
    if workspace.numel() < need:
        raise ValueError("workspace has %d bytes; this call needs %d" % (workspace.numel(), need))
    return workspace


def lpfa_dequantize_mxfp8_varlen(payload: torch.Tensor, scales: torch.Tensor, meta: VarlenMeta,
                                 out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """MXFP8 (head_dim orientation) payload + scale storage -> BF16 (T, H, 128), exactly."""
    if payload.dtype != torch.uint8 or payload.dim() != 3 or not payload.is_contiguous():
        raise ValueError("payload must be a contiguous uint8 (tokens, heads, 128) tensor")
    T, H = payload.shape[0], payload.shape[1]
    if out is None:
        out = torch.empty((T, H, 128), dtype=torch.bfloat16, device=payload.device)
    if out.dtype != torch.bfloat16 or tuple(out.shape) != (T, H, 128) or not out.is_contiguous():
        raise ValueError("out must be a contiguous bf16 (tokens, heads, 128) tensor")
    with torch.cuda.device(payload.device):
        _check(_lib.lpfa_dequantize_mxfp8_varlen(payload.data_ptr(), scales.data_ptr(), ctypes.byref(meta._c), H,
                                                 128, out.data_ptr(), _stream_ptr(stream)))
    return out


def lpfa_attn_fwd_shared_q(q: torch.Tensor, q_sf: torch.Tensor, k: torch.Tensor, k_sf: torch.Tensor,
                           v: torch.Tensor, v_sf: Optional[torch.Tensor], meta_q: VarlenMeta, meta_k: VarlenMeta,
                           pv_mode: str = "bf16", q_descale: Optional[torch.Tensor] = None,
                           k_descale: Optional[torch.Tensor] = None, v_descale: Optional[torch.Tensor] = None,
                           out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None, stream=None,
                           workspace=True):
    """Shared-query forward (see include/lpfa.h): one query sequence (meta_q has one sequence of Lq
    tokens) attends to each of the n key/value sequences of meta_k. Returns (out bf16 (n*Lq,H,128),
    lse fp32 (H,n*Lq)); rows [i*Lq, (i+1)*Lq) belong to key/value sequence i. Descales and
    workspace as for lpfa_attn_fwd_varlen; descales are indexed by the key/value sequence."""
    if pv_mode not in PV_MODES:
        raise ValueError("pv_mode must be 'bf16', 'fp8', 'bf16v' or 'mxfp8'")
    if meta_q.num_seqs != 1:
        raise ValueError("a shared query set is one sequence")
    for name, t in (("q", q), ("k", k), ("v", v)):
        want = torch.bfloat16 if (name == "v" and pv_mode == "bf16v") else torch.uint8
        if t.dtype != want or t.dim() != 3 or not t.is_contiguous():
            raise ValueError("%s must be a contiguous %s (tokens, heads, 128) tensor" % (name, want))
    Lq, H = q.shape[0], q.shape[1]
    rows = Lq * meta_k.num_seqs
    descs = []
    for name, t in (("q_descale", q_descale), ("k_descale", k_descale), ("v_descale", v_descale)):
        if t is None:
            descs.append(_Descale(None, 0, 0))
            continue
        ss, hs = descale_strides(t, meta_k.num_seqs, H)
        if t.device != q.device:
            raise ValueError("%s must be on the device of q" % name)
        descs.append(_Descale(t.data_ptr(), ss, hs))
    if out is None:
        out = torch.empty((rows, H, 128), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((H, rows), dtype=torch.float32, device=q.device)
    if tuple(out.shape) != (rows, H, 128) or tuple(lse.shape) != (H, rows):
        raise ValueError("out must be (n*Lq, H, 128) and lse (H, n*Lq)")
    ws = _workspace(workspace, meta_k, H, pv_mode, q.device, stream)
    args = (q.data_ptr(), q_sf.data_ptr(), k.data_ptr(), k_sf.data_ptr(), v.data_ptr(), _ptr(v_sf),
            ctypes.byref(meta_q._c), ctypes.byref(meta_k._c), H, 128, PV_MODES[pv_mode], ctypes.byref(descs[0]),
            ctypes.byref(descs[1]), ctypes.byref(descs[2]), out.data_ptr(), lse.data_ptr())
    with torch.cuda.device(q.device):
        if ws is not None:
            _check(_lib.lpfa_attn_fwd_shared_q_ws(*args, ws.data_ptr(), ctypes.c_size_t(ws.numel()),
                                                  _stream_ptr(stream)))
        else:
            _check(_lib.lpfa_attn_fwd_shared_q(*args, _stream_ptr(stream)))
    return out, lse


def lpfa_attn_bwd_varlen(q: torch.Tensor, q_sf: torch.Tensor, k: torch.Tensor, k_sf: torch.Tensor,
                         v: torch.Tensor, v_sf: torch.Tensor, out: torch.Tensor, dout: torch.Tensor,
                         lse: torch.Tensor, meta_q: VarlenMeta, meta_k: VarlenMeta,
                         q_descale: Optional[torch.Tensor] = None, k_descale: Optional[torch.Tensor] = None,
                         v_descale: Optional[torch.Tensor] = None, output_mxfp8_dkv: bool = False, stream=None,
                         dq: Optional[torch.Tensor] = None, dk: Optional[torch.Tensor] = None,
                         dv: Optional[torch.Tensor] = None, dk_sf: Optional[torch.Tensor] = None,
                         dv_sf: Optional[torch.Tensor] = None, debug_flags: int = 0):
    """Attention backward (see include/lpfa.h). q/k/v with their head_dim-orientation scales, out and
    dout bf16 (Tq,H,128), lse fp32 (H,Tq). Returns (dq, dk, dv) in bf16, or with output_mxfp8_dkv
    (dq, dk_payload, dv_payload, dk_scales, dv_scales) like LP-FA4's mxfp8_flash_attn_varlen_backward.
    Output tensors may be passed in (contiguous, of the returned shapes and dtypes); debug_flags != 0
    calls the test hook lpfa_attn_bwd_varlen_debug.
    """
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != torch.uint8 or t.dim() != 3 or not t.is_contiguous():
            raise ValueError("%s must be a contiguous uint8 (tokens, heads, 128) tensor" % name)
    for name, t in (("out", out), ("dout", dout)):
        if t.dtype != torch.bfloat16 or t.shape != q.shape or not t.is_contiguous():
            raise ValueError("%s must be a contiguous bf16 tensor shaped like q" % name)
    Tq, H = q.shape[0], q.shape[1]
    Tk = k.shape[0]
    if lse.dtype != torch.float32 or tuple(lse.shape) != (H, Tq) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 (heads, tokens) tensor")
    descs = []
    for name, t in (("q_descale", q_descale), ("k_descale", k_descale), ("v_descale", v_descale)):
        if t is None:
            descs.append(_Descale(None, 0, 0))
        else:
            ss, hs = descale_strides(t, meta_q.num_seqs, H)
            descs.append(_Descale(t.data_ptr(), ss, hs))
    def _out(t, shape, dtype, name):
        if t is None:
            return torch.empty(shape, dtype=dtype, device=q.device)
        if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
            raise ValueError("%s must be a contiguous %s tensor of shape %s" % (name, dtype, tuple(shape)))
        return t

    kv_dtype = torch.uint8 if output_mxfp8_dkv else torch.bfloat16
    dq = _out(dq, (Tq, H, 128), torch.bfloat16, "dq")
    dk = _out(dk, (Tk, H, 128), kv_dtype, "dk")
    dv = _out(dv, (Tk, H, 128), kv_dtype, "dv")
    if output_mxfp8_dkv:
        dk_sf = _out(dk_sf, (meta_k.scale_bytes(H),), torch.uint8, "dk_sf")
        dv_sf = _out(dv_sf, (meta_k.scale_bytes(H),), torch.uint8, "dv_sf")
    else:
        dk_sf = dv_sf = None
    args = (q.data_ptr(), q_sf.data_ptr(), k.data_ptr(), k_sf.data_ptr(), v.data_ptr(), v_sf.data_ptr(),
            out.data_ptr(), dout.data_ptr(), lse.data_ptr(), ctypes.byref(meta_q._c), ctypes.byref(meta_k._c), H, 128,
            ctypes.byref(descs[0]), ctypes.byref(descs[1]), ctypes.byref(descs[2]), dq.data_ptr(), dk.data_ptr(),
            dv.data_ptr(), _ptr(dk_sf), _ptr(dv_sf), 1 if output_mxfp8_dkv else 0, _stream_ptr(stream))
    with torch.cuda.device(q.device):
        if debug_flags:
            _check(_lib.lpfa_attn_bwd_varlen_debug(*args, int(debug_flags)))
        else:
            _check(_lib.lpfa_attn_bwd_varlen(*args))
    if output_mxfp8_dkv:
        return dq, dk, dv, dk_sf, dv_sf
    return dq, dk, dv


def lpfa_device_status(stream=None):
    """Synchronize `stream` and return (status, detail) of the device status word (then reset)."""
    detail = _i32(0)
    st = _lib.lpfa_device_status(_stream_ptr(stream), ctypes.byref(detail))
    return st, detail.value


# LP-FA4 README names.
Mxfp8VarlenMeta = VarlenMeta
quantize_mxfp8_varlen = lpfa_quantize_mxfp8_varlen
mxfp8_flash_attn_varlen_forward = lpfa_attn_fwd_varlen
mxfp8_flash_attn_varlen_backward = lpfa_attn_bwd_varlen
fa4_v_to_fp8 = lpfa_cast_e4m3
