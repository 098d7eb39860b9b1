"""ctypes binding of libattn_b200.so (the C ABI in include/attn.h).

Argument marshalling only: tensors are passed as raw device pointers with
their sizes, the CUDA stream as its handle.  Every step of the computation
runs in the library's kernels; there is no fallback of any kind -- if the
library or a GPU is missing, calls raise.
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_NAME = "libattn_b200.so"
_lock = threading.Lock()
_lib = None

ATTN_OK = 0
ATTN_ERR_INVALID_ARG = 1
ATTN_ERR_UNSUPPORTED = 2
ATTN_ERR_ALIGNMENT = 3
ATTN_ERR_WORKSPACE = 4
ATTN_ERR_CUDA = 5
ATTN_ERR_DEVICE = 6

DEVERR_WAIT_TIMEOUT = 0x1
DEVERR_BAD_PAGE = 0x2
DEVERR_BAD_LENGTH = 0x4

# Every function the header declares, with its ctypes signature.
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_SZ = ctypes.c_size_t
SIGNATURES = {
    "attn_fwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P]),
    "attn_fwd_masked": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P, _P]),
    "attn_fwd_host_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I]),
    "attn_fwd_host": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P, _P, _SZ, _P]),
    "attn_fwd_window": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P, _I, _I, _P]),
    "attn_fwd_fp8": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P,
                          _P]),
    "attn_fwd_block_sparse": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P, _P, _I,
                                   _P]),
    "attn_fwd_varlen_workspace_size": (_SZ, [_I, ctypes.c_longlong, _I]),
    "attn_fwd_varlen": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, ctypes.c_longlong,
                             ctypes.c_longlong, _I, _I, _I, _F, _P, _SZ, _P]),
    "attn_fwd_paged": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, ctypes.c_longlong, _I, _I,
                            _I, _I, _I, _F, _P, _P, _P, _SZ, _P]),
    "attn_fwd_paged_fp8_workspace_size": (_SZ, [_I, ctypes.c_longlong, _I, _I, _I, _I, _I]),
    "attn_fwd_paged_fp8": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I,
                                ctypes.c_longlong, _I, _I, _I, _I, _I, _F, _P, _P, _P, _SZ, _P]),
    "attn_decode_workspace_size": (_SZ, [_I, _I, _I, _I, _I]),
    "attn_decode_paged": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P,
                               _SZ, _P]),
    "attn_decode_paged_fp8": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P,
                                   _P, _P, _SZ, _P]),
    "attn_decode_paged_noalloc": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P,
                                       _P, _P]),
    "attn_bwd_workspace_size": (_SZ, [_I, _I, _I]),
    "attn_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P, _P,
                      _SZ, _P]),
    "attn_bwd_window": (_I, [_P] * 9 + [_I] * 6 + [_F, _P, _I, _I, _P, _SZ, _P]),
    "attn_bwd_block_sparse": (_I, [_P] * 9 + [_I] * 7 + [_F, _P, _P, _I, _P, _SZ, _P]),
    "attn_bwd_varlen_workspace_size": (_SZ, [_I, _I, _I]),
    "attn_bwd_varlen": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I,
                             ctypes.c_longlong, ctypes.c_longlong, _I, _I, _I, _I, _F, _P, _SZ,
                             _P]),
    "attn_get_device_error": (_I, [_P, ctypes.POINTER(ctypes.c_uint)]),
    "attn_strerror": (ctypes.c_char_p, [_I]),
    "attn_split_tokens": (_I, []),
}


class AttnError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {attn_strerror(status)} (status {status})" if what
                         else f"{attn_strerror(status)} (status {status})")


def library_path() -> str:
    return os.path.join(_HERE, LIB_NAME)


def load_library():
    """Load libattn_b200.so from the package directory (raises if it is missing)."""
    global _lib
    with _lock:
        if _lib is None:
            path = library_path()
            if not os.path.exists(path):
                raise RuntimeError(
                    f"{path} is missing: build it with `python -m exact_softmax_attention_fwd_b200.build`")
            lib = ctypes.CDLL(path)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def attn_strerror(status: int) -> str:
    try:
        return load_library().attn_strerror(int(status)).decode()
    except Exception:  # library not loadable: still describe the code
        return {0: "success"}.get(int(status), f"status {status}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(status, what):
    if status != ATTN_OK:
        raise AttnError(status, what)


def _out(t, shape, dtype, device, name):
    """A caller-supplied output buffer, checked against what the kernels write
    (shape, dtype, contiguity, device), or a new one when ``t`` is None."""
    import torch
    if t is None:
        return torch.empty(tuple(shape), dtype=dtype, device=device)
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {dtype} tensor of shape {tuple(shape)}")
    if t.device != device:
        raise ValueError(f"{name} must be on {device}")
    return t


def _require_bf16(**tensors):
    """Raise unless every named tensor is bfloat16 (the kernels read these bytes
    as bf16: any other dtype would be misread, or read past its allocation)."""
    import torch
    for name, t in tensors.items():
        if t.dtype != torch.bfloat16:
            raise ValueError(f"{name} must be torch.bfloat16, got {t.dtype}")


def _require_cuda(*tensors):
    for t in tensors:
        if t is not None and not t.is_cuda:
            raise ValueError("tensors must be CUDA tensors (device memory)")


def attn_fwd_masked(q, k, v, causal: bool, scale: float, k_lens=None, out=None, lse=None,
                    return_lse: bool = True, stream=None):
    """O, LSE = exact attention.  q [B,Hq,Sq,d], k/v [B,Hkv,Sk,d] bf16 CUDA tensors."""
    import torch
    _require_cuda(q, k, v, k_lens)
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous bfloat16")
    B, Hq, Sq, d = q.shape
    Bk, Hkv, Sk, dk = k.shape
    if tuple(v.shape) != tuple(k.shape) or Bk != B or dk != d:
        raise ValueError("q/k/v shapes disagree")
    if k_lens is not None and (k_lens.dtype != torch.int32 or tuple(k_lens.shape) != (B,)):
        raise ValueError("k_lens must be int32 [B]")
    out = _out(out, q.shape, torch.bfloat16, q.device, "out")
    if lse is not None or return_lse:
        lse = _out(lse, (B, Hq, Sq), torch.float32, q.device, "lse")
    st = load_library().attn_fwd_masked(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq,
                                        Hkv, Sq, Sk, d, int(bool(causal)), float(scale),
                                        _ptr(k_lens), _stream(stream))
    _check(st, "attn_fwd_masked")
    return out, lse


def attn_fwd_host_workspace_size(B: int, Hq: int, Hkv: int, Sq: int, Sk: int, d: int) -> int:
    return int(load_library().attn_fwd_host_workspace_size(B, Hq, Hkv, Sq, Sk, d))


def attn_fwd_host(q, k, v, causal: bool, scale: float, k_lens=None, out=None, lse=None,
                  workspace=None, return_lse: bool = True, device=None, stream=None):
    """attn_fwd_masked on HOST tensors (pinned for copy/compute overlap): q [B,Hq,Sq,d],
    k/v [B,Hkv,Sk,d] bf16 CPU tensors, k_lens int32 [B] CPU tensor or None.  O and LSE
    are host tensors, complete once ``stream`` (default: the current stream of
    ``device``) reaches this call's end; synchronise it before reading them."""
    import torch
    for name, t in (("q", q), ("k", k), ("v", v), ("k_lens", k_lens)):
        if t is not None and t.device.type != "cpu":
            raise ValueError(f"{name} must be a host (CPU) tensor")
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous bfloat16")
    B, Hq, Sq, d = q.shape
    Bk, Hkv, Sk, dk = k.shape
    if tuple(v.shape) != tuple(k.shape) or Bk != B or dk != d:
        raise ValueError("q/k/v shapes disagree")
    if k_lens is not None and (k_lens.dtype != torch.int32 or tuple(k_lens.shape) != (B,)
                               or not k_lens.is_contiguous()):
        raise ValueError("k_lens must be contiguous int32 [B]")
    if device is None:
        device = torch.device("cuda", torch.cuda.current_device())
    device = torch.device(device)
    cpu = torch.device("cpu")
    pin = q.is_pinned()
    if out is None:
        out = torch.empty(tuple(q.shape), dtype=torch.bfloat16, pin_memory=pin)
    out = _out(out, q.shape, torch.bfloat16, cpu, "out")
    if lse is not None or return_lse:
        if lse is None:
            lse = torch.empty((B, Hq, Sq), dtype=torch.float32, pin_memory=pin)
        lse = _out(lse, (B, Hq, Sq), torch.float32, cpu, "lse")
    if stream is None:
        stream = torch.cuda.current_stream(device)
    need = attn_fwd_host_workspace_size(B, Hq, Hkv, Sq, Sk, d)
    if workspace is None:
        # allocated on ``stream``: the allocator reuses it only after the call's last copy
        with torch.cuda.stream(stream):
            workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=device)
    if not workspace.is_cuda or workspace.device != device:
        raise ValueError(f"workspace must be on {device}")
    ws_bytes = workspace.numel() * workspace.element_size()
    with torch.cuda.device(device):
        st = load_library().attn_fwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B,
                                          Hq, Hkv, Sq, Sk, d, int(bool(causal)), float(scale),
                                          _ptr(k_lens), _ptr(workspace), ws_bytes,
                                          _stream(stream))
    _check(st, "attn_fwd_host")
    return out, lse


def attn_fwd(q, k, v, causal: bool, scale: float, out=None, lse=None, return_lse: bool = True,
             stream=None):
    """attn_fwd_masked without key padding."""
    return attn_fwd_masked(q, k, v, causal, scale, None, out, lse, return_lse, stream)


def attn_fwd_window(q, k, v, scale: float, window: int = 0, prefix: int = 0, k_lens=None,
                    out=None, lse=None, return_lse: bool = True, stream=None):
    """Causal prefill with a sliding window (window > 0) or a prefix-LM mask (prefix > 0);
    q [B,Hq,Sq,d], k/v [B,Hkv,Sk,d] bf16 CUDA tensors (layouts as attn_fwd_masked)."""
    import torch
    _require_cuda(q, k, v, k_lens)
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous bfloat16")
    B, Hq, Sq, d = q.shape
    Bk, Hkv, Sk, dk = k.shape
    if tuple(v.shape) != tuple(k.shape) or Bk != B or dk != d:
        raise ValueError("q/k/v shapes disagree")
    if k_lens is not None and (k_lens.dtype != torch.int32 or tuple(k_lens.shape) != (B,)):
        raise ValueError("k_lens must be int32 [B]")
    out = _out(out, q.shape, torch.bfloat16, q.device, "out")
    if lse is not None or return_lse:
        lse = _out(lse, (B, Hq, Sq), torch.float32, q.device, "lse")
    st = load_library().attn_fwd_window(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq,
                                        Hkv, Sq, Sk, d, float(scale), _ptr(k_lens), int(window),
                                        int(prefix), _stream(stream))
    _check(st, "attn_fwd_window")
    return out, lse


def attn_fwd_block_sparse(q, k, v, block_mask, causal: bool, scale: float, k_lens=None,
                          out=None, lse=None, return_lse: bool = True, stream=None):
    """Prefill with a block-sparse mask: block_mask uint8 [B, 1 or Hq, ceil(Sq/128),
    ceil(Sk/128)] on the device (0 = the 128 x 128 block is skipped)."""
    import torch
    _require_cuda(q, k, v, k_lens, block_mask)
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous bfloat16")
    B, Hq, Sq, d = q.shape
    Bk, Hkv, Sk, dk = k.shape
    if tuple(v.shape) != tuple(k.shape) or Bk != B or dk != d:
        raise ValueError("q/k/v shapes disagree")
    if block_mask.dtype != torch.uint8 or not block_mask.is_contiguous() or block_mask.dim() != 4 \
            or block_mask.shape[0] != B or block_mask.shape[1] not in (1, Hq) \
            or block_mask.shape[2] != -(-Sq // 128) or block_mask.shape[3] != -(-Sk // 128):
        raise ValueError("block_mask must be contiguous uint8 [B, 1 or Hq, ceil(Sq/128), ceil(Sk/128)]")
    if k_lens is not None and (k_lens.dtype != torch.int32 or tuple(k_lens.shape) != (B,)):
        raise ValueError("k_lens must be int32 [B]")
    out = _out(out, q.shape, torch.bfloat16, q.device, "out")
    if lse is not None or return_lse:
        lse = _out(lse, (B, Hq, Sq), torch.float32, q.device, "lse")
    st = load_library().attn_fwd_block_sparse(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B,
                                              Hq, Hkv, Sq, Sk, d, int(bool(causal)), float(scale),
                                              _ptr(k_lens), _ptr(block_mask), block_mask.shape[1],
                                              _stream(stream))
    _check(st, "attn_fwd_block_sparse")
    return out, lse


def attn_fwd_fp8(q, k, v, q_scale, k_scale, v_scale, causal: bool, scale: float, k_lens=None,
                 out=None, lse=None, return_lse: bool = True, stream=None):
    """Prefill over block-scaled E4M3 inputs: q [B,Hq,Sq,128], k/v [B,Hkv,Sk,128] uint8
    codes; q_scale [B,Hq,ceil(Sq/128)], k_scale/v_scale [B,Hkv,ceil(Sk/128)] float32.
    Returns O [B,Hq,Sq,128] bf16 and LSE [B,Hq,Sq] fp32."""
    import torch
    for t in (q, k, v):
        if t.dtype != torch.uint8 or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous uint8 E4M3 codes")
    B, Hq, Sq, d = q.shape
    Bk, Hkv, Sk, dk = k.shape
    if tuple(v.shape) != tuple(k.shape) or Bk != B or dk != d:
        raise ValueError("q/k/v shapes disagree")
    for t, shape in ((q_scale, (B, Hq, -(-Sq // 128))), (k_scale, (B, Hkv, -(-Sk // 128))),
                     (v_scale, (B, Hkv, -(-Sk // 128)))):
        if t.dtype != torch.float32 or tuple(t.shape) != shape or not t.is_contiguous():
            raise ValueError(f"block scales must be contiguous float32 {shape}")
    _require_cuda(q, k, v, q_scale, k_scale, v_scale, k_lens)
    if k_lens is not None and (k_lens.dtype != torch.int32 or tuple(k_lens.shape) != (B,)):
        raise ValueError("k_lens must be int32 [B]")
    out = _out(out, q.shape, torch.bfloat16, q.device, "out")
    if lse is not None or return_lse:
        lse = _out(lse, (B, Hq, Sq), torch.float32, q.device, "lse")
    st = load_library().attn_fwd_fp8(_ptr(q), _ptr(k), _ptr(v), _ptr(q_scale), _ptr(k_scale),
                                     _ptr(v_scale), _ptr(out), _ptr(lse), B, Hq, Hkv, Sq, Sk, d,
                                     int(bool(causal)), float(scale), _ptr(k_lens),
                                     _stream(stream))
    _check(st, "attn_fwd_fp8")
    return out, lse


def attn_bwd_workspace_size(B: int, Hq: int, Sq: int) -> int:
    return int(load_library().attn_bwd_workspace_size(B, Hq, Sq))


def attn_bwd(q, k, v, o, lse, d_o, causal: bool, scale: float, k_lens=None, dq=None, dk=None,
             dv=None, workspace=None, stream=None):
    """dQ, dK, dV of attn_fwd_masked.  q, o, d_o [B,Hq,Sq,d], k/v [B,Hkv,Sk,d] bf16; lse
    [B,Hq,Sq] fp32 as the forward returned it for the same causal / scale / k_lens."""
    import torch
    _require_cuda(q, k, v, o, lse, d_o, k_lens, dq, dk, dv, workspace)
    for t in (q, k, v, o, d_o):
        if t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("q, k, v, o, d_o must be contiguous bfloat16")
    B, Hq, Sq, d = q.shape
    Bk, Hkv, Sk, dk_ = k.shape
    if tuple(v.shape) != tuple(k.shape) or Bk != B or dk_ != d:
        raise ValueError("q/k/v shapes disagree")
    if tuple(o.shape) != tuple(q.shape) or tuple(d_o.shape) != tuple(q.shape):
        raise ValueError("o and d_o must have q's shape")
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, Hq, Sq) or not lse.is_contiguous():
        raise ValueError("lse must be contiguous float32 [B, Hq, Sq]")
    if k_lens is not None and (k_lens.dtype != torch.int32 or tuple(k_lens.shape) != (B,)):
        raise ValueError("k_lens must be int32 [B]")
    dq = _out(dq, q.shape, torch.bfloat16, q.device, "dq")
    dk = _out(dk, k.shape, torch.bfloat16, q.device, "dk")
    dv = _out(dv, v.shape, torch.bfloat16, q.device, "dv")
    need = attn_bwd_workspace_size(B, Hq, Sq)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    st = load_library().attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(d_o),
                                 _ptr(dq), _ptr(dk), _ptr(dv), B, Hq, Hkv, Sq, Sk, d,
                                 int(bool(causal)), float(scale), _ptr(k_lens), _ptr(workspace),
                                 ws_bytes, _stream(stream))
    _check(st, "attn_bwd")
    return dq, dk, dv


def _bwd_fixed_checks(q, k, v, o, lse, d_o, k_lens):
    import torch
    _require_bf16(q=q, k=k, v=v, o=o, d_o=d_o)
    _require_cuda(q, k, v, o, lse, d_o, k_lens)
    for t in (q, k, v, o, d_o):
        if not t.is_contiguous():
            raise ValueError("q, k, v, o, d_o must be contiguous")
    B, Hq, Sq, d = q.shape
    Bk, Hkv, Sk, dk_ = k.shape
    if tuple(v.shape) != tuple(k.shape) or Bk != B or dk_ != d:
        raise ValueError("q/k/v shapes disagree")
    if tuple(o.shape) != tuple(q.shape) or tuple(d_o.shape) != tuple(q.shape):
        raise ValueError("o and d_o must have q's shape")
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, Hq, Sq) or not lse.is_contiguous():
        raise ValueError("lse must be contiguous float32 [B, Hq, Sq]")
    if k_lens is not None and (k_lens.dtype != torch.int32 or tuple(k_lens.shape) != (B,)):
        raise ValueError("k_lens must be int32 [B]")
    return B, Hq, Hkv, Sq, Sk, d


def attn_bwd_window(q, k, v, o, lse, d_o, scale: float, window: int = 0, prefix: int = 0,
                    k_lens=None, dq=None, dk=None, dv=None, workspace=None, stream=None):
    """dQ, dK, dV of attn_fwd_window (causal, sliding window or prefix-LM)."""
    import torch
    B, Hq, Hkv, Sq, Sk, d = _bwd_fixed_checks(q, k, v, o, lse, d_o, k_lens)
    dq = _out(dq, q.shape, torch.bfloat16, q.device, "dq")
    dk = _out(dk, k.shape, torch.bfloat16, q.device, "dk")
    dv = _out(dv, v.shape, torch.bfloat16, q.device, "dv")
    if workspace is None:
        workspace = torch.empty(max(attn_bwd_workspace_size(B, Hq, Sq), 16), dtype=torch.uint8,
                                device=q.device)
    st = load_library().attn_bwd_window(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(d_o), _ptr(dq), _ptr(dk), _ptr(dv), B,
        Hq, Hkv, Sq, Sk, d, float(scale), _ptr(k_lens), int(window), int(prefix), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "attn_bwd_window")
    return dq, dk, dv


def attn_bwd_block_sparse(q, k, v, o, lse, d_o, block_mask, causal: bool, scale: float,
                          k_lens=None, dq=None, dk=None, dv=None, workspace=None, stream=None):
    """dQ, dK, dV of attn_fwd_block_sparse; block_mask uint8 [B, 1 or Hq, ceil(Sq/128),
    ceil(Sk/128)] on the device, as given to the forward."""
    import torch
    B, Hq, Hkv, Sq, Sk, d = _bwd_fixed_checks(q, k, v, o, lse, d_o, k_lens)
    _require_cuda(block_mask)
    nq, nk = -(-Sq // 128), -(-Sk // 128)
    if (block_mask.dtype != torch.uint8 or block_mask.dim() != 4 or
            tuple(block_mask.shape) not in ((B, 1, nq, nk), (B, Hq, nq, nk)) or
            not block_mask.is_contiguous()):
        raise ValueError(f"block_mask must be contiguous uint8 [B, 1 or Hq, {nq}, {nk}]")
    dq = _out(dq, q.shape, torch.bfloat16, q.device, "dq")
    dk = _out(dk, k.shape, torch.bfloat16, q.device, "dk")
    dv = _out(dv, v.shape, torch.bfloat16, q.device, "dv")
    if workspace is None:
        workspace = torch.empty(max(attn_bwd_workspace_size(B, Hq, Sq), 16), dtype=torch.uint8,
                                device=q.device)
    st = load_library().attn_bwd_block_sparse(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(d_o), _ptr(dq), _ptr(dk), _ptr(dv), B,
        Hq, Hkv, Sq, Sk, d, int(bool(causal)), float(scale), _ptr(k_lens), _ptr(block_mask),
        block_mask.shape[1], _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream))
    _check(st, "attn_bwd_block_sparse")
    return dq, dk, dv


def attn_bwd_varlen_workspace_size(B: int, Hq: int, max_seqlen_q: int) -> int:
    return int(load_library().attn_bwd_varlen_workspace_size(B, Hq, max_seqlen_q))


def attn_bwd_varlen(q, k, v, o, lse, d_o, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int,
                    max_seqlen_k: int, causal: bool, scale: float, dq=None, dk=None, dv=None,
                    workspace=None, stream=None):
    """dQ, dK, dV of attn_fwd_varlen.  q, o, d_o [total_q, Hq, d], k/v [total_k, Hkv, d]
    bf16 packed; lse [Hq, total_q] fp32 as the forward returned it; cu_seqlens_q/k int32
    [B+1] on the device; max_seqlen_q/k bound the sequences' lengths."""
    import torch
    _require_bf16(q=q, k=k, v=v, o=o, d_o=d_o)
    _require_cuda(q, k, v, o, lse, d_o, cu_seqlens_q, cu_seqlens_k, dq, dk, dv, workspace)
    for t in (q, k, v, o, d_o):
        if not t.is_contiguous():
            raise ValueError("q, k, v, o, d_o must be contiguous")
    if q.dim() != 3 or k.dim() != 3 or tuple(v.shape) != tuple(k.shape):
        raise ValueError("q [total_q, Hq, d]; k, v [total_k, Hkv, d]")
    total_q, Hq, d = q.shape
    total_k, Hkv, dk_ = k.shape
    if dk_ != d or tuple(o.shape) != tuple(q.shape) or tuple(d_o.shape) != tuple(q.shape):
        raise ValueError("o and d_o must have q's shape and the head dims must agree")
    if lse.dtype != torch.float32 or tuple(lse.shape) != (Hq, total_q) or not lse.is_contiguous():
        raise ValueError("lse must be contiguous float32 [Hq, total_q]")
    B = cu_seqlens_q.shape[0] - 1
    for t in (cu_seqlens_q, cu_seqlens_k):
        if t.dtype != torch.int32 or tuple(t.shape) != (B + 1,) or not t.is_contiguous():
            raise ValueError("cu_seqlens_q / cu_seqlens_k must be contiguous int32 [B+1]")
    dq = _out(dq, q.shape, torch.bfloat16, q.device, "dq")
    dk = _out(dk, k.shape, torch.bfloat16, q.device, "dk")
    dv = _out(dv, v.shape, torch.bfloat16, q.device, "dv")
    need = attn_bwd_varlen_workspace_size(B, Hq, max_seqlen_q)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    st = load_library().attn_bwd_varlen(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(d_o), _ptr(dq), _ptr(dk), _ptr(dv),
        _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), B, Hq, Hkv, total_q, total_k, int(max_seqlen_q),
        int(max_seqlen_k), d, int(bool(causal)), float(scale), _ptr(workspace), ws_bytes,
        _stream(stream))
    _check(st, "attn_bwd_varlen")
    return dq, dk, dv


def attn_fwd_varlen_workspace_size(B: int, total_q: int, max_seqlen_q: int) -> int:
    return int(load_library().attn_fwd_varlen_workspace_size(B, total_q, max_seqlen_q))


def attn_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, causal: bool,
                    scale: float, out=None, lse=None, workspace=None, return_lse: bool = True,
                    stream=None):
    """Prefill over a ragged batch: q [total_q, Hq, d], k/v [total_k, Hkv, d] bf16, packed;
    cu_seqlens_q/k int32 [B+1] on the device.  Returns O [total_q, Hq, d], LSE [Hq, total_q]."""
    import torch
    _require_cuda(q, k, v, cu_seqlens_q, cu_seqlens_k)
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or not t.is_contiguous() or t.dim() != 3:
            raise ValueError("q, k, v must be contiguous 3-d bfloat16 tensors")
    total_q, Hq, d = q.shape
    total_k, Hkv, dk = k.shape
    if tuple(v.shape) != tuple(k.shape) or dk != d:
        raise ValueError("q/k/v shapes disagree")
    for t in (cu_seqlens_q, cu_seqlens_k):
        if t.dtype != torch.int32 or t.dim() != 1 or not t.is_contiguous():
            raise ValueError("cu_seqlens must be contiguous int32 [B+1]")
    if cu_seqlens_q.shape != cu_seqlens_k.shape or cu_seqlens_q.shape[0] < 2:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must both be [B+1], B >= 1")
    B = cu_seqlens_q.shape[0] - 1
    need = attn_fwd_varlen_workspace_size(B, total_q, max_seqlen_q)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    out = _out(out, q.shape, torch.bfloat16, q.device, "out")
    if lse is not None or return_lse:
        lse = _out(lse, (Hq, total_q), torch.float32, q.device, "lse")
    ws_bytes = workspace.numel() * workspace.element_size()
    st = load_library().attn_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                                        _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), B, Hq, Hkv,
                                        total_q, total_k, int(max_seqlen_q), d,
                                        int(bool(causal)), float(scale), _ptr(workspace),
                                        ws_bytes, _stream(stream))
    _check(st, "attn_fwd_varlen")
    return out, lse


def attn_fwd_paged(q, k_cache, v_cache, block_table, cu_seqlens_q, seq_lens_k, max_seqlen_q: int,
                   causal: bool, scale: float, out=None, lse=None, workspace=None,
                   return_lse: bool = True, stream=None):
    """Prefill/append of packed queries q [total_q, Hq, d] over a paged cache
    [num_pages, page_size, Hkv, d]; returns O [total_q, Hq, d], LSE [Hq, total_q]."""
    import torch
    _require_cuda(q, k_cache, v_cache, block_table, cu_seqlens_q, seq_lens_k)
    for t in (q, k_cache, v_cache):
        if t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("q and the caches must be contiguous bfloat16")
    if q.dim() != 3 or k_cache.dim() != 4 or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("q [total_q, Hq, d]; caches [num_pages, page_size, Hkv, d]")
    total_q, Hq, d = q.shape
    num_pages, page_size, Hkv, dk = k_cache.shape
    if dk != d:
        raise ValueError("head dims disagree")
    B = cu_seqlens_q.shape[0] - 1
    for t, shape in ((cu_seqlens_q, (B + 1,)), (seq_lens_k, (B,))):
        if t.dtype != torch.int32 or tuple(t.shape) != shape or not t.is_contiguous():
            raise ValueError("cu_seqlens_q int32 [B+1], seq_lens_k int32 [B]")
    if block_table.dtype != torch.int32 or block_table.dim() != 2 or block_table.shape[0] != B \
            or not block_table.is_contiguous():
        raise ValueError("block_table must be contiguous int32 [B, max_pages_per_seq]")
    need = attn_fwd_varlen_workspace_size(B, total_q, max_seqlen_q)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    out = _out(out, q.shape, torch.bfloat16, q.device, "out")
    if lse is not None or return_lse:
        lse = _out(lse, (Hq, total_q), torch.float32, q.device, "lse")
    ws_bytes = workspace.numel() * workspace.element_size()
    st = load_library().attn_fwd_paged(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                       _ptr(cu_seqlens_q), _ptr(seq_lens_k), page_size, B, Hq,
                                       Hkv, total_q, int(max_seqlen_q), block_table.shape[1],
                                       num_pages, d, int(bool(causal)), float(scale), _ptr(out),
                                       _ptr(lse), _ptr(workspace), ws_bytes, _stream(stream))
    _check(st, "attn_fwd_paged")
    return out, lse


def attn_fwd_paged_fp8_workspace_size(B: int, total_q: int, max_seqlen_q: int,
                                      max_pages_per_seq: int, page_size: int, Hkv: int,
                                      d: int) -> int:
    return int(load_library().attn_fwd_paged_fp8_workspace_size(
        B, total_q, max_seqlen_q, max_pages_per_seq, page_size, Hkv, d))


def attn_fwd_paged_fp8(q, k_cache, v_cache, k_scale, v_scale, block_table, cu_seqlens_q,
                       seq_lens_k, max_seqlen_q: int, causal: bool, scale: float, out=None,
                       lse=None, workspace=None, return_lse: bool = True, stream=None):
    """attn_fwd_paged over an E4M3 cache: k_cache / v_cache uint8 [num_pages, page_size,
    Hkv, d] codes, k_scale / v_scale float32 [num_pages, Hkv]; q [total_q, Hq, d] bf16."""
    import torch
    _require_bf16(q=q)
    if k_cache.dtype != torch.uint8 or v_cache.dtype != torch.uint8:
        raise ValueError("FP8 caches are uint8 E4M3 codes")
    _require_cuda(q, k_cache, v_cache, k_scale, v_scale, block_table, cu_seqlens_q, seq_lens_k)
    if q.dim() != 3 or k_cache.dim() != 4 or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("q [total_q, Hq, d]; caches [num_pages, page_size, Hkv, d]")
    total_q, Hq, d = q.shape
    num_pages, page_size, Hkv, dk = k_cache.shape
    if dk != d:
        raise ValueError("head dims disagree")
    for t in (k_scale, v_scale):
        if t.dtype != torch.float32 or tuple(t.shape) != (num_pages, Hkv) or not t.is_contiguous():
            raise ValueError("scales must be contiguous float32 [num_pages, Hkv]")
    B = cu_seqlens_q.shape[0] - 1
    for t, shape in ((cu_seqlens_q, (B + 1,)), (seq_lens_k, (B,))):
        if t.dtype != torch.int32 or tuple(t.shape) != shape or not t.is_contiguous():
            raise ValueError("cu_seqlens_q int32 [B+1], seq_lens_k int32 [B]")
    if block_table.dtype != torch.int32 or block_table.dim() != 2 or block_table.shape[0] != B \
            or not block_table.is_contiguous():
        raise ValueError("block_table must be contiguous int32 [B, max_pages_per_seq]")
    for t in (q, k_cache, v_cache):
        if not t.is_contiguous():
            raise ValueError("q and the caches must be contiguous")
    max_pages = block_table.shape[1]
    need = attn_fwd_paged_fp8_workspace_size(B, total_q, max_seqlen_q, max_pages, page_size, Hkv,
                                             d)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    out = _out(out, q.shape, torch.bfloat16, q.device, "out")
    if lse is not None or return_lse:
        lse = _out(lse, (Hq, total_q), torch.float32, q.device, "lse")
    st = load_library().attn_fwd_paged_fp8(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_scale), _ptr(v_scale), _ptr(block_table),
        _ptr(cu_seqlens_q), _ptr(seq_lens_k), page_size, B, Hq, Hkv, total_q, int(max_seqlen_q),
        max_pages, num_pages, d, int(bool(causal)), float(scale), _ptr(out), _ptr(lse),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "attn_fwd_paged_fp8")
    return out, lse


def attn_decode_workspace_size(B: int, Hq: int, max_pages_per_seq: int, page_size: int,
                               d: int) -> int:
    return int(load_library().attn_decode_workspace_size(B, Hq, max_pages_per_seq, page_size, d))


def attn_decode_paged(q, k_cache, v_cache, block_table, seq_lens, scale: float, out=None,
                      lse=None, workspace=None, return_lse: bool = True, stream=None):
    """Single-query attention over a paged cache (see include/attn.h for layouts)."""
    import torch
    _require_bf16(q=q, k_cache=k_cache, v_cache=v_cache)
    _require_cuda(q, k_cache, v_cache, block_table, seq_lens)
    B, Hq, d = q.shape
    num_pages, page_size, Hkv, dk = k_cache.shape
    if tuple(v_cache.shape) != tuple(k_cache.shape) or dk != d:
        raise ValueError("cache shapes disagree")
    if block_table.dtype != torch.int32 or block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError("block_table must be int32 [B, max_pages_per_seq]")
    if seq_lens.dtype != torch.int32 or tuple(seq_lens.shape) != (B,):
        raise ValueError("seq_lens must be int32 [B]")
    for t in (q, k_cache, v_cache, block_table, seq_lens):
        if not t.is_contiguous():
            raise ValueError("inputs must be contiguous")
    max_pages = block_table.shape[1]
    need = attn_decode_workspace_size(B, Hq, max_pages, page_size, d)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    out = _out(out, (B, Hq, d), torch.bfloat16, q.device, "out")
    if lse is not None or return_lse:
        lse = _out(lse, (B, Hq), torch.float32, q.device, "lse")
    ws_bytes = workspace.numel() * workspace.element_size()
    st = load_library().attn_decode_paged(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                          _ptr(seq_lens), page_size, B, Hq, Hkv, d, max_pages,
                                          num_pages, float(scale), _ptr(out), _ptr(lse),
                                          _ptr(workspace), ws_bytes, _stream(stream))
    _check(st, "attn_decode_paged")
    return out, lse


def attn_decode_paged_fp8(q, k_cache, v_cache, k_scale, v_scale, block_table, seq_lens,
                          scale: float, out=None, lse=None, workspace=None,
                          return_lse: bool = True, stream=None):
    """attn_decode_paged over an E4M3 cache: k_cache / v_cache uint8 [num_pages,
    page_size, Hkv, d] codes, k_scale / v_scale float32 [num_pages, Hkv]."""
    import torch
    _require_bf16(q=q)
    _require_cuda(q, k_cache, v_cache, k_scale, v_scale, block_table, seq_lens)
    B, Hq, d = q.shape
    num_pages, page_size, Hkv, dk = k_cache.shape
    if k_cache.dtype != torch.uint8 or v_cache.dtype != torch.uint8:
        raise ValueError("FP8 caches are uint8 E4M3 codes")
    if tuple(v_cache.shape) != tuple(k_cache.shape) or dk != d:
        raise ValueError("cache shapes disagree")
    for t in (k_scale, v_scale):
        if t.dtype != torch.float32 or tuple(t.shape) != (num_pages, Hkv):
            raise ValueError("scales must be float32 [num_pages, Hkv]")
    if block_table.dtype != torch.int32 or block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError("block_table must be int32 [B, max_pages_per_seq]")
    if seq_lens.dtype != torch.int32 or tuple(seq_lens.shape) != (B,):
        raise ValueError("seq_lens must be int32 [B]")
    for t in (q, k_cache, v_cache, k_scale, v_scale, block_table, seq_lens):
        if not t.is_contiguous():
            raise ValueError("inputs must be contiguous")
    max_pages = block_table.shape[1]
    need = attn_decode_workspace_size(B, Hq, max_pages, page_size, d)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    out = _out(out, (B, Hq, d), torch.bfloat16, q.device, "out")
    if lse is not None or return_lse:
        lse = _out(lse, (B, Hq), torch.float32, q.device, "lse")
    ws_bytes = workspace.numel() * workspace.element_size()
    st = load_library().attn_decode_paged_fp8(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_scale), _ptr(v_scale), _ptr(block_table),
        _ptr(seq_lens), page_size, B, Hq, Hkv, d, max_pages, num_pages, float(scale), _ptr(out),
        _ptr(lse), _ptr(workspace), ws_bytes, _stream(stream))
    _check(st, "attn_decode_paged_fp8")
    return out, lse


# Size of the library's static decode scratch area (ATTN_NOALLOC_SCRATCH_BYTES).
NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024


def attn_decode_paged_noalloc(q, k_cache, v_cache, block_table, seq_lens, scale, out=None,
                              lse=None, return_lse: bool = True, stream=None):
    """attn_decode_paged for callers that may not allocate device memory.

    The library keeps the split partials in its own static device scratch area
    (NOALLOC_SCRATCH_BYTES per GPU), so no workspace is passed and the C call
    allocates nothing.  Only `out`/`lse` are created here when not supplied --
    callers that cannot allocate pass their own.  Calls that overlap on the GPU
    share that scratch area and race; serialise them.  The first call on a
    device caches the area's address: make it before any stream capture.
    """
    import torch
    _require_bf16(q=q, k_cache=k_cache, v_cache=v_cache)
    _require_cuda(q, k_cache, v_cache, block_table, seq_lens)
    B, Hq, d = q.shape
    num_pages, page_size, Hkv, dk = k_cache.shape
    if tuple(v_cache.shape) != tuple(k_cache.shape) or dk != d:
        raise ValueError("cache shapes disagree")
    if block_table.dtype != torch.int32 or block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError("block_table must be int32 [B, max_pages_per_seq]")
    if seq_lens.dtype != torch.int32 or tuple(seq_lens.shape) != (B,):
        raise ValueError("seq_lens must be int32 [B]")
    for t in (q, k_cache, v_cache, block_table, seq_lens):
        if not t.is_contiguous():
            raise ValueError("inputs must be contiguous")
    out = _out(out, (B, Hq, d), torch.bfloat16, q.device, "out")
    if lse is not None or return_lse:
        lse = _out(lse, (B, Hq), torch.float32, q.device, "lse")
    st = load_library().attn_decode_paged_noalloc(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(seq_lens), page_size, B,
        Hq, Hkv, d, block_table.shape[1], num_pages, float(scale), _ptr(out), _ptr(lse),
        _stream(stream))
    _check(st, "attn_decode_paged_noalloc")
    return out, lse


def attn_get_device_error(stream=None):
    """(status, flags): synchronises the stream, reads and clears the device error word."""
    flags = ctypes.c_uint(0)
    st = load_library().attn_get_device_error(_stream(stream), ctypes.byref(flags))
    return st, int(flags.value)
