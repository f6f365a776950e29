"""Python binding of libsas (include/sas.h): argument marshalling only.

Each function has the name of the C entry point it calls. Tensors are torch
CUDA tensors (torch provides device memory and the current stream); every step
of the computation runs in the library's CUDA kernels. There is no CPU
fallback: if libsas.so is missing or no GPU is present, calls raise.
"""
from __future__ import annotations

import ctypes
import os

import torch

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libsas.so")

SAS_F32, SAS_BF16 = 0, 1
SAS_PREFILL, SAS_DECODE = 0, 1
STATUS = {0: "SAS_OK", 1: "SAS_ERR_INVALID_ARG", 2: "SAS_ERR_UNSUPPORTED", 3: "SAS_ERR_CUDA",
          4: "SAS_ERR_TIMEOUT", 5: "SAS_ERR_INTERNAL"}

# exported symbol -> (restype, argtypes)
_P, _I, _F, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "sas_strerror": (ctypes.c_char_p, [_I]),
    "sas_last_error_message": (ctypes.c_char_p, []),
    "sas_version": (_I, []),
    "sas_block_summary": (_I, [_P, _I, _I, _I, _I, _I, _P, _P, _P]),
    "sas_select_workspace_size": (_Z, [_I, _I, _I, _I, _I, _I, _I]),
    "sas_select": (_I, [_P, _I, _P, _I, _I, _I, _I, _I, _I, _I, _P, _F, _P, _P, _P, _P, _P, _Z,
                        _P]),
    "sas_select_prefill_noalloc_capacity": (_Z, []),
    "sas_select_prefill_noalloc": (_I, [_P, _I, _P, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P, _P]),
    "sas_attn_fwd_workspace_size": (_Z, [_I, _I, _I, _I, _I, _I, _I]),
    "sas_attn_fwd": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _I, _F, _P, _P, _P, _Z,
                          _P]),
    "sas_attn_bwd_workspace_size": (_Z, [_I, _I, _I, _I, _I, _I, _I]),
    "sas_attn_bwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _I, _F, _P,
                          _P, _P, _P, _P, _Z, _P]),
    "sas_decode_workspace_size": (_Z, [_I, _I, _I, _I, _I, _I]),
    "sas_decode_attend_workspace_size": (_Z, [_I, _I, _I, _I, _I, _I]),
    "sas_decode_attend": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _I, _I, _F,
                               _P, _P, _Z, _P]),
    "sas_decode": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _I, _I, _F, _P, _P, _P, _Z,
                        _P]),
    "sas_decode_paged": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _I, _P, _I, _I, _F,
                              _P, _P, _P]),
    "sas_decode_paged_ex": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _I, _P, _I, _I,
                                 _F, _P, _P, _P]),
    "sas_decode_host": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _I, _I, _F, _P, _P,
                             _P, _P]),
    "sas_block_summary_ex": (_I, [_P, _I, _I, _I, _I, _I, _P, _P, _I, _P]),
    "sas_block_summary_last": (_I, [_P, _I, _I, _I, _I, _I, _P, _P, _I, _P, _I, _P]),
    "sas_select_tokens": (_I, [_P, _I, _P, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P, _P]),
    "sas_attn_fwd_tokens": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _I, _F, _P,
                                 _P, _P]),
    "sas_attn_bwd_tokens_workspace_size": (ctypes.c_size_t, [_I, _I, _I, _I, _I]),
    "sas_attn_bwd_tokens": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _I,
                                 _F, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "sas_select_bwd_tokens_workspace_size": (_Z, [_I, _I, _I, _I, _I]),
    "sas_select_bwd_tokens": (_I, [_P, _I, _P, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P, _P, _P,
                                   _P, _Z, _P]),
    "sas_decode_ex": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _I, _I, _I, _F, _P, _P,
                           _P]),
    "sas_select_bwd_workspace_size": (_Z, [_I, _I, _I, _I, _I]),
    "sas_select_bwd": (_I, [_P, _I, _P, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P, _P, _P, _P, _Z,
                            _P]),
    "sas_device_status": (_I, [_I, _P]),
    "sas_debug_wait_timeout": (_I, [_P]),
}

_lib = None


class SasError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn} failed: {STATUS.get(status, status)}: {msg}")
        self.status = status


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libsas.so (built in-tree by gated_block_sparse_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: run `python -m gated_block_sparse_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _check(fn: str, status: int) -> None:
    if status != 0:
        msg = load_library().sas_last_error_message().decode()
        raise SasError(fn, status, msg)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SAS_BF16
    if t.dtype == torch.float32:
        return SAS_F32
    raise TypeError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int | None:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _ws(nbytes: int, device, ws: torch.Tensor | None) -> torch.Tensor:
    if ws is not None and ws.numel() * ws.element_size() >= nbytes:
        return ws
    return torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)


def sas_block_summary(k: torch.Tensor, lens: torch.Tensor | None = None,
                      out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Mean of each complete 64-key block: k [B][H][N][d] -> [B][H][N//64][d] fp32."""
    B, H, N, d = k.shape
    if out is None:
        out = torch.empty((B, H, N // 64, d), dtype=torch.float32, device=k.device)
    _check("sas_block_summary", load_library().sas_block_summary(
        _ptr(k), _dt(k), B, H, N, d, _ptr(lens), _ptr(out), _stream(stream)))
    return out


def sas_select(q: torch.Tensor, ksum: torch.Tensor, Hkv: int, topk: int, mode: str = "prefill",
               lens: torch.Tensor | None = None, scale: float = 0.0, out=None, ws=None,
               stream=None, scores_out: torch.Tensor | None = None):
    """Scores, gate and Top-K. Returns (idx int32, cnt int32, logg fp32).

    prefill: q [B][Hq][N][d] -> idx/logg [B][Hkv][T][topk], cnt [B][Hkv][T].
    decode:  q [B][Hq][d], N = Lmax = 64 * ksum.shape[2] -> idx/logg
             [B][Hkv][topk], cnt [B][Hkv].
    scores_out (optional, fp32): receives the raw scores, [B][Hkv][T][T]
    (prefill) or [B][Hkv][N/64] (decode), -inf past each row's C blocks.
    """
    lib = load_library()
    if mode == "prefill":
        B, Hq, N, d = q.shape
        T = -(-N // 64)
        shape = (B, Hkv, T)
        m = SAS_PREFILL
    elif mode == "decode":
        B, Hq, d = q.shape
        N = ksum.shape[2] * 64
        shape = (B, Hkv)
        m = SAS_DECODE
    else:
        raise ValueError(mode)
    if out is None:
        out = (torch.empty(shape + (topk,), dtype=torch.int32, device=q.device),
               torch.empty(shape, dtype=torch.int32, device=q.device),
               torch.empty(shape + (topk,), dtype=torch.float32, device=q.device))
    idx, cnt, logg = out
    need = lib.sas_select_workspace_size(B, Hq, Hkv, N, d, topk, m)
    w = _ws(need, q.device, ws)
    _check("sas_select", lib.sas_select(
        _ptr(q), _dt(q), _ptr(ksum), B, Hq, Hkv, N, d, topk, m, _ptr(lens), float(scale),
        _ptr(idx) if topk else None, _ptr(cnt), _ptr(logg) if topk else None,
        _ptr(scores_out), _ptr(w), w.numel(), _stream(stream)))
    return idx, cnt, logg


def sas_select_prefill_noalloc(q: torch.Tensor, ksum: torch.Tensor, Hkv: int, topk: int,
                               scale: float = 0.0, out=None, stream=None):
    """Prefill selection whose scratch is the library's fixed device array:
    the call itself allocates no device memory (pass `out` to supply the
    output buffers too). Returns (idx, cnt, logg) like sas_select."""
    lib = load_library()
    B, Hq, N, d = q.shape
    T = -(-N // 64)
    if out is None:
        out = (torch.empty((B, Hkv, T, topk), dtype=torch.int32, device=q.device),
               torch.empty((B, Hkv, T), dtype=torch.int32, device=q.device),
               torch.empty((B, Hkv, T, topk), dtype=torch.float32, device=q.device))
    idx, cnt, logg = out
    _check("sas_select_prefill_noalloc", lib.sas_select_prefill_noalloc(
        _ptr(q), _dt(q), _ptr(ksum), B, Hq, Hkv, N, d, topk, float(scale),
        _ptr(idx) if topk else None, _ptr(cnt), _ptr(logg) if topk else None, _stream(stream)))
    return idx, cnt, logg


def sas_attn_fwd(q, k, v, idx, cnt, logg, scale: float = 0.0, out=None, ws=None, stream=None):
    """Gated sparse prefill forward. Returns (o [B][Hq][N][d], lse [B][Hq][N] fp32)."""
    lib = load_library()
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    topk = idx.shape[-1]
    if out is None:
        out = (torch.empty_like(q), torch.empty((B, Hq, N), dtype=torch.float32, device=q.device))
    o, lse = out
    need = lib.sas_attn_fwd_workspace_size(B, Hq, Hkv, N, d, topk, _dt(q))
    w = _ws(need, q.device, ws)
    _check("sas_attn_fwd", lib.sas_attn_fwd(
        _ptr(q), _ptr(k), _ptr(v), _dt(q), B, Hq, Hkv, N, d, _ptr(idx) if topk else None,
        _ptr(cnt), _ptr(logg) if topk else None, topk, float(scale), _ptr(o), _ptr(lse),
        _ptr(w), w.numel(), _stream(stream)))
    return o, lse


def sas_attn_bwd(q, k, v, o, dout, lse, idx, cnt, logg, scale: float = 0.0, out=None, ws=None,
                 stream=None):
    """Backward of sas_attn_fwd. Returns (dq, dk, dv, dlogg)."""
    lib = load_library()
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    topk = idx.shape[-1]
    if out is None:
        out = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v),
               torch.empty(idx.shape, dtype=torch.float32, device=q.device))
    dq, dk, dv, dlogg = out
    need = lib.sas_attn_bwd_workspace_size(B, Hq, Hkv, N, d, topk, _dt(q))
    w = _ws(need, q.device, ws)
    _check("sas_attn_bwd", lib.sas_attn_bwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _dt(q), B, Hq, Hkv, N, d, _ptr(lse),
        _ptr(idx) if topk else None, _ptr(cnt), _ptr(logg) if topk else None, topk,
        float(scale), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dlogg) if topk else None, _ptr(w),
        w.numel(), _stream(stream)))
    return dq, dk, dv, dlogg


def sas_decode_workspace_size(B: int, Hq: int, Hkv: int, Lmax: int, d: int, topk: int) -> int:
    return load_library().sas_decode_workspace_size(B, Hq, Hkv, Lmax, d, topk)


def sas_decode(q, kc, vc, lens, ksum, topk: int, gated: int = 1, scale: float = 0.0, out=None,
               idx_out=None, ws=None, stream=None):
    """One decode step: q [B][Hq][d], caches [B][Hkv][Lmax][d] -> o [B][Hq][d]."""
    lib = load_library()
    B, Hq, d = q.shape
    Hkv, Lmax = kc.shape[1], kc.shape[2]
    if out is None:
        out = torch.empty_like(q)
    need = lib.sas_decode_workspace_size(B, Hq, Hkv, Lmax, d, topk)
    w = _ws(need, q.device, ws) if need else None  # the one-launch step needs none
    _check("sas_decode", lib.sas_decode(
        _ptr(q), _ptr(kc), _ptr(vc), _dt(q), B, Hq, Hkv, Lmax, d, _ptr(lens), _ptr(ksum), topk,
        int(gated), float(scale), _ptr(out), _ptr(idx_out), _ptr(w), 0 if w is None else w.numel(),
        _stream(stream)))
    return out


def sas_decode_attend(q, kc, vc, lens, idx, cnt, logg, gated: int = 1, scale: float = 0.0,
                      out=None, ws=None, stream=None):
    """Decode attention for a given selection (idx/cnt/logg as sas_select's
    decode outputs): q [B][Hq][d] -> o [B][Hq][d]."""
    lib = load_library()
    B, Hq, d = q.shape
    Hkv, Lmax = kc.shape[1], kc.shape[2]
    topk = idx.shape[-1]
    if out is None:
        out = torch.empty_like(q)
    need = lib.sas_decode_attend_workspace_size(B, Hq, Hkv, Lmax, d, topk)
    w = _ws(need, q.device, ws)
    _check("sas_decode_attend", lib.sas_decode_attend(
        _ptr(q), _ptr(kc), _ptr(vc), _dt(q), B, Hq, Hkv, Lmax, d, _ptr(lens),
        _ptr(idx) if topk else None, _ptr(cnt), _ptr(logg) if topk else None, topk, int(gated),
        float(scale), _ptr(out), _ptr(w), w.numel(), _stream(stream)))
    return out


def sas_block_summary_ex(k, sum_dtype=torch.float32, lens=None, out=None, stream=None):
    """Block summaries stored as sum_dtype (torch.float32 or torch.bfloat16)."""
    lib = load_library()
    B, H, N, d = k.shape
    if out is None:
        out = torch.empty((B, H, N // 64, d), dtype=sum_dtype, device=k.device)
    _check("sas_block_summary_ex", lib.sas_block_summary_ex(
        _ptr(k), _dt(k), B, H, N, d, _ptr(lens), _ptr(out), _dt(out), _stream(stream)))
    return out


def sas_block_summary_last(k, lens, ksum, block_table=None, npages: int = 0, stream=None):
    """Refresh each row's last complete block summary in place (decode upkeep).

    Contiguous: k [B][H][N][d], ksum [B][H][N/64][d]. Paged (block_table
    [B][max_blocks]): k is the pool [npages][H][64][d], ksum [npages][H][d],
    N = 64 * max_blocks. ksum's dtype (fp32 or bf16) is the summary type.
    """
    lib = load_library()
    if block_table is None:
        B, H, N, d = k.shape
    else:
        B, N = block_table.shape[0], 64 * block_table.shape[1]
        npages = npages or k.shape[0]
        H, d = k.shape[1], k.shape[3]
    _check("sas_block_summary_last", lib.sas_block_summary_last(
        _ptr(k), _dt(k), B, H, N, d, _ptr(lens), _ptr(ksum), _dt(ksum), _ptr(block_table),
        int(npages), _stream(stream)))
    return ksum


def sas_select_tokens(q, ksum, Hkv: int, topk: int, scale: float = 0.0, out=None, stream=None):
    """Per-token selection rows: idx/logg [B][Hkv][N][topk], cnt [B][Hkv][N]."""
    lib = load_library()
    B, Hq, N, d = q.shape
    if out is None:
        out = (torch.empty((B, Hkv, N, topk), dtype=torch.int32, device=q.device),
               torch.empty((B, Hkv, N), dtype=torch.int32, device=q.device),
               torch.empty((B, Hkv, N, topk), dtype=torch.float32, device=q.device))
    idx, cnt, logg = out
    _check("sas_select_tokens", lib.sas_select_tokens(
        _ptr(q), _dt(q), _ptr(ksum), B, Hq, Hkv, N, d, topk, float(scale), _ptr(idx), _ptr(cnt),
        _ptr(logg), _stream(stream)))
    return idx, cnt, logg


def sas_attn_fwd_tokens(q, k, v, idx, cnt, logg, scale: float = 0.0, out=None, stream=None):
    """Forward with per-token selection rows; returns (o, lse)."""
    lib = load_library()
    B, Hq, N, d = q.shape
    Hkv, topk = k.shape[1], idx.shape[-1]
    if out is None:
        out = (torch.empty_like(q), torch.empty((B, Hq, N), dtype=torch.float32, device=q.device))
    o, lse = out
    _check("sas_attn_fwd_tokens", lib.sas_attn_fwd_tokens(
        _ptr(q), _ptr(k), _ptr(v), _dt(q), B, Hq, Hkv, N, d, _ptr(idx), _ptr(cnt), _ptr(logg),
        topk, float(scale), _ptr(o), _ptr(lse), _stream(stream)))
    return o, lse


def sas_attn_bwd_tokens(q, k, v, o, do, lse, idx, cnt, logg, scale: float = 0.0, out=None,
                        ws=None, stream=None):
    """Backward with per-token selection rows; returns (dq, dk, dv, dlogg)."""
    lib = load_library()
    B, Hq, N, d = q.shape
    Hkv, topk = k.shape[1], idx.shape[-1]
    if out is None:
        out = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v),
               torch.empty((B, Hkv, N, topk), dtype=torch.float32, device=q.device))
    dq, dk, dv, dlogg = out
    nws = lib.sas_attn_bwd_tokens_workspace_size(B, Hq, Hkv, N, d)
    w = _ws(nws, q.device, ws)
    _check("sas_attn_bwd_tokens", lib.sas_attn_bwd_tokens(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _dt(q), B, Hq, Hkv, N, d, _ptr(lse),
        _ptr(idx), _ptr(cnt), _ptr(logg), topk, float(scale), _ptr(dq), _ptr(dk), _ptr(dv),
        _ptr(dlogg), _ptr(w), w.numel(), _stream(stream)))
    return dq, dk, dv, dlogg


def sas_select_bwd_tokens(q, ksum, Hkv: int, idx, cnt, dlogg, dq, dk, scale: float = 0.0,
                          ws=None, stream=None):
    """Per-token selector gradient (eq. 8), added into dq and dk in place."""
    lib = load_library()
    B, Hq, N, d = q.shape
    topk = idx.shape[-1]
    need = lib.sas_select_bwd_tokens_workspace_size(B, Hq, Hkv, N, d)
    w = _ws(need, q.device, ws)
    _check("sas_select_bwd_tokens", lib.sas_select_bwd_tokens(
        _ptr(q), _dt(q), _ptr(ksum), B, Hq, Hkv, N, d, topk, float(scale), _ptr(idx), _ptr(cnt),
        _ptr(dlogg), _ptr(dq), _ptr(dk), _ptr(w), w.numel(), _stream(stream)))
    return dq, dk


def sas_decode_ex(q, kc, vc, lens, ksum, topk: int, gated: int = 1, scale: float = 0.0, out=None,
                  idx_out=None, stream=None):
    """sas_decode reading summaries of ksum's dtype (fp32 or bf16)."""
    lib = load_library()
    B, Hq, d = q.shape
    Hkv, Lmax = kc.shape[1], kc.shape[2]
    if out is None:
        out = torch.empty_like(q)
    _check("sas_decode_ex", lib.sas_decode_ex(
        _ptr(q), _ptr(kc), _ptr(vc), _dt(q), B, Hq, Hkv, Lmax, d, _ptr(lens), _ptr(ksum),
        _dt(ksum), topk, int(gated), float(scale), _ptr(out), _ptr(idx_out), _stream(stream)))
    return out


def sas_decode_host(q_host, q_dev, kc, vc, lens, ksum, topk: int, o_dev, o_host, gated: int = 1,
                    scale: float = 0.0, idx_out=None, stream=None):
    """One decode step from pinned host q to pinned host o (copies and the
    kernel enqueued by one C call); q_dev and o_dev are device staging."""
    lib = load_library()
    if q_host.is_cuda or o_host.is_cuda:
        raise ValueError("q_host and o_host must be host tensors")
    B, Hq, d = q_dev.shape
    Hkv, Lmax = kc.shape[1], kc.shape[2]
    _check("sas_decode_host", lib.sas_decode_host(
        q_host.data_ptr(), _ptr(q_dev), _ptr(kc), _ptr(vc), _dt(q_dev), B, Hq, Hkv, Lmax, d,
        _ptr(lens), _ptr(ksum), topk, int(gated), float(scale), _ptr(o_dev), o_host.data_ptr(),
        _ptr(idx_out), _stream(stream)))
    return o_host


def sas_decode_paged(q, kpool, vpool, kspool, block_table, lens, topk: int, gated: int = 1,
                     scale: float = 0.0, out=None, idx_out=None, stream=None):
    """Decode over paged caches: kpool, vpool [npages][Hkv][64][d], kspool
    [npages][Hkv][d] fp32, block_table [B][max_blocks] -> o [B][Hq][d]."""
    lib = load_library()
    B, Hq, d = q.shape
    npages, Hkv = kpool.shape[0], kpool.shape[1]
    max_blocks = block_table.shape[1]
    if out is None:
        out = torch.empty_like(q)
    _check("sas_decode_paged", lib.sas_decode_paged(
        _ptr(q), _ptr(kpool), _ptr(vpool), _ptr(kspool), _dt(q), B, Hq, Hkv, npages, d,
        _ptr(block_table), max_blocks, _ptr(lens), topk, int(gated), float(scale), _ptr(out),
        _ptr(idx_out), _stream(stream)))
    return out


def sas_decode_paged_ex(q, kpool, vpool, kspool, block_table, lens, topk: int, gated: int = 1,
                        scale: float = 0.0, out=None, idx_out=None, stream=None):
    """sas_decode_paged with page summaries kspool [npages][Hkv][d] in fp32 or bf16
    (the summaries' dtype is taken from kspool)."""
    lib = load_library()
    B, Hq, d = q.shape
    npages, Hkv = kpool.shape[0], kpool.shape[1]
    max_blocks = block_table.shape[1]
    if out is None:
        out = torch.empty_like(q)
    _check("sas_decode_paged_ex", lib.sas_decode_paged_ex(
        _ptr(q), _ptr(kpool), _ptr(vpool), _ptr(kspool), _dt(kspool), _dt(q), B, Hq, Hkv, npages,
        d, _ptr(block_table), max_blocks, _ptr(lens), topk, int(gated), float(scale), _ptr(out),
        _ptr(idx_out), _stream(stream)))
    return out


def sas_select_bwd(q, ksum, Hkv: int, idx, cnt, dlogg, dq, dk, scale: float = 0.0, ws=None,
                   stream=None):
    """Add the gradient through the selector (eq. 8 of the gate) into dq and dk, in place."""
    lib = load_library()
    B, Hq, N, d = q.shape
    topk = idx.shape[-1]
    need = lib.sas_select_bwd_workspace_size(B, Hq, Hkv, N, d)
    w = _ws(need, q.device, ws)
    _check("sas_select_bwd", lib.sas_select_bwd(
        _ptr(q), _dt(q), _ptr(ksum), B, Hq, Hkv, N, d, topk, float(scale), _ptr(idx), _ptr(cnt),
        _ptr(dlogg), _ptr(dq), _ptr(dk), _ptr(w), w.numel(), _stream(stream)))
    return dq, dk


def sas_device_status(clear: bool = False, stream=None) -> tuple[int, str]:
    """Synchronise `stream` and read the kernels' device error words.

    Returns (status, message): SAS_ERR_TIMEOUT (4) if a bounded wait gave up,
    SAS_ERR_INTERNAL (5) if a selection index was out of range, 0 otherwise.
    clear=True resets the words after reading them. Does not raise.
    """
    lib = load_library()
    st = lib.sas_device_status(int(bool(clear)), _stream(stream))
    return st, lib.sas_last_error_message().decode()


def sas_debug_wait_timeout(stream=None) -> None:
    """Launch the self-test kernel whose wait nothing completes (gives up after 200 ms)."""
    lib = load_library()
    _check("sas_debug_wait_timeout", lib.sas_debug_wait_timeout(_stream(stream)))
