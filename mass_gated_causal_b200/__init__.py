"""Python binding of the MALA C ABI (include/mala.h): argument marshalling only.

Every step of the computation runs in the sm_100a kernels of ``libmala.so``;
this module only turns torch tensors into device pointers, allocates outputs
with torch and passes the current CUDA stream. There is no CPU fallback: if the
library is missing, importing this package raises.

Raw entry points keep the C names (``mala_fwd``, ``mala_prefill``, ``mala_fwd_varlen``,
``mala_bwd``, ``mala_bwd_varlen``, ``mala_decode``, ``mala_decode_paged``, ...).
``forward``, ``prefill``, ``forward_varlen``, ``backward``, ``backward_varlen``,
``decode`` and ``decode_paged`` are conveniences that allocate the outputs and
workspaces.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmala.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"MALA CUDA library not built: {LIB_PATH} is missing "
        "(run `python -m mass_gated_causal_b200.build` or __graft_entry__.build())")

_lib = ctypes.CDLL(LIB_PATH)

MALA_OK = 0
MALA_ERR_INVALID_ARG = 1
MALA_ERR_UNSUPPORTED = 2
MALA_ERR_WORKSPACE = 3
MALA_ERR_CUDA = 4
MALA_ERR_DEVICE_TIMEOUT = 5
MALA_ERR_RANGE = 6
MALA_FWD_PREFETCH_V = 1

EXPORTED = ("mala_status_string", "mala_abi_version", "mala_fwd", "mala_fwd_ex", "mala_prefill", "mala_fwd_varlen",
            "mala_fwd_workspace_size", "mala_bwd_workspace_size", "mala_bwd", "mala_bwd_varlen",
            "mala_decode_workspace_size", "mala_decode_default_splits", "mala_decode", "mala_decode_paged",
            "mala_decode_exact_workspace_size", "mala_decode_exact",
            "mala_decode_noalloc_max_bytes", "mala_decode_noalloc", "mala_test_hooks", "mala_check_status")

_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_lib.mala_status_string.argtypes = [_i]
_lib.mala_status_string.restype = ctypes.c_char_p
_lib.mala_abi_version.restype = _i
_lib.mala_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _f, _i, _i, _vp, _sz, _vp, _vp, _vp]
_lib.mala_fwd.restype = _i
_lib.mala_fwd_ex.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _f, _i, _i, _vp, _sz, _vp, _vp, _vp,
                             ctypes.c_uint]
_lib.mala_fwd_ex.restype = _i
_lib.mala_prefill.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _f, _i, _i, _vp, _sz, _vp, _vp,
                              _vp]
_lib.mala_prefill.restype = _i
_lib.mala_fwd_varlen.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _f, _f, _i, _i,
                                 _vp, _sz, _vp, _vp, _vp]
_lib.mala_fwd_varlen.restype = _i
_lib.mala_bwd_varlen.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _f,
                                 _i, _i, _vp, _sz, _vp, _vp, _vp]
_lib.mala_bwd_varlen.restype = _i
_lib.mala_decode_paged.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _f, _f, _i, _vp,
                                   _sz, _vp, _vp, _vp]
_lib.mala_decode_paged.restype = _i
_lib.mala_decode_exact_workspace_size.argtypes = [_i, _i, _i, _i, _i, _i]
_lib.mala_decode_exact_workspace_size.restype = _sz
_lib.mala_decode_exact.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _f, _i, _i, _vp, _sz, _vp, _vp,
                                   _vp]
_lib.mala_decode_exact.restype = _i
_lib.mala_fwd_workspace_size.argtypes = [_i, _i, _i, _i]
_lib.mala_fwd_workspace_size.restype = _sz
_lib.mala_bwd_workspace_size.argtypes = [_i, _i, _i, _i]
_lib.mala_bwd_workspace_size.restype = _sz
_lib.mala_bwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _f, _i, _i,
                          _vp, _sz, _vp, _vp, _vp]
_lib.mala_bwd.restype = _i
_lib.mala_decode_workspace_size.argtypes = [_i, _i, _i, _i]
_lib.mala_decode_workspace_size.restype = _sz
_lib.mala_decode_default_splits.argtypes = [_i, _i, _i, _i]
_lib.mala_decode_default_splits.restype = _i
_lib.mala_decode.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _f, _i, _i, _vp, _sz, _vp, _vp,
                             _vp]
_lib.mala_decode.restype = _i
_lib.mala_decode_noalloc_max_bytes.restype = _sz
_lib.mala_decode_noalloc.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _f, _i, _i, _vp, _vp, _vp]
_lib.mala_decode_noalloc.restype = _i
_lib.mala_test_hooks.argtypes = [ctypes.c_ulonglong, _i, _vp]
_lib.mala_test_hooks.restype = _i
_lib.mala_check_status.argtypes = [_vp]
_lib.mala_check_status.restype = _i


class MalaError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {mala_status_string(code)} ({code})")
        self.code = code


def _p(x) -> Optional[int]:
    """Device pointer of a tensor (or pass an int / None through)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int, where: str) -> None:
    if rc != MALA_OK:
        raise MalaError(rc, where)


# ------------------------------------------------------------- raw C names
def mala_status_string(code: int) -> str:
    return _lib.mala_status_string(int(code)).decode()


def mala_abi_version() -> int:
    return int(_lib.mala_abi_version())


def mala_fwd(q, k, v, o, lse, B, Hq, Hkv, L, d, scale, tau, Bq, Bk, workspace, workspace_bytes, kept_tiles,
             keep_map=None, stream=None) -> int:
    return int(_lib.mala_fwd(_p(q), _p(k), _p(v), _p(o), _p(lse), B, Hq, Hkv, L, d, float(scale), float(tau),
                             Bq, Bk, _p(workspace), int(workspace_bytes), _p(kept_tiles), _p(keep_map),
                             _stream(stream)))


def mala_fwd_ex(q, k, v, o, lse, B, Hq, Hkv, L, d, scale, tau, Bq, Bk, workspace, workspace_bytes, kept_tiles,
                keep_map=None, stream=None, flags=0) -> int:
    return int(_lib.mala_fwd_ex(_p(q), _p(k), _p(v), _p(o), _p(lse), B, Hq, Hkv, L, d, float(scale), float(tau),
                                Bq, Bk, _p(workspace), int(workspace_bytes), _p(kept_tiles), _p(keep_map),
                                _stream(stream), int(flags)))


def mala_prefill(q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, d, scale, tau, Bq, Bk, workspace, workspace_bytes,
                 kept_tiles, keep_map=None, stream=None) -> int:
    return int(_lib.mala_prefill(_p(q), _p(k), _p(v), _p(o), _p(lse), B, Hq, Hkv, Lq, Lk, d, float(scale),
                                 float(tau), Bq, Bk, _p(workspace), int(workspace_bytes), _p(kept_tiles),
                                 _p(keep_map), _stream(stream)))


def mala_fwd_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, num_seqs, max_seqlen_q, max_seqlen_k, total_q,
                    total_k, Hq, Hkv, d, scale, tau, Bq, Bk, workspace, workspace_bytes, kept_tiles, keep_map=None,
                    stream=None) -> int:
    return int(_lib.mala_fwd_varlen(_p(q), _p(k), _p(v), _p(o), _p(lse), _p(cu_seqlens_q), _p(cu_seqlens_k),
                                    num_seqs, max_seqlen_q, max_seqlen_k, total_q, total_k, Hq, Hkv, d,
                                    float(scale), float(tau), Bq, Bk, _p(workspace), int(workspace_bytes),
                                    _p(kept_tiles), _p(keep_map), _stream(stream)))


def mala_bwd_varlen(q, k, v, o, do, lse, dq, dk, dv, cu_seqlens, num_seqs, max_seqlen, total, Hq, Hkv, d, scale,
                    tau, Bq, Bk, workspace, workspace_bytes, kept_tiles, keep_map=None, stream=None) -> int:
    return int(_lib.mala_bwd_varlen(_p(q), _p(k), _p(v), _p(o), _p(do), _p(lse), _p(dq), _p(dk), _p(dv),
                                    _p(cu_seqlens), num_seqs, max_seqlen, total, Hq, Hkv, d, float(scale),
                                    float(tau), Bq, Bk, _p(workspace), int(workspace_bytes), _p(kept_tiles),
                                    _p(keep_map), _stream(stream)))


def mala_decode_paged(q, k_pages, v_pages, block_table, seqlens_k, o, lse, B, Hq, Hkv, num_pages, page_size,
                      max_pages_per_seq, d, scale, tau, n_splits, workspace, workspace_bytes, kept_tiles,
                      keep_map=None, stream=None) -> int:
    return int(_lib.mala_decode_paged(_p(q), _p(k_pages), _p(v_pages), _p(block_table), _p(seqlens_k), _p(o),
                                      _p(lse), B, Hq, Hkv, num_pages, page_size, max_pages_per_seq, d,
                                      float(scale), float(tau), n_splits, _p(workspace), int(workspace_bytes),
                                      _p(kept_tiles), _p(keep_map), _stream(stream)))


def mala_fwd_workspace_size(B, Hkv, L, d) -> int:
    return int(_lib.mala_fwd_workspace_size(B, Hkv, L, d))


def mala_bwd_workspace_size(B, Hq, L, d) -> int:
    return int(_lib.mala_bwd_workspace_size(B, Hq, L, d))


def mala_bwd(q, k, v, o, do, lse, dq, dk, dv, B, Hq, Hkv, L, d, scale, tau, Bq, Bk, workspace, workspace_bytes,
             kept_tiles, keep_map=None, stream=None) -> int:
    return int(_lib.mala_bwd(_p(q), _p(k), _p(v), _p(o), _p(do), _p(lse), _p(dq), _p(dk), _p(dv), B, Hq, Hkv, L,
                             d, float(scale), float(tau), Bq, Bk, _p(workspace), int(workspace_bytes),
                             _p(kept_tiles), _p(keep_map), _stream(stream)))


def mala_decode_workspace_size(B, Hq, d, n_splits) -> int:
    return int(_lib.mala_decode_workspace_size(B, Hq, d, n_splits))


def mala_decode_default_splits(B, Hkv, Lk, Bk) -> int:
    return int(_lib.mala_decode_default_splits(B, Hkv, Lk, Bk))


def mala_decode(q, kcache, vcache, o, lse, B, Hq, Hkv, Lk, d, scale, tau, Bk, n_splits, workspace,
                workspace_bytes, kept_tiles, keep_map=None, stream=None) -> int:
    return int(_lib.mala_decode(_p(q), _p(kcache), _p(vcache), _p(o), _p(lse), B, Hq, Hkv, Lk, d, float(scale),
                                float(tau), Bk, n_splits, _p(workspace), int(workspace_bytes), _p(kept_tiles),
                                _p(keep_map), _stream(stream)))


def mala_decode_exact_workspace_size(B, Hq, Lk, d, Bk, n_splits) -> int:
    return int(_lib.mala_decode_exact_workspace_size(B, Hq, Lk, d, Bk, n_splits))


def mala_decode_exact(q, kcache, vcache, o, lse, B, Hq, Hkv, Lk, d, scale, tau, Bk, n_splits, workspace,
                      workspace_bytes, kept_tiles, keep_map=None, stream=None) -> int:
    return int(_lib.mala_decode_exact(_p(q), _p(kcache), _p(vcache), _p(o), _p(lse), B, Hq, Hkv, Lk, d,
                                      float(scale), float(tau), Bk, n_splits, _p(workspace), int(workspace_bytes),
                                      _p(kept_tiles), _p(keep_map), _stream(stream)))


def mala_decode_noalloc_max_bytes() -> int:
    return int(_lib.mala_decode_noalloc_max_bytes())


def mala_decode_noalloc(q, kcache, vcache, o, lse, B, Hq, Hkv, Lk, d, scale, tau, Bk, n_splits, kept_tiles,
                        keep_map=None, stream=None) -> int:
    return int(_lib.mala_decode_noalloc(_p(q), _p(kcache), _p(vcache), _p(o), _p(lse), B, Hq, Hkv, Lk, d,
                                        float(scale), float(tau), Bk, n_splits, _p(kept_tiles), _p(keep_map),
                                        _stream(stream)))


def mala_test_hooks(wait_limit_ns: int = 0, stall_tile: int = -1, fwd_v_tiles=None) -> int:
    return int(_lib.mala_test_hooks(int(wait_limit_ns), int(stall_tile), _p(fwd_v_tiles)))


def mala_check_status(stream=None) -> int:
    return int(_lib.mala_check_status(_stream(stream)))


# ------------------------------------------------------------ conveniences
def forward(q, k, v, scale: float, tau: float, Bq: int = 128, Bk: int = 128, keep_map: bool = False,
            workspace=None, stream=None, prefetch_v: bool = False):
    """q [B,L,Hq,d], k/v [B,L,Hkv,d] bf16 CUDA tensors -> (o, lse, kept_tiles, keep_map|None).

    prefetch_v: fetch every V tile ahead of the gate (mala_fwd_ex with MALA_FWD_PREFETCH_V)."""
    import torch
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    if workspace is None:
        workspace = torch.empty((max(1, mala_fwd_workspace_size(B, Hkv, L, d)),), dtype=torch.uint8, device=q.device)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, L), dtype=torch.float32, device=q.device)
    kept = torch.empty((B * Hq,), dtype=torch.int32, device=q.device)
    km = None
    if keep_map:
        km = torch.full((B, Hq, -(-L // Bq), -(-L // Bk)), 255, dtype=torch.uint8, device=q.device)
    _check(mala_fwd_ex(q, k, v, o, lse, B, Hq, Hkv, L, d, scale, tau, Bq, Bk, workspace,
                       workspace.numel() * workspace.element_size(), kept, km, stream,
                       MALA_FWD_PREFETCH_V if prefetch_v else 0), "mala_fwd")
    return o, lse, kept, km


def prefill(q, k, v, scale: float, tau: float, Bq: int = 128, Bk: int = 128, keep_map: bool = False,
            workspace=None, stream=None):
    """q [B,Lq,Hq,d] (new queries), k/v [B,Lk,Hkv,d] (cache incl. the new keys)
    -> (o [B,Lq,Hq,d], lse [B,Hq,Lq], kept_tiles, keep_map|None)."""
    import torch
    B, Lq, Hq, d = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    if workspace is None:
        workspace = torch.empty((max(1, mala_fwd_workspace_size(B, Hkv, Lk, d)),), dtype=torch.uint8,
                                device=q.device)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    kept = torch.empty((B * Hq,), dtype=torch.int32, device=q.device)
    km = None
    if keep_map:
        km = torch.full((B, Hq, -(-Lq // Bq), -(-Lk // Bk)), 255, dtype=torch.uint8, device=q.device)
    _check(mala_prefill(q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, d, scale, tau, Bq, Bk, workspace,
                        workspace.numel() * workspace.element_size(), kept, km, stream), "mala_prefill")
    return o, lse, kept, km


def forward_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int, scale: float,
                   tau: float, Bq: int = 128, Bk: int = 128, keep_map: bool = False, workspace=None, stream=None):
    """Packed batch: q [total_q,Hq,d], k/v [total_k,Hkv,d] bf16; cu_seqlens_* int32 CUDA tensors
    [num_seqs+1] -> (o [total_q,Hq,d], lse [Hq,total_q], kept_tiles [num_seqs*Hq], keep_map|None)."""
    import torch
    total_q, Hq, d = q.shape
    total_k, Hkv = k.shape[0], k.shape[1]
    S = cu_seqlens_q.numel() - 1
    if workspace is None:
        workspace = torch.empty((max(1, mala_fwd_workspace_size(1, Hkv, total_k, d)),), dtype=torch.uint8,
                                device=q.device)
    o = torch.empty_like(q)
    lse = torch.empty((Hq, total_q), dtype=torch.float32, device=q.device)
    kept = torch.empty((S * Hq,), dtype=torch.int32, device=q.device)
    km = None
    if keep_map:
        km = torch.full((S, Hq, -(-max_seqlen_q // Bq), -(-max_seqlen_k // Bk)), 255, dtype=torch.uint8,
                        device=q.device)
    _check(mala_fwd_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, S, max_seqlen_q, max_seqlen_k, total_q,
                           total_k, Hq, Hkv, d, scale, tau, Bq, Bk, workspace,
                           workspace.numel() * workspace.element_size(), kept, km, stream), "mala_fwd_varlen")
    return o, lse, kept, km


def backward_varlen(q, k, v, o, do, lse, cu_seqlens, max_seqlen: int, scale: float, tau: float, Bq: int = 128,
                    Bk: int = 128, keep_map: bool = False, workspace=None, stream=None):
    """Packed training batch -> (dq, dk, dv, kept_tiles [num_seqs*Hq], keep_map|None)."""
    import torch
    total, Hq, d = q.shape
    Hkv = k.shape[1]
    S = cu_seqlens.numel() - 1
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    kept = torch.empty((S * Hq,), dtype=torch.int32, device=q.device)
    if workspace is None:
        workspace = torch.empty((mala_bwd_workspace_size(1, Hq, total, d),), dtype=torch.uint8, device=q.device)
    km = None
    if keep_map:
        km = torch.full((S, Hq, -(-max_seqlen // Bq), -(-max_seqlen // Bk)), 255, dtype=torch.uint8,
                        device=q.device)
    _check(mala_bwd_varlen(q, k, v, o, do, lse, dq, dk, dv, cu_seqlens, S, max_seqlen, total, Hq, Hkv, d, scale,
                           tau, Bq, Bk, workspace, workspace.numel() * workspace.element_size(), kept, km,
                           stream), "mala_bwd_varlen")
    return dq, dk, dv, kept, km


def backward(q, k, v, o, do, lse, scale: float, tau: float, Bq: int = 128, Bk: int = 128,
             keep_map: bool = False, workspace=None, stream=None):
    """-> (dq, dk, dv, kept_tiles, keep_map|None)."""
    import torch
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    kept = torch.empty((B * Hq,), dtype=torch.int32, device=q.device)
    ws_bytes = mala_bwd_workspace_size(B, Hq, L, d)
    if workspace is None:
        workspace = torch.empty((ws_bytes,), dtype=torch.uint8, device=q.device)
    km = None
    if keep_map:
        km = torch.full((B, Hq, -(-L // Bq), -(-L // Bk)), 255, dtype=torch.uint8, device=q.device)
    _check(mala_bwd(q, k, v, o, do, lse, dq, dk, dv, B, Hq, Hkv, L, d, scale, tau, Bq, Bk, workspace,
                    workspace.numel() * workspace.element_size(), kept, km, stream), "mala_bwd")
    return dq, dk, dv, kept, km


def decode(q, kcache, vcache, scale: float, tau: float, Bk: int = 128, n_splits: int = 0,
           keep_map: bool = False, workspace=None, stream=None):
    """q [B,Hq,d], kcache/vcache [B,Lk,Hkv,d] -> (o, lse, kept_tiles, keep_map|None, n_splits)."""
    import torch
    B, Hq, d = q.shape
    Lk, Hkv = kcache.shape[1], kcache.shape[2]
    if n_splits == 0:
        n_splits = mala_decode_default_splits(B, Hkv, Lk, Bk)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    kept = torch.empty((B * Hq,), dtype=torch.int32, device=q.device)
    ws_bytes = mala_decode_workspace_size(B, Hq, d, n_splits)
    if workspace is None:
        workspace = torch.empty((max(ws_bytes, 1),), dtype=torch.uint8, device=q.device)
    km = torch.full((B, Hq, -(-Lk // Bk)), 255, dtype=torch.uint8, device=q.device) if keep_map else None
    _check(mala_decode(q, kcache, vcache, o, lse, B, Hq, Hkv, Lk, d, scale, tau, Bk, n_splits, workspace,
                       workspace.numel() * workspace.element_size(), kept, km, stream), "mala_decode")
    return o, lse, kept, km, n_splits


def decode_paged(q, k_pages, v_pages, block_table, seqlens_k, scale: float, tau: float, n_splits: int = 0,
                 keep_map: bool = False, workspace=None, stream=None):
    """q [B,Hq,d]; k_pages/v_pages [num_pages,page,Hkv,d]; block_table [B,max_pages] and
    seqlens_k [B] int32 CUDA tensors -> (o, lse, kept_tiles, keep_map|None, n_splits)."""
    import torch
    B, Hq, d = q.shape
    num_pages, page, Hkv = k_pages.shape[0], k_pages.shape[1], k_pages.shape[2]
    maxp = block_table.shape[1]
    if n_splits == 0:
        n_splits = mala_decode_default_splits(B, Hkv, maxp * page, page)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    kept = torch.empty((B * Hq,), dtype=torch.int32, device=q.device)
    ws_bytes = mala_decode_workspace_size(B, Hq, d, n_splits)
    if workspace is None:
        workspace = torch.empty((max(ws_bytes, 1),), dtype=torch.uint8, device=q.device)
    km = torch.full((B, Hq, maxp), 255, dtype=torch.uint8, device=q.device) if keep_map else None
    _check(mala_decode_paged(q, k_pages, v_pages, block_table, seqlens_k, o, lse, B, Hq, Hkv, num_pages, page, maxp,
                             d, scale, tau, n_splits, workspace, workspace.numel() * workspace.element_size(), kept,
                             km, stream), "mala_decode_paged")
    return o, lse, kept, km, n_splits


def decode_exact(q, kcache, vcache, scale: float, tau: float, Bk: int = 128, n_splits: int = 0,
                 keep_map: bool = False, workspace=None, stream=None):
    """Split-independent decode -> (o, lse, kept_tiles, keep_map|None, n_splits)."""
    import torch
    B, Hq, d = q.shape
    Lk, Hkv = kcache.shape[1], kcache.shape[2]
    if n_splits == 0:
        n_splits = mala_decode_default_splits(B, Hkv, Lk, Bk)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    kept = torch.empty((B * Hq,), dtype=torch.int32, device=q.device)
    ws_bytes = mala_decode_exact_workspace_size(B, Hq, Lk, d, Bk, n_splits)
    if workspace is None:
        workspace = torch.empty((max(ws_bytes, 1),), dtype=torch.uint8, device=q.device)
    km = torch.full((B, Hq, -(-Lk // Bk)), 255, dtype=torch.uint8, device=q.device) if keep_map else None
    _check(mala_decode_exact(q, kcache, vcache, o, lse, B, Hq, Hkv, Lk, d, scale, tau, Bk, n_splits, workspace,
                             workspace.numel() * workspace.element_size(), kept, km, stream), "mala_decode_exact")
    return o, lse, kept, km, n_splits
