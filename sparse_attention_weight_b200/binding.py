"""Thin ctypes binding of libdsa.so (include/dsa.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  Tensors are torch tensors on the CUDA device; their data pointers
and the current torch stream are passed to the C ABI.  A missing library is an
error (there is no fallback).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdsa.so")

DSA_OK = 0
STATUS_NAMES = {0: "DSA_OK", 1: "DSA_ERR_INVALID_ARGUMENT", 2: "DSA_ERR_UNSUPPORTED",
                3: "DSA_ERR_WORKSPACE_TOO_SMALL", 4: "DSA_ERR_CUDA", 5: "DSA_ERR_DEVICE"}
DEV_BAD_QUERY, DEV_BAD_INDEX, DEV_TIMEOUT = 1, 2, 4
OP_INDEXER, OP_TOPK, OP_SPARSE_MLA, OP_FORWARD, OP_PROJECT, OP_MLA_BACKWARD, OP_FORWARD_HOST = 0, 1, 2, 3, 4, 5, 6

EXPORTS = ("dsa_workspace_size", "dsa_indexer_scores", "dsa_topk", "dsa_sparse_mla", "dsa_forward",
           "dsa_forward_ws_views", "dsa_read_device_status", "dsa_status_string", "dsa_abi_version",
           "dsa_indexer_scores_noalloc", "dsa_selftest_wait_timeout", "dsa_launch_count", "dsa_project_append",
           "dsa_indexer_scores_hist", "dsa_topk_hist", "dsa_topk_uses_hist", "dsa_sparse_mla_backward",
           "dsa_forward_host")
NOALLOC_MAX_Q = 16384


class DsaError(RuntimeError):
    def __init__(self, fn: str, status: int, flags: int | None = None):
        self.status = status
        self.flags = flags
        msg = f"{fn} returned {STATUS_NAMES.get(status, status)}"
        if flags is not None:
            msg += f" (device flags 0x{flags:x})"
        super().__init__(msg)


class DsaBatch(ctypes.Structure):
    _fields_ = [("num_seqs", ctypes.c_int32), ("num_q", ctypes.c_int32), ("max_kv_len", ctypes.c_int32),
                ("max_q_per_seq", ctypes.c_int32), ("kv_rows", ctypes.c_int64),
                ("kv_offset", ctypes.c_void_p), ("kv_len", ctypes.c_void_p), ("q_seq", ctypes.c_void_p),
                ("q_pos", ctypes.c_void_p), ("page_size", ctypes.c_int32), ("pages_per_seq", ctypes.c_int32),
                ("page_table", ctypes.c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    """Loads libdsa.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m sparse_attention_weight_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, sz, i32, i64, f32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_int64, ctypes.c_float
        bp = ctypes.POINTER(DsaBatch)
        L.dsa_workspace_size.argtypes = [i32, bp, i32, i32, i32, i64]
        L.dsa_workspace_size.restype = sz
        L.dsa_indexer_scores.argtypes = [bp, vp, vp, vp, i32, vp, i64, vp, sz, vp]
        L.dsa_topk.argtypes = [bp, vp, i64, i32, vp, vp, sz, vp]
        L.dsa_sparse_mla.argtypes = [bp, vp, vp, vp, i32, i32, f32, vp, vp, vp, sz, vp]
        L.dsa_forward.argtypes = [bp, vp, vp, vp, i32, vp, vp, i32, i32, f32, vp, vp, vp, sz, vp]
        L.dsa_indexer_scores_noalloc.argtypes = [bp, vp, vp, vp, i32, vp, i64, vp]
        L.dsa_project_append.argtypes = [bp, vp, vp, i32, i32, i32, f32, vp, vp, vp, vp, vp, vp, sz, vp]
        L.dsa_indexer_scores_hist.argtypes = [bp, vp, vp, vp, i32, vp, i64, vp, vp, sz, vp]
        L.dsa_topk_hist.argtypes = [bp, vp, i64, vp, i32, vp, vp, sz, vp]
        L.dsa_topk_uses_hist.argtypes = [bp, i32]
        L.dsa_sparse_mla_backward.argtypes = [bp, vp, vp, vp, i32, i32, f32, vp, vp, vp, vp, vp, vp, sz, vp]
        L.dsa_forward_host.argtypes = [bp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, f32, vp, vp, vp,
                                       vp, sz, ctypes.POINTER(vp)]
        L.dsa_topk_uses_hist.restype = i32
        L.dsa_selftest_wait_timeout.argtypes = [vp, sz, ctypes.c_uint32, vp]
        L.dsa_forward_ws_views.argtypes = [bp, i32, i32, i32, vp, ctypes.POINTER(vp), ctypes.POINTER(i64),
                                           ctypes.POINTER(vp)]
        L.dsa_read_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32), vp]
        L.dsa_status_string.argtypes = [i32]
        L.dsa_status_string.restype = ctypes.c_char_p
        L.dsa_abi_version.restype = i32
        L.dsa_launch_count.restype = ctypes.c_uint64
        for fn in ("dsa_indexer_scores", "dsa_topk", "dsa_sparse_mla", "dsa_forward", "dsa_forward_ws_views",
                   "dsa_read_device_status", "dsa_indexer_scores_noalloc", "dsa_selftest_wait_timeout",
                   "dsa_project_append", "dsa_indexer_scores_hist", "dsa_topk_hist", "dsa_sparse_mla_backward",
                   "dsa_forward_host"):
            getattr(L, fn).restype = i32
        _lib = L
    return _lib


def _ptr(t: torch.Tensor | None) -> int | None:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to the DSA library must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


@dataclass
class DeviceBatch:
    """Device arrays of a batch description plus the ctypes struct pointing at them."""
    kv_offset: torch.Tensor
    kv_len: torch.Tensor
    q_seq: torch.Tensor
    q_pos: torch.Tensor
    struct: DsaBatch
    page_table: torch.Tensor | None = None

    @classmethod
    def from_host(cls, b, device, kv_rows: int | None = None, max_kv_len: int | None = None,
                  max_q_per_seq: int | None = None, page_size: int = 0,
                  page_table=None) -> "DeviceBatch":
        """`b` has numpy kv_offset, kv_len, q_seq, q_pos (e.g. inputs.Batch).  With
        page_size > 0, `page_table` is an int32 array [B, pages_per_seq] of physical
        pages and `kv_rows` the physical rows; kv_offset is then not used."""
        off = torch.as_tensor(np.asarray(b.kv_offset, np.int64), device=device)
        ln = torch.as_tensor(np.asarray(b.kv_len, np.int32), device=device)
        qs = torch.as_tensor(np.asarray(b.q_seq, np.int32), device=device)
        qp = torch.as_tensor(np.asarray(b.q_pos, np.int32), device=device)
        kv_len = np.asarray(b.kv_len)
        if kv_rows is None:
            kv_rows = int((np.asarray(b.kv_offset) + kv_len).max()) if kv_len.size else 0
        if max_kv_len is None:
            max_kv_len = int(kv_len.max()) if kv_len.size else 1
        if max_q_per_seq is None:
            qsn = np.asarray(b.q_seq)
            max_q_per_seq = int(np.bincount(qsn).max()) if qsn.size else 0
        pt = None
        pps = 0
        if page_size:
            pt_host = np.ascontiguousarray(np.asarray(page_table, np.int32))
            pps = int(pt_host.shape[1])
            pt = torch.as_tensor(pt_host, device=device)
        st = DsaBatch(len(kv_len), len(np.asarray(b.q_pos)), max_kv_len, max_q_per_seq, kv_rows,
                      off.data_ptr(), ln.data_ptr(), qs.data_ptr(), qp.data_ptr(), int(page_size), pps,
                      pt.data_ptr() if pt is not None else None)
        return cls(off, ln, qs, qp, st, pt)


def workspace_size(op: int, batch: DeviceBatch, H_I: int = 64, H: int = 128, k: int = 2048, ld: int = 0) -> int:
    n = lib().dsa_workspace_size(op, ctypes.byref(batch.struct), H_I, H, k, ld)
    if n == 0:
        raise DsaError("dsa_workspace_size", 1)
    return int(n)


def workspace(op: int, batch: DeviceBatch, H_I: int = 64, H: int = 128, k: int = 2048, ld: int = 0,
              device="cuda") -> torch.Tensor:
    return torch.empty(workspace_size(op, batch, H_I, H, k, ld), dtype=torch.uint8, device=device)


def _check(fn: str, status: int):
    if status != DSA_OK:
        raise DsaError(fn, status)


def dsa_indexer_scores(batch: DeviceBatch, q_idx, k_idx, w, H_I: int, scores, ld: int, ws, stream=None):
    _check("dsa_indexer_scores", lib().dsa_indexer_scores(
        ctypes.byref(batch.struct), _ptr(q_idx), _ptr(k_idx), _ptr(w), H_I, _ptr(scores), ld, _ptr(ws),
        ws.numel(), _stream(stream)))


def dsa_indexer_scores_noalloc(batch: DeviceBatch, q_idx, k_idx, w, H_I: int, scores, ld: int, stream=None):
    """dsa_indexer_scores without a workspace (scratch in a fixed device array of the library)."""
    _check("dsa_indexer_scores_noalloc", lib().dsa_indexer_scores_noalloc(
        ctypes.byref(batch.struct), _ptr(q_idx), _ptr(k_idx), _ptr(w), H_I, _ptr(scores), ld, _stream(stream)))


def dsa_topk(batch: DeviceBatch, scores, ld: int, k: int, idx, ws, stream=None):
    _check("dsa_topk", lib().dsa_topk(ctypes.byref(batch.struct), _ptr(scores), ld, k, _ptr(idx), _ptr(ws),
                                      ws.numel(), _stream(stream)))


def dsa_sparse_mla(batch: DeviceBatch, q, kv, idx, k: int, H: int, sm_scale: float, out, lse, ws, stream=None):
    _check("dsa_sparse_mla", lib().dsa_sparse_mla(
        ctypes.byref(batch.struct), _ptr(q), _ptr(kv), _ptr(idx), k, H, sm_scale, _ptr(out), _ptr(lse), _ptr(ws),
        ws.numel(), _stream(stream)))


def dsa_forward_host(batch: DeviceBatch, host: dict, dev: dict, H_I: int, H: int, k: int, sm_scale: float, out,
                     lse, h_out, ws, streams=None):
    """dsa_forward from pinned host tensors `host` (q_idx, w, q, k_idx, kv) through the
    device buffers `dev` (same names), output copied into the pinned `h_out`;
    `streams` = (copy-in, compute, copy-out), default: the current stream thrice."""
    if streams is None:
        streams = (None, None, None)
    arr = (ctypes.c_void_p * 3)(*(_stream(s) for s in streams))
    _check("dsa_forward_host", lib().dsa_forward_host(
        ctypes.byref(batch.struct), _ptr(host["q_idx"]), _ptr(host["w"]), _ptr(host["q"]), _ptr(host["k_idx"]),
        _ptr(host["kv"]), _ptr(dev["q_idx"]), _ptr(dev["w"]), _ptr(dev["q"]), _ptr(dev["k_idx"]), _ptr(dev["kv"]),
        H_I, H, k, sm_scale, _ptr(out), _ptr(lse), _ptr(h_out), _ptr(ws), ws.numel(), arr))


def dsa_indexer_scores_hist(batch: DeviceBatch, q_idx, k_idx, w, H_I: int, scores, ld: int, hist, ws, stream=None):
    _check("dsa_indexer_scores_hist", lib().dsa_indexer_scores_hist(
        ctypes.byref(batch.struct), _ptr(q_idx), _ptr(k_idx), _ptr(w), H_I, _ptr(scores), ld, _ptr(hist), _ptr(ws),
        ws.numel(), _stream(stream)))


def dsa_topk_hist(batch: DeviceBatch, scores, ld: int, hist, k: int, idx, ws, stream=None):
    _check("dsa_topk_hist", lib().dsa_topk_hist(ctypes.byref(batch.struct), _ptr(scores), ld, _ptr(hist), k,
                                                _ptr(idx), _ptr(ws), ws.numel(), _stream(stream)))


def dsa_sparse_mla_backward(batch: DeviceBatch, q, kv, idx, k: int, H: int, sm_scale: float, out, lse, d_out, d_q,
                            d_kv, ws, stream=None):
    _check("dsa_sparse_mla_backward", lib().dsa_sparse_mla_backward(
        ctypes.byref(batch.struct), _ptr(q), _ptr(kv), _ptr(idx), k, H, sm_scale, _ptr(out), _ptr(lse), _ptr(d_out),
        _ptr(d_q), _ptr(d_kv), _ptr(ws), ws.numel(), _stream(stream)))


def topk_uses_hist(batch: DeviceBatch, k: int) -> bool:
    return bool(lib().dsa_topk_uses_hist(ctypes.byref(batch.struct), k))


def dsa_project_append(batch: DeviceBatch, hidden, w_all, d_model: int, H_I: int, H: int, rope_base: float, q_idx,
                       w, q, k_idx, kv, ws, stream=None):
    _check("dsa_project_append", lib().dsa_project_append(
        ctypes.byref(batch.struct), _ptr(hidden), _ptr(w_all), d_model, H_I, H, rope_base, _ptr(q_idx), _ptr(w),
        _ptr(q), _ptr(k_idx), _ptr(kv), _ptr(ws), ws.numel(), _stream(stream)))


def dsa_forward(batch: DeviceBatch, q_idx, k_idx, w, H_I: int, q, kv, H: int, k: int, sm_scale: float, out, lse,
                ws, stream=None):
    _check("dsa_forward", lib().dsa_forward(
        ctypes.byref(batch.struct), _ptr(q_idx), _ptr(k_idx), _ptr(w), H_I, _ptr(q), _ptr(kv), H, k, sm_scale,
        _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)))


def forward_ws_views(batch: DeviceBatch, H_I: int, H: int, k: int, ws) -> tuple[int, int, int]:
    """(scores pointer, ld, idx pointer) inside a forward workspace."""
    s, i = ctypes.c_void_p(), ctypes.c_void_p()
    ld = ctypes.c_int64()
    _check("dsa_forward_ws_views", lib().dsa_forward_ws_views(ctypes.byref(batch.struct), H_I, H, k, _ptr(ws),
                                                              ctypes.byref(s), ctypes.byref(ld), ctypes.byref(i)))
    return s.value, ld.value, i.value


def dsa_selftest_wait_timeout(ws, limit_us: int, stream=None):
    _check("dsa_selftest_wait_timeout", lib().dsa_selftest_wait_timeout(_ptr(ws), ws.numel(), limit_us,
                                                                        _stream(stream)))


def launch_count() -> int:
    """Kernels the library has launched in this process so far."""
    return int(lib().dsa_launch_count())


def read_device_status(ws, stream=None) -> int:
    """Synchronises the stream and returns the device status flags of `ws`."""
    flags = ctypes.c_uint32(0)
    st = lib().dsa_read_device_status(_ptr(ws), ctypes.byref(flags), _stream(stream))
    if st not in (DSA_OK, 5):
        raise DsaError("dsa_read_device_status", st)
    return int(flags.value)


def bits_to_tensor(a: np.ndarray, device) -> torch.Tensor:
    """Host numpy array (uint8 / uint16 bit patterns / float32 / int) -> device tensor of the same bits."""
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).to(device)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def tensor_to_bits(t: torch.Tensor) -> np.ndarray:
    a = t.cpu().numpy()
    if t.dtype == torch.int16:
        return a.view(np.uint16)
    return a
