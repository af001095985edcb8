"""Python binding of libdsa_indexer (the B200 lightning indexer).

Argument marshalling only: every step of the indexer runs in the CUDA
kernels of ``libdsa_indexer.so`` behind the C ABI of
``include/dsa_indexer.h``. Names mirror the C entry points. PyTorch is used
for device memory and streams; there is no CPU path. Importing this package
raises if the library has not been built
(``python sparse_attention_lightning_tcgen05_b200/build.py``).
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdsa_indexer.so")

DSA_OK = 0
DSA_ERR_INVALID_ARG = 1
DSA_ERR_UNSUPPORTED = 2
DSA_ERR_WORKSPACE = 3
DSA_ERR_CUDA = 4
DSA_ERR_TIMEOUT = 5
DSA_ERR_DEVICE = 6

DSA_KV_BF16 = 0
DSA_KV_FP8_E4M3_E8M0_B32 = 1
DSA_MASK_POSITIONS = 0
DSA_MASK_CAUSAL = 1
DSA_MASK_COMPRESSED = 2
DSA_MASK_BOUND = float.fromhex("-0x1.FEp127")
DSA_FLAG_SCORES_IN_WORKSPACE = 1
DSA_FLAG_SELFTEST_STALL = 2

# Every symbol include/dsa_indexer.h and include/dsa_sparse_mqa.h declare.
EXPORTS = ("dsa_indexer_workspace_size", "dsa_indexer_score", "dsa_indexer_topk",
           "dsa_indexer_forward", "dsa_indexer_forward_noalloc",
           "dsa_indexer_get_error", "dsa_sparse_mqa_workspace_size",
           "dsa_sparse_mqa_forward", "dsa_indexer_prepare_workspace_size",
           "dsa_indexer_prepare", "dsa_status_string")


class dsa_indexer_desc_t(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32),
                ("D", ctypes.c_int32), ("index_topk", ctypes.c_int32),
                ("S", ctypes.c_int64), ("k_seq_stride", ctypes.c_int64),
                ("num_seqs", ctypes.c_int32), ("cu_seqlens", ctypes.c_void_p),
                ("dtype", ctypes.c_int), ("mask", ctypes.c_int),
                ("query_start", ctypes.c_int64), ("compress_ratio", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("pages_per_seq", ctypes.c_int32),
                ("num_pages", ctypes.c_int32), ("block_table", ctypes.c_void_p),
                ("flags", ctypes.c_uint32), ("wait_limit_ns", ctypes.c_uint64),
                ("cu_seqlens_host", ctypes.c_void_p)]


class dsa_sparse_mqa_desc_t(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("S", ctypes.c_int32), ("H", ctypes.c_int32),
                ("D", ctypes.c_int32), ("K", ctypes.c_int64), ("K_top", ctypes.c_int32),
                ("sm_scale", ctypes.c_float), ("wait_limit_ns", ctypes.c_uint64)]


class dsa_prepare_desc_t(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("D", ctypes.c_int32),
                ("hidden", ctypes.c_int32), ("q_lora_rank", ctypes.c_int32),
                ("rope_dim", ctypes.c_int32), ("k_norm_eps", ctypes.c_float),
                ("w_scale", ctypes.c_float), ("S", ctypes.c_int64),
                ("k_seq_stride", ctypes.c_int64), ("wait_limit_ns", ctypes.c_uint64)]


class DsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {dsa_status_string(status)}")


_BUILD_HINT = "python sparse_attention_lightning_tcgen05_b200/build.py"
if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with '{_BUILD_HINT}'")

_lib = ctypes.CDLL(LIB_PATH)
for _f in EXPORTS:
    if not hasattr(_lib, _f):
        raise ImportError(f"{LIB_PATH} lacks {_f} (stale build): rebuild with '{_BUILD_HINT}'")
_vp, _sz = ctypes.c_void_p, ctypes.c_size_t
_P = ctypes.POINTER(dsa_indexer_desc_t)
_lib.dsa_indexer_workspace_size.argtypes = [_P, ctypes.POINTER(_sz)]
_lib.dsa_indexer_score.argtypes = [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
_lib.dsa_indexer_topk.argtypes = [_P, _vp, _vp, _vp, _vp, _sz, _vp]
_lib.dsa_indexer_forward.argtypes = [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
_lib.dsa_indexer_forward_noalloc.argtypes = [_P, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
_lib.dsa_indexer_get_error.argtypes = [_vp, _vp, ctypes.POINTER(ctypes.c_int)]
_M = ctypes.POINTER(dsa_sparse_mqa_desc_t)
_lib.dsa_sparse_mqa_workspace_size.argtypes = [_M, ctypes.POINTER(_sz)]
_lib.dsa_sparse_mqa_forward.argtypes = [_M, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
_R = ctypes.POINTER(dsa_prepare_desc_t)
_lib.dsa_indexer_prepare_workspace_size.argtypes = [_R, ctypes.POINTER(_sz)]
_lib.dsa_indexer_prepare.argtypes = [_R] + [_vp] * 14 + [_sz, _vp]
_lib.dsa_status_string.argtypes = [ctypes.c_int]
_lib.dsa_status_string.restype = ctypes.c_char_p
for _f in EXPORTS[:-1]:
    getattr(_lib, _f).restype = ctypes.c_int


def _ptr(x) -> int | None:
    """A device pointer from a torch tensor, an int, or None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def make_desc(T, H, index_topk, *, D=128, S=0, k_seq_stride=0, num_seqs=0,
              cu_seqlens=None, dtype=DSA_KV_BF16, mask=DSA_MASK_POSITIONS,
              query_start=0, compress_ratio=0, page_size=0, pages_per_seq=0,
              num_pages=0, block_table=None, flags=0, wait_limit_ns=0,
              cu_seqlens_host=None):
    """A descriptor. cu_seqlens_host: a contiguous int32 numpy array (host
    memory) that the caller keeps alive while the descriptor is used."""
    host_cu = None
    if cu_seqlens_host is not None:
        assert cu_seqlens_host.dtype.name == "int32" and cu_seqlens_host.flags.c_contiguous
        host_cu = cu_seqlens_host.ctypes.data
    return dsa_indexer_desc_t(T=T, H=H, D=D, index_topk=index_topk, S=S,
                              k_seq_stride=k_seq_stride, num_seqs=num_seqs,
                              cu_seqlens=_ptr(cu_seqlens), dtype=dtype,
                              mask=mask, query_start=query_start,
                              compress_ratio=compress_ratio, page_size=page_size,
                              pages_per_seq=pages_per_seq, num_pages=num_pages,
                              block_table=_ptr(block_table), flags=flags,
                              wait_limit_ns=wait_limit_ns, cu_seqlens_host=host_cu)


def dsa_status_string(status: int) -> str:
    return _lib.dsa_status_string(int(status)).decode()


def _check(status: int, where: str) -> int:
    if status != DSA_OK:
        raise DsaError(status, where)
    return status


def dsa_indexer_workspace_size(desc) -> int:
    n = _sz(0)
    _check(_lib.dsa_indexer_workspace_size(ctypes.byref(desc), ctypes.byref(n)),
           "dsa_indexer_workspace_size")
    return n.value


def dsa_indexer_score(desc, q, q_scale, w, k, k_scale, positions, scores,
                      workspace, workspace_bytes, stream=None) -> int:
    return _check(_lib.dsa_indexer_score(
        ctypes.byref(desc), _ptr(q), _ptr(q_scale), _ptr(w), _ptr(k),
        _ptr(k_scale), _ptr(positions), _ptr(scores), _ptr(workspace),
        workspace_bytes, stream), "dsa_indexer_score")


def dsa_indexer_topk(desc, scores, positions, topk, workspace,
                     workspace_bytes, stream=None) -> int:
    return _check(_lib.dsa_indexer_topk(
        ctypes.byref(desc), _ptr(scores), _ptr(positions), _ptr(topk),
        _ptr(workspace), workspace_bytes, stream), "dsa_indexer_topk")


def dsa_indexer_forward(desc, q, q_scale, w, k, k_scale, positions, scores,
                        topk, workspace, workspace_bytes, stream=None) -> int:
    return _check(_lib.dsa_indexer_forward(
        ctypes.byref(desc), _ptr(q), _ptr(q_scale), _ptr(w), _ptr(k),
        _ptr(k_scale), _ptr(positions), _ptr(scores), _ptr(topk),
        _ptr(workspace), workspace_bytes, stream), "dsa_indexer_forward")


def dsa_indexer_forward_noalloc(desc, q, q_scale, w, k, k_scale, positions,
                                scores, topk, stream=None) -> int:
    """dsa_indexer_forward without a workspace: for callers that cannot
    allocate device memory; the library's fixed scratch is used instead
    (calls must not overlap on the GPU)."""
    return _check(_lib.dsa_indexer_forward_noalloc(
        ctypes.byref(desc), _ptr(q), _ptr(q_scale), _ptr(w), _ptr(k),
        _ptr(k_scale), _ptr(positions), _ptr(scores), _ptr(topk), stream),
        "dsa_indexer_forward_noalloc")


def dsa_indexer_get_error(workspace, stream=None) -> int:
    """Device-side status of the last call that used `workspace` (syncs)."""
    st = ctypes.c_int(0)
    _check(_lib.dsa_indexer_get_error(_ptr(workspace), stream, ctypes.byref(st)),
           "dsa_indexer_get_error")
    return st.value


def raw_status(fn_name: str, *args) -> int:
    """Call a C entry point and return its status code without raising
    (for callers that inspect error codes)."""
    return getattr(_lib, fn_name)(*args)


def current_stream_handle():
    """The cudaStream_t of torch's current CUDA stream."""
    import torch
    return torch.cuda.current_stream().cuda_stream


def make_mqa_desc(B, S, H, K, K_top, sm_scale, *, D=128, wait_limit_ns=0):
    return dsa_sparse_mqa_desc_t(B=B, S=S, H=H, D=D, K=K, K_top=K_top,
                                 sm_scale=sm_scale, wait_limit_ns=wait_limit_ns)


def dsa_sparse_mqa_workspace_size(desc) -> int:
    n = _sz(0)
    _check(_lib.dsa_sparse_mqa_workspace_size(ctypes.byref(desc), ctypes.byref(n)),
           "dsa_sparse_mqa_workspace_size")
    return n.value


def dsa_sparse_mqa_forward(desc, q, kv, sinks, topk, out, workspace, workspace_bytes,
                           stream=None) -> int:
    return _check(_lib.dsa_sparse_mqa_forward(
        ctypes.byref(desc), _ptr(q), _ptr(kv), _ptr(sinks), _ptr(topk), _ptr(out),
        _ptr(workspace), workspace_bytes, stream), "dsa_sparse_mqa_forward")


def make_prepare_desc(T, H, hidden, q_lora_rank, rope_dim, *, D=128, k_norm_eps=1e-6,
                      w_scale=1.0, S=None, k_seq_stride=0, wait_limit_ns=0):
    return dsa_prepare_desc_t(T=T, H=H, D=D, hidden=hidden, q_lora_rank=q_lora_rank,
                              rope_dim=rope_dim, k_norm_eps=k_norm_eps, w_scale=w_scale,
                              S=T if S is None else S, k_seq_stride=k_seq_stride,
                              wait_limit_ns=wait_limit_ns)


def dsa_indexer_prepare_workspace_size(desc) -> int:
    n = _sz(0)
    _check(_lib.dsa_indexer_prepare_workspace_size(ctypes.byref(desc), ctypes.byref(n)),
           "dsa_indexer_prepare_workspace_size")
    return n.value


def dsa_indexer_prepare(desc, x, qr, wq_b, wk, weights_proj, k_norm_weight, k_norm_bias,
                        cos, sin, positions, q_out, w_out, key_cache, workspace,
                        workspace_bytes, stream=None) -> int:
    return _check(_lib.dsa_indexer_prepare(
        ctypes.byref(desc), _ptr(x), _ptr(qr), _ptr(wq_b), _ptr(wk), _ptr(weights_proj),
        _ptr(k_norm_weight), _ptr(k_norm_bias), _ptr(cos), _ptr(sin), _ptr(positions),
        _ptr(q_out), _ptr(w_out), _ptr(key_cache), _ptr(workspace), workspace_bytes,
        stream), "dsa_indexer_prepare")
