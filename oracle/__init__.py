"""fp64 CPU oracle of the lightning indexer -- TEST INFRASTRUCTURE.

Only ``tests/``, the smoke check and the benchmark's CPU-baseline leg use this
package. It shares no code with the CUDA library: the arithmetic lives in
``dsa_oracle.c`` (plain C, fp64, OpenMP over rows); this module only builds
that file with gcc and marshals numpy arrays through ctypes.

Parity status: pinned (see ``tests/test_oracle_pins.py``) -- by brute-force
Python sorts, a BLAS matmul for H=1/w=1, head-permutation / additivity /
homogeneity / Hadamard invariants, exact integer cases, hand-derived golden
rows and the torch e4m3 decoding table.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

import dsa_synth

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsa_oracle.c")
_LIB = os.path.join(_HERE, "libdsa_oracle.so")


def build(force: bool = False) -> str:
    """Compile dsa_oracle.c into libdsa_oracle.so (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or \
            os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared",
                               "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Problem(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("T", ctypes.c_int32), ("H", ctypes.c_int32),
                ("D", ctypes.c_int32), ("num_seqs", ctypes.c_int32),
                ("S", ctypes.c_int64), ("k_seq_stride", ctypes.c_int64),
                ("positions", ctypes.c_void_p), ("cu_seqlens", ctypes.c_void_p),
                ("q", ctypes.c_void_p), ("q_scale", ctypes.c_void_p),
                ("w", ctypes.c_void_p), ("k", ctypes.c_void_p),
                ("k_scale", ctypes.c_void_p), ("query_start", ctypes.c_int64),
                ("compress_ratio", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("pages_per_seq", ctypes.c_int32), ("num_pages", ctypes.c_int32),
                ("block_table", ctypes.c_void_p)]


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.POINTER(_Problem)
        i64p = ctypes.POINTER(ctypes.c_int64)
        lib.orc_row_info.argtypes = [P, ctypes.c_int64, i64p, i64p, i64p, i64p]
        lib.orc_row_info.restype = ctypes.c_int
        lib.orc_score_rows.argtypes = [P, ctypes.c_int64, ctypes.c_void_p,
                                       ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.c_int]
        lib.orc_score_rows.restype = ctypes.c_int
        lib.orc_topk_rows.argtypes = [P, ctypes.c_int64, ctypes.c_void_p,
                                      ctypes.c_void_p, ctypes.c_void_p,
                                      ctypes.c_int32, ctypes.c_void_p,
                                      ctypes.c_int]
        lib.orc_topk_rows.restype = ctypes.c_int
        for name, argt in (("orc_bf16_value", ctypes.c_uint16),
                           ("orc_e4m3_value", ctypes.c_uint8),
                           ("orc_e8m0_value", ctypes.c_uint8)):
            getattr(lib, name).argtypes = [argt]
            getattr(lib, name).restype = ctypes.c_double
        lib.orc_mask_bound.argtypes = []
        lib.orc_mask_bound.restype = ctypes.c_double
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


class Problem:
    """An indexer problem: a workload description plus its host inputs."""

    def __init__(self, wl: dsa_synth.Workload, inputs: dict):
        self.wl = wl
        # keep contiguous references alive for the C side
        self._arrs = {k: (None if v is None else np.ascontiguousarray(v))
                      for k, v in inputs.items()}
        a = self._arrs
        assert a["w"].dtype == np.float32
        if wl.dtype == dsa_synth.DTYPE_FP8:
            assert a["q_scale"] is not None and a["k_scale"] is not None
        self._p = _Problem(
            mode=wl.mode, dtype=wl.dtype, T=wl.T, H=wl.H, D=wl.D,
            num_seqs=wl.num_seqs, S=wl.S, k_seq_stride=wl.k_seq_stride,
            positions=_ptr(a.get("positions")),
            cu_seqlens=_ptr(a.get("cu_seqlens")),
            q=_ptr(a["q"]), q_scale=_ptr(a.get("q_scale")),
            w=_ptr(a["w"]),
            k=_ptr(a["k"]), k_scale=_ptr(a.get("k_scale")),
            query_start=wl.query_start, compress_ratio=wl.compress_ratio,
            page_size=wl.page_size if wl.paged else 0,
            pages_per_seq=wl.pages_per_seq, num_pages=wl.num_pages,
            block_table=_ptr(a.get("block_table")))
        if wl.paged:
            bt = a["block_table"]
            assert bt is not None and bt.dtype == np.int32
            assert bt.shape == (wl.T, wl.pages_per_seq)

    def row_info(self, t: int):
        """(first_slot, row_len, last_valid, score_offset) of query row t."""
        out = [ctypes.c_int64() for _ in range(4)]
        rc = _load().orc_row_info(ctypes.byref(self._p), int(t),
                                  *[ctypes.byref(o) for o in out])
        if rc:
            raise IndexError(t)
        return tuple(o.value for o in out)

    def scores(self, rows, nthreads: int | None = None):
        """fp64 score rows (list of arrays, one per requested row)."""
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        lens = np.array([self.row_info(t)[1] for t in rows], np.int64)
        offs = np.concatenate([[0], np.cumsum(lens)[:-1]]).astype(np.int64)
        buf = np.empty(int(lens.sum()), np.float64)
        rc = _load().orc_score_rows(ctypes.byref(self._p), rows.size,
                                    _ptr(rows), _ptr(buf), _ptr(offs),
                                    nthreads or os.cpu_count() or 1)
        if rc:
            raise RuntimeError(f"orc_score_rows failed ({rc})")
        return [buf[o:o + n] for o, n in zip(offs, lens)]

    def topk(self, rows, score_rows, k: int, nthreads: int | None = None):
        """Top-k slot sets ([nrows, k] int32, -1 padded) of the given rows,
        selected from the given score rows (any source, fp64 or fp32)."""
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        lens = np.array([len(r) for r in score_rows], np.int64)
        for t, n in zip(rows, lens):
            assert n == self.row_info(t)[1]
        offs = np.concatenate([[0], np.cumsum(lens)[:-1]]).astype(np.int64)
        buf = np.concatenate([np.asarray(r, np.float64) for r in score_rows]) \
            if len(score_rows) else np.empty(0, np.float64)
        out = np.empty((rows.size, k), np.int32)
        rc = _load().orc_topk_rows(ctypes.byref(self._p), rows.size,
                                   _ptr(rows), _ptr(buf), _ptr(offs), int(k),
                                   _ptr(out), nthreads or os.cpu_count() or 1)
        if rc:
            raise RuntimeError(f"orc_topk_rows failed ({rc})")
        return out


def bf16_value(bits: int) -> float:
    return _load().orc_bf16_value(int(bits))


def e4m3_value(code: int) -> float:
    return _load().orc_e4m3_value(int(code))


def e8m0_value(code: int) -> float:
    return _load().orc_e8m0_value(int(code))


def mask_bound() -> float:
    return _load().orc_mask_bound()
