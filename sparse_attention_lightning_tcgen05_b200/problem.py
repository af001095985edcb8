"""Device buffers of one indexer problem, and calls through the C ABI.

Holds the inputs (moved to the GPU with torch), the score / top-k outputs and
the workspace, and calls ``dsa_indexer_score`` / ``_topk`` / ``_forward`` on
them. Memory and marshalling only.
"""
from __future__ import annotations

import numpy as np
import torch

from . import (DSA_FLAG_SCORES_IN_WORKSPACE, DSA_KV_BF16, DSA_MASK_CAUSAL, DSA_MASK_COMPRESSED, DSA_MASK_POSITIONS,
               dsa_indexer_forward, dsa_indexer_get_error, dsa_indexer_score,
               dsa_indexer_topk, dsa_indexer_workspace_size, make_desc)


def _dev(a, device, dtype=None):
    if a is None:
        return None
    if isinstance(a, torch.Tensor):
        return a.to(device)
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).to(device)


class DeviceProblem:
    """One indexer problem resident on a CUDA device."""

    def __init__(self, *, mode, T, H, index_topk, q, w, k, dtype=DSA_KV_BF16,
                 S=0, k_seq_stride=0, cu_seqlens=None, positions=None,
                 q_scale=None, k_scale=None, query_start=0, compress_ratio=0,
                 page_size=0, block_table=None, num_pages=0, device="cuda",
                 topk_only=False, wait_limit_ns=0):
        """topk_only: scores stay in the workspace (DSA_FLAG_SCORES_IN_WORKSPACE,
        forward with scores = NULL); self.scores is then a view of them."""
        self.mode, self.T, self.H, self.k = mode, T, H, index_topk
        self.S, self.dtype = S, dtype
        self.q = _dev(q, device)
        self.q_scale = _dev(q_scale, device)
        self.w = _dev(w, device)
        self.k_cache = _dev(k, device)
        self.k_scale = _dev(k_scale, device)
        self.positions = _dev(positions, device)
        self.cu_seqlens = _dev(cu_seqlens, device)
        self.block_table = _dev(block_table, device)
        self._cu_host = None
        if mode == DSA_MASK_CAUSAL:
            cu = np.asarray(cu_seqlens if not isinstance(cu_seqlens, torch.Tensor)
                            else cu_seqlens.cpu().numpy(), np.int64)
            lens = np.diff(cu)
            self.num_seqs = len(lens)
            n_scores = int((lens * lens).sum())
            self._cu_host = np.ascontiguousarray(cu, np.int32)
        else:
            self.num_seqs = 0
            n_scores = T * S
        self.topk_only = topk_only
        self.desc = make_desc(T, H, index_topk, S=S, k_seq_stride=k_seq_stride,
                              num_seqs=self.num_seqs, cu_seqlens=self.cu_seqlens,
                              dtype=dtype, mask=mode, query_start=query_start,
                              compress_ratio=compress_ratio, page_size=page_size,
                              pages_per_seq=(0 if block_table is None
                                             else int(block_table.shape[1])),
                              num_pages=num_pages, block_table=self.block_table,
                              flags=DSA_FLAG_SCORES_IN_WORKSPACE if topk_only else 0,
                              wait_limit_ns=wait_limit_ns,
                              cu_seqlens_host=self._cu_host)
        self.topk = torch.empty((T, index_topk), dtype=torch.int32, device=device)
        self.ws_bytes = dsa_indexer_workspace_size(self.desc)
        self.workspace = torch.zeros(self.ws_bytes, dtype=torch.uint8, device=device)
        if topk_only:
            # the rows the library keeps in the workspace, after its header
            self.scores = self.workspace[256:256 + 4 * n_scores].view(torch.float32)
        else:
            self.scores = torch.empty(n_scores, dtype=torch.float32, device=device)

    @classmethod
    def from_workload(cls, wl, inputs, device="cuda", **kw):
        """From a dsa_synth.Workload and its generated inputs."""
        mode = {0: DSA_MASK_POSITIONS, 1: DSA_MASK_CAUSAL,
                2: DSA_MASK_COMPRESSED}[wl.mode]
        return cls(mode=mode, T=wl.T, H=wl.H, index_topk=wl.index_topk,
                   q=inputs["q"], w=inputs["w"], k=inputs["k"], dtype=wl.dtype,
                   S=wl.S, k_seq_stride=wl.k_seq_stride,
                   cu_seqlens=inputs.get("cu_seqlens"),
                   positions=inputs.get("positions"),
                   q_scale=inputs.get("q_scale"), k_scale=inputs.get("k_scale"),
                   query_start=wl.query_start, compress_ratio=wl.compress_ratio,
                   page_size=wl.page_size if wl.paged else 0,
                   block_table=inputs.get("block_table"), num_pages=wl.num_pages,
                   device=device, **kw)

    def _stream(self, stream):
        if stream is None:
            return torch.cuda.current_stream().cuda_stream
        return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream

    def score(self, stream=None):
        dsa_indexer_score(self.desc, self.q, self.q_scale, self.w, self.k_cache,
                          self.k_scale, self.positions, self.scores,
                          self.workspace, self.ws_bytes, self._stream(stream))

    def run_topk(self, stream=None):
        dsa_indexer_topk(self.desc, self.scores, self.positions, self.topk,
                         self.workspace, self.ws_bytes, self._stream(stream))

    def forward(self, stream=None):
        dsa_indexer_forward(self.desc, self.q, self.q_scale, self.w,
                            self.k_cache, self.k_scale, self.positions,
                            None if self.topk_only else self.scores, self.topk,
                            self.workspace, self.ws_bytes, self._stream(stream))

    def device_status(self, stream=None) -> int:
        return dsa_indexer_get_error(self.workspace, self._stream(stream))
