"""One layer of the decode step: append the new token, select, attend.

Owns the per-layer output and workspace buffers so that a decode step is three library calls
(or one fused call) with no allocation. Every step runs in libckv's kernels.
"""

from __future__ import annotations

import torch

from . import binding as B


def cache_from_tensors(cfg: B.LayerConfig, batch: int, comp_codes, comp_scales, win_codes,
                       win_scales, comp_table, win_table) -> B.LayerCache:
    """Wraps caller-allocated pools and tables; allocates the residue ring [batch, r, D]."""
    dev = comp_codes.device
    return B.LayerCache(
        comp_codes=comp_codes, comp_scales=comp_scales, win_codes=win_codes,
        win_scales=win_scales,
        residue_kv=torch.zeros((batch, cfg.ratio, cfg.head_dim), dtype=torch.float32, device=dev),
        residue_logit=torch.zeros((batch, cfg.ratio), dtype=torch.float32, device=dev),
        comp_table=comp_table, win_table=win_table)


class DecodeLayer:
    """Buffers and calls of one layer for a batch of requests.

    top_k=None makes a dense layer (every completed entry attended, no indexer call)."""

    def __init__(self, cfg: B.LayerConfig, cache: B.LayerCache, batch: int, max_seq_len: int,
                 top_k: int | None):
        dev = cache.comp_codes.device
        self.cfg, self.cache, self.batch, self.max_seq_len, self.top_k = cfg, cache, batch, max_seq_len, top_k
        H, D = cfg.num_heads, cfg.head_dim
        self.out = torch.empty((batch, H, D), dtype=torch.float32, device=dev)
        self.status = torch.zeros(4, dtype=torch.int32, device=dev)  # word 0 is the status
        if top_k is not None:
            self.idx = torch.empty((batch, top_k), dtype=torch.int32, device=dev)
            self.cnt = torch.empty((batch,), dtype=torch.int32, device=dev)
            n = B.indexer_workspace_bytes(cfg, batch, max_seq_len, top_k)
            self.ws_index = torch.empty(max(n, 16), dtype=torch.uint8, device=dev)
        else:
            self.idx = self.cnt = self.ws_index = None
        n = B.attention_workspace_bytes(cfg, batch, max_seq_len, top_k or 0)
        self.ws_attn = torch.empty(max(n, 16), dtype=torch.uint8, device=dev)
        self.ws_step = None  # fused-step workspace, allocated by the first fused_step

    def append(self, prev_len, kv_new, logit_new, cu_new=None, max_new=1, stream=None):
        B.kv_compress_append(self.cfg, self.cache, prev_len, kv_new, logit_new, self.status,
                             cu_new=cu_new, max_new=max_new, max_seq_len=self.max_seq_len,
                             stream=stream)

    def replay_window(self, seq_len, kv, logit, stream=None):
        """SWA bounded replay: the recomputed raw tokens of the last min(W, L) positions of each
        request (kv [batch][W][D], logit [batch][W]) rewrite its window and unfinished group."""
        B.kv_window_replay(self.cfg, self.cache, seq_len, kv, logit, self.status,
                           max_seq_len=self.max_seq_len, stream=stream)

    def select(self, seq_len, q, scores=None, stream=None):
        B.sparse_indexer_topk(self.cfg, self.cache, seq_len, self.max_seq_len, q, self.top_k,
                              self.idx, self.cnt, self.ws_index, self.status, scores=scores,
                              stream=stream)

    def attend(self, seq_len, q, idx=None, cnt=None, stream=None):
        if idx is None and self.top_k is not None:
            idx, cnt = self.idx, self.cnt
        B.compressed_window_attention(self.cfg, self.cache, seq_len, self.max_seq_len, q, idx,
                                      cnt, self.out, self.ws_attn, self.status, stream=stream)
        return self.out

    def step(self, seq_len, prev_len, q, kv_new, logit_new, stream=None):
        """Append the decode token (position L-1), select (sparse layers), attend."""
        self.append(prev_len, kv_new, logit_new, stream=stream)
        if self.top_k is not None:
            self.select(seq_len, q, stream=stream)
        return self.attend(seq_len, q, stream=stream)

    def fused_step(self, seq_len, q, kv_new, logit_new, stream=None):
        """The same step as one ckv_decode_step call (its own workspace, allocated once)."""
        if self.ws_step is None:
            n = B.decode_step_workspace_bytes(self.cfg, self.batch, self.max_seq_len, self.top_k or 0)
            self.ws_step = torch.empty(max(n, 16), dtype=torch.uint8, device=self.out.device)
        B.decode_step(self.cfg, self.cache, seq_len, self.max_seq_len, q, kv_new, logit_new,
                      self.top_k or 0, self.idx, self.cnt, self.out, self.ws_step, self.status,
                      stream=stream)
        return self.out
