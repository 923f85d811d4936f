"""A CSA layer's decode state on one GPU and one decode step through the C ABI.

Plumbing only: caches, window buffer, workspaces and outputs are torch allocations made once at
construction, so a step allocates nothing and can be captured in a CUDA graph.  The step is the
layer's hot path (sources: "DeepSeek-V4: エージェントが実際に使える100万トークンのコンテキスト", §ハイブリッド注意,
Fig. 3): the token that completes a group of r folds the group into one compressed entry
(csa_compress, pooling mode: C and Z are the token projections the model already computed) and the
same launch appends the entry and its indexer key to the FP4 caches; the lightning indexer scores every
entry (csa_index_scores, with the row histogram) and the top-k entries are selected (csa_topk), or both in
one cluster per sequence with the scores kept on chip (csa_index_topk with CSA_ONCHIP_TOPK), and attention
runs over them plus the window (csa_sparse_attn; optionally merging its splits inside their cluster).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import PackedCache, attn_kernel_count, attn_workspace_size, compress, index_scores, index_topk, \
    index_topk_workspace_size, pack_fp4, sparse_attn, topk, topk_workspace_size


@dataclass
class LayerShape:
    B: int
    n_max: int          # cache capacity (compressed entries per sequence)
    r: int = 4
    H: int = 64
    d: int = 512
    d_r: int = 64
    H_I: int = 8
    d_I: int = 128
    k: int = 512
    W: int = 128
    g_kv: float = 1.0
    g_k: float = 1.0
    g_q: float = 1.0
    rope_theta: float = 10000.0


class CSADecodeLayer:
    def __init__(self, s: LayerShape, device="cuda", early_start: bool = True, fused_index: bool = False,
                 cluster_merge: bool = False):
        """early_start: the step's indexer streams the key tiles below the new entry while the compressor
        still runs, and attention runs each query's window tile while the top-k still runs
        (CSA_EARLY_START; the step's inputs q, q_I, w and the window are never written by its kernels).
        fused_index: one csa_index_topk call with CSA_ONCHIP_TOPK (the scores stay on chip and each row is
        selected by its cluster); default: csa_index_scores into `scores` with its histogram + csa_topk
        (measured faster for the 128K decode step).
        cluster_merge: a query's attention splits merge inside their cluster (CSA_CLUSTER_MERGE); default:
        through the workspace and a merge kernel (measured faster for the 128K decode step)."""
        self.s = s
        self.early = early_start
        self.fused = fused_index
        self.cluster = cluster_merge
        dev = torch.device(device)
        self.kv = PackedCache(s.B, s.n_max, s.d, s.d_r, dev, s.g_kv)
        self.ki = PackedCache(s.B, s.n_max, s.d_I, 0, dev, s.g_k)
        self.win = torch.zeros((s.B, s.W, s.d), dtype=torch.bfloat16, device=dev)
        self.win_pos0 = torch.zeros((s.B,), dtype=torch.int64, device=dev)
        self.n_c = torch.zeros((s.B,), dtype=torch.int32, device=dev)
        self.row0 = torch.zeros((s.B,), dtype=torch.int32, device=dev)      # slot of the new entry
        self.pos0 = torch.zeros((s.B,), dtype=torch.int64, device=dev)      # first token of its group
        self.q_pos = torch.zeros((s.B, 1), dtype=torch.int64, device=dev)
        self.c_new = torch.empty((s.B, 1, s.d), dtype=torch.bfloat16, device=dev)
        self.kI_new = torch.empty((s.B, 1, s.d_I), dtype=torch.bfloat16, device=dev)
        self.idx = torch.empty((s.B, 1, s.k), dtype=torch.int32, device=dev)
        self.out = torch.empty((s.B, 1, s.H, s.d), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((s.B, 1, s.H), dtype=torch.float32, device=dev)
        qI = torch.empty((s.B, 1, s.H_I, s.d_I), dtype=torch.bfloat16, device=dev)
        w = torch.empty((s.B, 1, s.H_I), dtype=torch.float32, device=dev)
        q = torch.empty((s.B, 1, s.H, s.d), dtype=torch.bfloat16, device=dev)
        self.scores = torch.empty((s.B, s.n_max), dtype=torch.float32, device=dev)
        self.hist = torch.zeros((s.B, 4096), dtype=torch.int32, device=dev)   # score histogram (uint32 bits)
        ws_i = max(topk_workspace_size(self.ki, self.n_c, self.q_pos, B=s.B, Nq=1, ratio=s.r, k=s.k),
                   index_topk_workspace_size(qI, w, self.ki, self.n_c, self.q_pos, ratio=s.r, k=s.k))
        # sized for both launch plans (the flag may be switched off later, e.g. for stage-by-stage timing)
        ws_a = max(attn_workspace_size(q, self.q_pos, self.kv, self.n_c, self.idx, self.win, self.win_pos0,
                                       ratio=s.r, window=s.W, early_start=e, cluster=cluster_merge)
                   for e in (True, False))
        self.ws_index = torch.empty(max(ws_i, 1), dtype=torch.uint8, device=dev)
        self.ws_attn = torch.empty(max(ws_a, 1), dtype=torch.uint8, device=dev)
        self._attn_kernels = {e: attn_kernel_count(q, self.q_pos, self.kv, self.n_c, self.idx, self.win,
                                                   self.win_pos0, ratio=s.r, window=s.W, early_start=e,
                                                   cluster=cluster_merge) for e in (True, False)}

    def load_history(self, kv_src, kI_src, n_c: int):
        """Pack a prefix of n_c - 1 compressed entries (and index keys) into the caches: rows [B, n, d]."""
        pack_fp4(kv_src[:, : n_c - 1].contiguous(), self.kv)
        pack_fp4(kI_src[:, : n_c - 1].contiguous(), self.ki)
        self.set_position(n_c)

    def set_position(self, n_c: int):
        """The next step's token is the last one of group n_c - 1 (t = r n_c - 1)."""
        s = self.s
        t = s.r * n_c - 1
        self.n_c.fill_(n_c)
        self.row0.fill_(n_c - 1)
        self.pos0.fill_(s.r * (n_c - 1))
        self.q_pos.fill_(t)
        self.win_pos0.fill_(t - s.W + 1)

    @property
    def kernels_per_step(self):
        """pool + FP4 append, index scores and top-k (one launch with the on-chip top-k), and the attention
        call's kernels (csa_attn_kernel_count: the attention, and the split merge when a query is split)."""
        return (2 if self.fused else 3) + self._attn_kernels[self.early]

    def step(self, C, Z, b_pos, W_IK, q, q_I, w, stream=None, marks=None):
        """One decode step.  C, Z [B, r, d] bf16 (projections of the group's r tokens), q [B,1,H,d],
        q_I [B,1,H_I,d_I], w [B,1,H_I].  The window buffer must already hold tokens t-W+1 .. t.
        marks: optional 5 CUDA events recorded between the stages (compress+pack | index scores |
        top-k | attention; with the fused index the second stage is the whole index + top-k and the third
        is empty).  Returns (out [B,1,H,d] bf16, lse [B,1,H] fp32, idx [B,1,k] int32)."""
        s = self.s
        st = stream if stream is not None else torch.cuda.current_stream()

        def mark(i):
            if marks is not None:
                marks[i].record(st)

        mark(0)
        compress(C=C, Z=Z, b_pos=b_pos, ratio=s.r, d_rope=s.d_r, rope_theta=s.rope_theta, pos0=self.pos0,
                 W_IK=W_IK, c_out=self.c_new, kI_out=self.kI_new, kv_cache=self.kv, ki_cache=self.ki, row0=self.row0,
                 stream=st)
        mark(1)
        if self.fused:
            index_topk(q_I, w, self.ki, self.n_c, self.q_pos, ratio=s.r, k=s.k, g_q=s.g_q, idx_out=self.idx,
                       ws=self.ws_index, early_start=self.early, onchip=True, stream=st)
            mark(2)
        else:
            index_scores(q_I, w, self.ki, self.n_c, self.q_pos, self.scores, ratio=s.r, g_q=s.g_q, hist=self.hist,
                         k=s.k, early_start=self.early, stream=st)
            mark(2)
            topk(self.scores, self.ki, self.n_c, self.q_pos, B=s.B, Nq=1, ratio=s.r, k=s.k, idx_out=self.idx,
                 hist=self.hist, ws=self.ws_index, early_start=self.early, stream=st)
        mark(3)
        sparse_attn(q, self.q_pos, self.kv, self.n_c, self.idx, self.win, self.win_pos0, ratio=s.r, window=s.W,
                    out=self.out, lse=self.lse, ws=self.ws_attn, early_start=self.early, cluster=self.cluster,
                    stream=st)
        mark(4)
        return self.out, self.lse, self.idx
