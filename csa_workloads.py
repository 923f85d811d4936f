"""Seeded synthetic inputs for the CSA layer (shapes, sizes and value distributions only).

This module holds none of the layer's arithmetic: it draws Gaussian / Student-t tensors with
torch's seeded generators, casts them to the input dtypes and lays them out.  Both the CUDA path
(tests, bench, smoke) and the CPU oracle (tests) take their inputs from here.

Workloads (the long-context agent shapes the pages describe; no dataset is used):
  cfg1  "small layer": B=1, T=4096 (1024 entries), 16 decode positions t=4080..4095, H=8, d=128
        (96 FP4 + 32 RoPE), indexer 4x64, top-64, window 128, x and all W ~ N(0, 1/d_m), d_m=1024,
        b_pos ~ N(0, 0.1^2), global scale 2^-4.
  cfg2  "decode 128K": B=32, 131072 tokens (32768 entries), 1 new token, H=64, d=512 (448+64),
        indexer 8x128, top-512, window 128, N(0,1) entries / queries, w ~ N(0,1/8), 8 planted needles.
  cfg3  "prefill 32K": B=1, 32768 tokens in chunks of 4096, d_m=4096, x ~ N(0,1), W ~ N(0, 1/d_m).
  cfg4  "HCA 1M": C, Z ~ N(0,1) over 1048576 tokens, r=128 -> 8192 entries, decode B=16; plus
        reuse: Full over 262144 entries -> top-2048, Reindex -> top-512.
  cfg5  "decode 1M hierarchical": B=4, 262144 entries, top-2048, pool 8192, Student-t(3) query norms.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Shape:
    name: str
    B: int
    T: int                 # context tokens per sequence
    r: int                 # compression ratio
    H: int                 # query heads
    d: int                 # head dim (d_n + d_r)
    d_r: int               # RoPE slice kept in bf16
    H_I: int               # indexer heads
    d_I: int               # indexer head dim
    k: int                 # top-k
    W: int = 128           # window
    Nq: int = 1            # query positions per sequence
    d_m: int = 4096        # model width (compressor projection only)
    g: float = 1.0         # per-tensor FP4 global scale
    pool_blocks: int = 0   # hierarchical pool (blocks of 8), 0 = off
    extra: dict = field(default_factory=dict)

    @property
    def d_n(self) -> int:
        return self.d - self.d_r

    @property
    def n_c(self) -> int:
        return self.T // self.r


CFG1 = Shape("cfg1_small_layer_4k", B=1, T=4096, r=4, H=8, d=128, d_r=32, H_I=4, d_I=64, k=64,
             Nq=16, d_m=1024, g=2.0 ** -4)
CFG2 = Shape("cfg2_decode_b32_128k", B=32, T=131072, r=4, H=64, d=512, d_r=64, H_I=8, d_I=128, k=512)
CFG3 = Shape("cfg3_prefill_32k_chunk4096", B=1, T=32768, r=4, H=64, d=512, d_r=64, H_I=8, d_I=128,
             k=512, Nq=4096, d_m=4096, extra={"chunk": 4096})
CFG4_HCA = Shape("cfg4_hca_1m_b16", B=16, T=1048576, r=128, H=64, d=512, d_r=64, H_I=8, d_I=128, k=0)
CFG4_REUSE = Shape("cfg4_reuse_1m_b16", B=16, T=1048576, r=4, H=64, d=512, d_r=64, H_I=8, d_I=128,
                   k=2048, extra={"k2": 512})
CFG5 = Shape("cfg5_decode_b4_1m_hier", B=4, T=1048576, r=4, H=64, d=512, d_r=64, H_I=8, d_I=128,
             k=2048, pool_blocks=1024)
CONFIGS = {s.name: s for s in (CFG1, CFG2, CFG3, CFG4_HCA, CFG4_REUSE, CFG5)}


def gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def normal(shape, std, g, device="cpu", dtype=torch.bfloat16):
    """N(0, std^2) drawn in fp32 and cast to ``dtype`` (torch casts round to nearest even)."""
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def student_t_norms(n, df, g, device="cpu"):
    """|t_df| = |z| / sqrt(chi2_df / df), chi2 from df squared normals."""
    z = torch.randn((n,), generator=g, device=device)
    chi = torch.randn((n, df), generator=g, device=device).pow(2).sum(1)
    return (z / torch.sqrt(chi / df)).abs()


def plant_needles(kI_rows, q_I, w, positions, gain=4.0):
    """Overwrite indexer-key rows at ``positions`` with a vector aligned to the positively weighted
    query heads: gain * sqrt(d_I) * unit(sum_h max(w_h, 0) q_h).  kI_rows [n, d_I] (bf16, in place),
    q_I [H_I, d_I], w [H_I]."""
    dirn = (w.float().clamp(min=0)[:, None] * q_I.float()).sum(0)
    dirn = dirn / dirn.norm().clamp(min=1e-30)
    v = (gain * (q_I.shape[1] ** 0.5) * dirn).to(kI_rows.dtype)
    kI_rows[positions] = v


def decode_inputs(s: Shape, seed: int, device="cpu", n_c=None, B=None, needles: int = 8,
                  qnorm_student_t: bool = False):
    """One decode step of the CSA layer (all sequences at the same context length).

    Returns a dict of tensors:
      kv_src [B, n_c, d] bf16     compressed entries 0..n_c-2 (entry n_c-1 comes from the compressor)
      kI_src [B, n_c, d_I] bf16   indexer keys 0..n_c-2
      C, Z  [B, r, d] bf16        projections of the r tokens of the group that completes at t
      b_pos [r, d] f32, W_IK [d, d_I] bf16
      q [B, 1, H, d] bf16, q_I [B, 1, H_I, d_I] bf16, w [B, 1, H_I] f32
      win_kv [B, W, d] bf16 (positions t-W+1 .. t), win_pos0 [B] i64, q_pos [B, 1] i64, n_c [B] i32
      needle_pos [B, needles] i64
    """
    B = s.B if B is None else B
    n_c = s.n_c if n_c is None else n_c
    T = n_c * s.r
    t = T - 1
    g = gen(seed, device)
    d, dI = s.d, s.d_I
    out = {}
    out["kv_src"] = normal((B, n_c, d), 1.0, g, device)
    out["kI_src"] = normal((B, n_c, dI), 1.0, g, device)
    out["C"] = normal((B, s.r, d), 1.0, g, device)
    out["Z"] = normal((B, s.r, d), 1.0, g, device)
    out["b_pos"] = normal((s.r, d), 0.1, g, device, torch.float32)
    out["W_IK"] = normal((d, dI), d ** -0.5, g, device)
    q = normal((B, 1, s.H, d), 1.0, g, device)
    qI = normal((B, 1, s.H_I, dI), 1.0, g, device)
    if qnorm_student_t:
        dirs = torch.randn((B, 1, s.H_I, dI), generator=g, device=device)
        dirs = dirs / dirs.norm(dim=-1, keepdim=True)
        nrm = student_t_norms(B * s.H_I, 3, g, device).view(B, 1, s.H_I, 1) * dI ** 0.5
        qI = (dirs * nrm).to(torch.bfloat16)
        qd = torch.randn((B, 1, s.H, d), generator=g, device=device)
        qd = qd / qd.norm(dim=-1, keepdim=True)
        qn = student_t_norms(B * s.H, 3, g, device).view(B, 1, s.H, 1) * d ** 0.5
        q = (qd * qn).to(torch.bfloat16)
    out["q"] = q
    out["q_I"] = qI
    out["w"] = normal((B, 1, s.H_I), s.H_I ** -0.5, g, device, torch.float32)
    out["win_kv"] = normal((B, s.W, d), 1.0, g, device)
    out["win_pos0"] = torch.full((B,), t - s.W + 1, dtype=torch.int64, device=device)
    out["q_pos"] = torch.full((B, 1), t, dtype=torch.int64, device=device)
    out["n_c"] = torch.full((B,), n_c, dtype=torch.int32, device=device)
    if needles:
        pos = torch.randint(0, max(n_c - 1, 1), (B, needles), generator=g, device=device)
        for b in range(B):
            plant_needles(out["kI_src"][b], out["q_I"][b, 0], out["w"][b, 0], pos[b])
        out["needle_pos"] = pos
    return out


def small_layer_inputs(s: Shape = CFG1, seed: int = 0, device="cpu", peaked: bool = False):
    """cfg1: a 4096-token sequence through the compressor (projection mode), 16 decode positions."""
    g = gen(seed, device)
    T, d, dI, dm = s.T, s.d, s.d_I, s.d_m
    std = dm ** -0.5
    out = {}
    out["x"] = normal((s.B, T, dm), std, g, device)
    out["W_kv"] = normal((dm, d), std, g, device)
    out["W_g"] = normal((dm, d), std, g, device)
    out["b_pos"] = normal((s.r, d), 0.1, g, device, torch.float32)
    out["W_IK"] = normal((d, dI), d ** -0.5, g, device)
    q = normal((s.B, s.Nq, s.H, d), 1.0, g, device)
    if peaked:
        q = (q.float() * d ** 0.5).to(torch.bfloat16)
    out["q"] = q
    out["q_I"] = normal((s.B, s.Nq, s.H_I, dI), 1.0, g, device)
    out["w"] = normal((s.B, s.Nq, s.H_I), s.H_I ** -0.5, g, device, torch.float32)
    t0 = T - s.Nq
    out["q_pos"] = torch.arange(t0, T, dtype=torch.int64, device=device).repeat(s.B, 1)
    out["win_pos0"] = torch.full((s.B,), t0 - s.W + 1, dtype=torch.int64, device=device)
    return out
