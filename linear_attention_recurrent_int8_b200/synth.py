"""Seeded synthetic inputs for the decode / prefill workloads.

This module holds no arithmetic of the method: it only draws numbers.  Both the
CUDA path (through the tests and the benchmark) and the CPU oracle consume what
it produces.

Generator (counter-based, so any (b, h) slice can be drawn on its own):

* SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014): ``mix(z)`` is its output function, and the n-th
  output of a generator started at state ``s`` is ``mix(s + n * GOLDEN)``.
* The stream of tensor ``tid`` under ``seed`` starts at
  ``s = mix(seed * 2**32 + tid)``; element coordinate ``(a, b, c, j)`` (batch,
  head, time-or-row, channel) has counter
  ``n = ((a * 2**10 + b) * 2**24 + c) * 2**9 + j``.
* Uniforms: ``u = ((x >> 11) + 1) * 2**-53`` in (0, 1].
* Normals: Box-Muller (Box & Muller 1958), cosine branch,
  ``z = sqrt(-2 ln u(2n+1)) cos(2 pi u(2n+2))``.

The numpy implementation is the reference for tests (exact integer arithmetic
in uint64).  ``torch_normal`` draws the same integer streams with torch int64
ops on any device (used to fill large benchmark tensors on the GPU); its
floating-point transforms may differ from numpy's in the last ulp.

Workloads (seed 0 everywhere):
  q, k ~ N(0,1) then each d_k vector L2-normalised; v ~ N(0,1); for bf16 io
  all three are rounded to bf16 (round half to even) before anyone uses them.
  beta = sigmoid(x), alpha = exp(-softplus(x)) = sigmoid(-x), x ~ N(0,1),
  FP32; alpha per head ([B,T,H]) or per key channel ([B,T,H,d_k]).
  Initial state N(0,1) [B,H,d_v,d_k] with outlier rows (and columns) scaled.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

GOLDEN = 0x9E3779B97F4A7C15
M1 = 0xBF58476D1CE4E5B9
M2 = 0x94D049BB133111EB
MASK64 = (1 << 64) - 1

TID_Q, TID_K, TID_V, TID_ALPHA, TID_BETA, TID_S0, TID_OUT_ROWS, TID_OUT_COLS = range(1, 9)

CAP_B, CAP_H, CAP_T, CAP_D = 1 << 12, 1 << 10, 1 << 24, 1 << 9


# --------------------------------------------------------------------------
# SplitMix64, numpy (uint64, wrapping arithmetic is well defined)
# --------------------------------------------------------------------------

def mix64_int(z: int) -> int:
    """SplitMix64 output function on a Python int (reference for the tests)."""
    z &= MASK64
    z = ((z ^ (z >> 30)) * M1) & MASK64
    z = ((z ^ (z >> 27)) * M2) & MASK64
    return z ^ (z >> 31)


def splitmix64_sequence(seed: int, count: int) -> list[int]:
    """The first ``count`` outputs of SplitMix64 started at ``seed``."""
    return [mix64_int(seed + (i + 1) * GOLDEN) for i in range(count)]


def _mix64(z: np.ndarray) -> np.ndarray:
    z = z.astype(np.uint64, copy=True)
    with np.errstate(over="ignore"):
        z ^= z >> np.uint64(30)
        z *= np.uint64(M1)
        z ^= z >> np.uint64(27)
        z *= np.uint64(M2)
        z ^= z >> np.uint64(31)
    return z


def stream_base(seed: int, tid: int) -> int:
    return mix64_int(((seed & 0xFFFFFFFF) << 32) + tid)


def counters(a, b, c, j) -> np.ndarray:
    """Counter of element (a, b, c, j); arguments broadcast."""
    a, b, c, j = (np.asarray(x, np.uint64) for x in (a, b, c, j))
    return ((a * np.uint64(CAP_H) + b) * np.uint64(CAP_T) + c) * np.uint64(CAP_D) + j


def raw_u64(seed: int, tid: int, n: np.ndarray) -> np.ndarray:
    """The (n+1)-th SplitMix64 output of stream (seed, tid), for each counter n."""
    base = np.uint64(stream_base(seed, tid))
    with np.errstate(over="ignore"):
        return _mix64(base + (np.asarray(n, np.uint64) + np.uint64(1)) * np.uint64(GOLDEN))


def uniform(seed: int, tid: int, n: np.ndarray) -> np.ndarray:
    x = raw_u64(seed, tid, n)
    return ((x >> np.uint64(11)).astype(np.float64) + 1.0) * 2.0 ** -53


def normal(seed: int, tid: int, n: np.ndarray) -> np.ndarray:
    n = np.asarray(n, np.uint64)
    u1 = uniform(seed, tid, n * np.uint64(2))
    u2 = uniform(seed, tid, n * np.uint64(2) + np.uint64(1))
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)


def grid(seed: int, tid: int, bs, hs, cs, js) -> np.ndarray:
    """N(0,1) draws on the grid bs x cs x hs x js (layout [B, T, H, d])."""
    bs, hs, cs, js = (np.asarray(x, np.uint64) for x in (bs, hs, cs, js))
    n = counters(bs[:, None, None, None], hs[None, None, :, None],
                 cs[None, :, None, None], js[None, None, None, :])
    return normal(seed, tid, n)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round to the nearest bfloat16 (ties to even); returns float32 values."""
    f = np.ascontiguousarray(x, np.float32)
    bits = f.view(np.uint32).astype(np.uint64)
    bias = np.uint64(0x7FFF) + ((bits >> np.uint64(16)) & np.uint64(1))
    out = (((bits + bias) >> np.uint64(16)) << np.uint64(16)).astype(np.uint32)
    return out.view(np.float32)


def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


# --------------------------------------------------------------------------
# Workloads
# --------------------------------------------------------------------------

@dataclass
class DecodeWorkload:
    """One decode workload: shapes, gate kind, window, compensators, io type."""
    name: str
    batch: int
    heads: int
    d_k: int
    d_v: int
    steps: int
    window: int
    n_comp: int
    gate: str = "scalar"          # "scalar" (Gated DeltaNet) or "diag" (KDA)
    io: str = "bf16"              # "fp32" or "bf16"
    smoothing: bool = True
    outlier_rows: int = 0
    outlier_cols: int = 0
    outlier_scale: float = 30.0
    seed: int = 0
    delta: int = 1                # 1: delta rule (b = D k); 0: b = 0 (Mamba2 / GLA rows)
    extra: dict = field(default_factory=dict)

    @property
    def nh(self):
        return self.batch * self.heads


def _outlier_count(d: int) -> int:
    return max(1, int(round(0.01 * d)))


WORKLOADS = {
    # single GDN head, d=64, 256 steps, W=16, r=4, fp32, 2 rows x50
    "gdn_1x1_d64_fp32": DecodeWorkload("gdn_1x1_d64_fp32", 1, 1, 64, 64, 256, 16, 4, "scalar",
                                       "fp32", True, 2, 0, 50.0),
    # GDN decode B=64, H=16, d=128, 1024 steps, bf16, W=16, r=4
    "gdn_64x16_d128_bf16": DecodeWorkload("gdn_64x16_d128_bf16", 64, 16, 128, 128, 1024, 16, 4,
                                          "scalar", "bf16", True, _outlier_count(128),
                                          _outlier_count(128), 30.0),
    # KDA-style diag gate B=128, H=32, d=128, 2048 steps, bf16, W=16, r=8
    "kda_128x32_d128_bf16": DecodeWorkload("kda_128x32_d128_bf16", 128, 32, 128, 128, 2048, 16, 8,
                                           "diag", "bf16", True, _outlier_count(128),
                                           _outlier_count(128), 30.0),
    # large-batch GDN decode B=256, H=32, d=128, 4096 steps, bf16, W=16, r=4 (headline)
    "gdn_256x32_d128_bf16": DecodeWorkload("gdn_256x32_d128_bf16", 256, 32, 128, 128, 4096, 16, 4,
                                           "scalar", "bf16", True, _outlier_count(128),
                                           _outlier_count(128), 30.0),
}

# chunked GDN prefill: B=2, H=32, d=128, T=65536, bf16, snapshot every 1024,
# then 512 decode steps (W=16, r=4) from the last snapshot
PREFILL_WORKLOAD = dict(name="gdn_prefill_2x32_d128_T65536_bf16", batch=2, heads=32, d_k=128,
                        d_v=128, T=65536, chunk=64, snapshot_every=1024, n_comp=4, window=16,
                        decode_steps=512, io="bf16", seed=0)


def tokens(seed: int, batch_idx, head_idx, t0: int, t1: int, d_k: int, d_v: int,
           gate: str, io: str):
    """Inputs for tokens t0..t1-1 of sequences ``batch_idx`` and heads ``head_idx``.

    Returns dict q, k [nb, T, nh, d_k], v [nb, T, nh, d_v] (float32 holding io
    values), alpha [nb, T, nh] or [nb, T, nh, d_k] and beta [nb, T, nh] (float32)."""
    bs = np.asarray(batch_idx)
    hs = np.asarray(head_idx)
    ts = np.arange(t0, t1)
    jk = np.arange(d_k)
    jv = np.arange(d_v)
    q = grid(seed, TID_Q, bs, hs, ts, jk)
    k = grid(seed, TID_K, bs, hs, ts, jk)
    v = grid(seed, TID_V, bs, hs, ts, jv)
    q = q / np.linalg.norm(q, axis=-1, keepdims=True)
    k = k / np.linalg.norm(k, axis=-1, keepdims=True)
    cast = round_bf16 if io == "bf16" else (lambda a: np.asarray(a, np.float32))
    q, k, v = cast(q), cast(k), cast(v)
    xb = grid(seed, TID_BETA, bs, hs, ts, np.arange(1))[..., 0]
    beta = sigmoid(xb).astype(np.float32)
    if gate == "diag":
        xa = grid(seed, TID_ALPHA, bs, hs, ts, jk)
    else:
        xa = grid(seed, TID_ALPHA, bs, hs, ts, np.arange(1))[..., 0]
    alpha = sigmoid(-xa).astype(np.float32)  # exp(-softplus(x))
    return dict(q=q, k=k, v=v, alpha=alpha, beta=beta)


def _pick(seed: int, tid: int, b: int, h: int, d: int, count: int) -> np.ndarray:
    """``count`` distinct seeded indices in [0, d) for head (b, h)."""
    keys = raw_u64(seed, tid, counters(b, h, 0, np.arange(d)))
    return np.sort(np.argsort(keys, kind="stable")[:count])


def initial_state(seed: int, batch_idx, head_idx, d_k: int, d_v: int, outlier_rows: int,
                  outlier_cols: int, outlier_scale: float) -> np.ndarray:
    """N(0,1) initial state [nb, nh, d_v, d_k] (float32) with seeded outlier
    rows and columns multiplied by ``outlier_scale``."""
    bs = np.asarray(batch_idx)
    hs = np.asarray(head_idx)
    S = grid(seed, TID_S0, bs, hs, np.arange(d_v), np.arange(d_k))  # [nb, dv, nh, dk]
    S = np.ascontiguousarray(S.transpose(0, 2, 1, 3))
    for ib, b in enumerate(bs):
        for ih, h in enumerate(hs):
            if outlier_rows:
                S[ib, ih, _pick(seed, TID_OUT_ROWS, int(b), int(h), d_v, outlier_rows), :] *= outlier_scale
            if outlier_cols:
                S[ib, ih, :, _pick(seed, TID_OUT_COLS, int(b), int(h), d_k, outlier_cols)] *= outlier_scale
    return S.astype(np.float32)


# --------------------------------------------------------------------------
# torch path (same integer streams; for filling large tensors on a device)
# --------------------------------------------------------------------------

def _to_i64(x: int) -> int:
    x &= MASK64
    return x - (1 << 64) if x >= 1 << 63 else x


def _torch_mix64(z):
    import torch

    def srl(x, s):  # logical right shift on int64 bit patterns
        return (x >> s) & ((1 << (64 - s)) - 1)

    z = z ^ srl(z, 30)
    z = z * torch.tensor(_to_i64(M1), dtype=torch.int64, device=z.device)
    z = z ^ srl(z, 27)
    z = z * torch.tensor(_to_i64(M2), dtype=torch.int64, device=z.device)
    return z ^ srl(z, 31)


def torch_raw_u64(seed: int, tid: int, n):
    """Same as :func:`raw_u64` on an int64 torch tensor of counters (bit pattern)."""
    import torch
    base = torch.tensor(_to_i64(stream_base(seed, tid)), dtype=torch.int64, device=n.device)
    gold = torch.tensor(_to_i64(GOLDEN), dtype=torch.int64, device=n.device)
    return _torch_mix64(base + (n + 1) * gold)


def torch_grid(seed: int, tid: int, bs, hs, cs, js, device):
    """N(0,1) draws on the grid [len(bs), len(cs), len(hs), len(js)] on ``device`` (float64)."""
    import torch
    t = lambda x: torch.as_tensor(np.asarray(x, np.int64), device=device)
    b, h, c, j = t(bs), t(hs), t(cs), t(js)
    n = (((b[:, None, None, None] * CAP_H + h[None, None, :, None]) * CAP_T
          + c[None, :, None, None]) * CAP_D + j[None, None, None, :])

    def unif(m):
        x = torch_raw_u64(seed, tid, m)
        hi = ((x >> 11) & ((1 << 53) - 1)).to(torch.float64)
        return (hi + 1.0) * 2.0 ** -53

    u1 = unif(2 * n)
    u2 = unif(2 * n + 1)
    return torch.sqrt(-2.0 * torch.log(u1)) * torch.cos(2.0 * math.pi * u2)


def torch_tokens(seed: int, batch, heads: int, t0: int, t1: int, d_k: int, d_v: int,
                 gate: str, io: str, device):
    """Device-side counterpart of :func:`tokens` for all heads of the sequences
    ``batch`` (a count B, meaning sequences 0..B-1, or the sequences' global
    indices, so that a shard draws exactly its slice of the global batch).

    Returns q, k, v in the io dtype and alpha, beta in float32, layout [B, T, H, d]."""
    import torch
    bs = np.arange(batch) if np.ndim(batch) == 0 else np.asarray(batch)
    hs, ts = np.arange(heads), np.arange(t0, t1)
    jk, jv = np.arange(d_k), np.arange(d_v)
    q = torch_grid(seed, TID_Q, bs, hs, ts, jk, device)
    k = torch_grid(seed, TID_K, bs, hs, ts, jk, device)
    v = torch_grid(seed, TID_V, bs, hs, ts, jv, device)
    q = q / torch.linalg.vector_norm(q, dim=-1, keepdim=True)
    k = k / torch.linalg.vector_norm(k, dim=-1, keepdim=True)
    dt = torch.bfloat16 if io == "bf16" else torch.float32
    q, k, v = (x.to(torch.float32).to(dt) for x in (q, k, v))
    beta = torch.sigmoid(torch_grid(seed, TID_BETA, bs, hs, ts, [0], device)[..., 0]).float()
    xa = torch_grid(seed, TID_ALPHA, bs, hs, ts, jk if gate == "diag" else [0], device)
    if gate != "diag":
        xa = xa[..., 0]
    alpha = torch.sigmoid(-xa).float()
    return dict(q=q.contiguous(), k=k.contiguous(), v=v.contiguous(), alpha=alpha.contiguous(),
                beta=beta.contiguous())


def torch_initial_state(seed: int, batch_idx, head_idx, d_k: int, d_v: int, outlier_rows: int,
                        outlier_cols: int, outlier_scale: float, device):
    """Device-side counterpart of :func:`initial_state`: [nb, nh, d_v, d_k] float32."""
    import torch
    bs = np.asarray(batch_idx)
    hs = np.asarray(head_idx)
    S = torch_grid(seed, TID_S0, bs, hs, np.arange(d_v), np.arange(d_k), device)
    S = S.permute(0, 2, 1, 3).contiguous().float()  # [nb, nh, dv, dk]
    if outlier_rows or outlier_cols:
        scale_r = np.ones((len(bs), len(hs), d_v), np.float32)
        scale_c = np.ones((len(bs), len(hs), d_k), np.float32)
        for ib, b in enumerate(bs):
            for ih, h in enumerate(hs):
                if outlier_rows:
                    scale_r[ib, ih, _pick(seed, TID_OUT_ROWS, int(b), int(h), d_v, outlier_rows)] = outlier_scale
                if outlier_cols:
                    scale_c[ib, ih, _pick(seed, TID_OUT_COLS, int(b), int(h), d_k, outlier_cols)] = outlier_scale
        S *= torch.from_numpy(scale_r).to(device)[..., :, None]
        S *= torch.from_numpy(scale_c).to(device)[..., None, :]
    return S
