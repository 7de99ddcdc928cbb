"""CPU oracle for int8 per-window recurrent-state decode (LeapQuant).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` import this
package.  It shares no code with the CUDA library and the library never calls
it.

The arithmetic lives in ``lq_oracle.c`` (plain C, FP64, OpenMP over heads);
this module only marshals numpy arrays and holds the mapping from a model's
gate parameters to the (D_t, k~_t, b_t) of equation 1, which is the
arithmetic of one Table 4 row each:

* "LeapQuant: Efficient Linear Attention with Accurate Recurrent State
  Quantization", Appendix, Table 4: Gated DeltaNet is D_t = alpha_t I,
  k~_t = beta_t k_t, b_t = alpha_t k_t.
* Kimi Delta Attention (named in the same page's Abstract, no Table 4 row in
  the text): D_t = Diag(alpha_t), k~_t = beta_t k_t, b_t = alpha_t * k_t, the
  diagonal-gate analogue, whose record size 2 d_k + d_v matches the GLA row.

Layouts are head-major: a state is ``[nh, d_v, d_k]``, a token tensor is
``[nh, n, d]``.  Every function accepts any array-like and returns float64
(or the stored formats int8 / float32 / int32 for snapshots).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lq_oracle.c")
_LIB = os.path.join(_HERE, "liblq_oracle.so")
_lock = threading.Lock()
_lib = None


def compile_oracle(force: bool = False) -> str:
    """Compiles ``lq_oracle.c`` into ``liblq_oracle.so`` (gcc, -O2, strict IEEE)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-Wall", "-Wextra", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            # LQ_ORACLE_LIB lets the mutation meta-test load a deliberately
            # broken build of this oracle to show that the pins catch it.
            path = os.environ.get("LQ_ORACLE_LIB") or compile_oracle()
            lib = ctypes.CDLL(path)
            P = ctypes.c_void_p
            I = ctypes.c_int
            lib.lqo_eq1_steps.argtypes = [I, I, I, I, P, P, P, P, P, P, P]
            lib.lqo_quantize.argtypes = [I, I, I, I, I, I, P, P, P, P, P, P, P, P]
            lib.lqo_dequantize.argtypes = [I, I, I, I, P, P, P, P, P, P, P, P]
            lib.lqo_window.argtypes = [I] * 9 + [P] * 16
            lib.lqo_rebuild.argtypes = [I] * 7 + [P] * 11
            for f in (lib.lqo_eq1_steps, lib.lqo_quantize, lib.lqo_dequantize,
                      lib.lqo_window, lib.lqo_rebuild):
                f.restype = None
            _lib = lib
    return _lib


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


# --------------------------------------------------------------------------
# Table 4 instances (the gate parameters of a model -> D_t, k~_t, b_t).
# --------------------------------------------------------------------------

def gdn_instance(alpha, beta, k):
    """Gated DeltaNet row of Table 4: D = alpha I, k~ = beta k, b = alpha k.

    alpha, beta: [nh, n]; k: [nh, n, d_k].  Returns d [nh, n, 1], k~, b."""
    alpha = np.asarray(alpha, np.float64)
    beta = np.asarray(beta, np.float64)
    k = np.asarray(k, np.float64)
    return alpha[..., None], beta[..., None] * k, alpha[..., None] * k


def kda_instance(alpha, beta, k):
    """Diagonal (per key channel) gate: D = Diag(alpha), k~ = beta k, b = alpha * k.

    alpha: [nh, n, d_k]; beta: [nh, n]; k: [nh, n, d_k]."""
    alpha = np.asarray(alpha, np.float64)
    beta = np.asarray(beta, np.float64)
    k = np.asarray(k, np.float64)
    return alpha, beta[..., None] * k, alpha * k


def gated_linear_instance(alpha, beta, k, diagonal: bool):
    """The b = 0 rows of Table 4 (linear attention with D = I, RetNet with a
    constant decay, Mamba2 with a per-token scalar decay, GLA with a per-channel
    decay): D = alpha I or Diag(alpha), k~ = beta k (those rows print k~ = k,
    i.e. beta = 1), b = 0, so u_t = v_t.

    alpha: [nh, n] (scalar) or [nh, n, d_k] (diagonal); beta: [nh, n]; k: [nh, n, d_k]."""
    alpha = np.asarray(alpha, np.float64)
    beta = np.asarray(beta, np.float64)
    k = np.asarray(k, np.float64)
    d = alpha if diagonal else alpha[..., None]
    return d, beta[..., None] * k, np.zeros_like(k)


def deltaproduct_instance(alpha, beta, k, v):
    """DeltaProduct ([LQ] Table 4 caption: n delta-rule sub-steps per token,
    each an instance of equation 1) as micro-tokens in sub-step order: the
    token's gate alpha acts once, at its first sub-step (the Gated DeltaNet
    row: D = alpha I, k~ = beta_1 k_1, b = alpha k_1), the other sub-steps are
    DeltaNet rows (D = I, k~ = beta_j k_j, b = k_j).  The token's output is
    the output of its last sub-step.

    alpha [nh, T]; beta [nh, T, n]; k [nh, T, n, dk]; v [nh, T, n, dv].
    Returns d [nh, T n, 1], k~ [nh, T n, dk], b [nh, T n, dk], v [nh, T n, dv]."""
    alpha = np.asarray(alpha, np.float64)
    beta = np.asarray(beta, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    nh, T, n, dk = k.shape
    g = np.ones((nh, T, n))
    g[:, :, 0] = alpha
    d = g.reshape(nh, T * n, 1)
    kt = (beta[..., None] * k).reshape(nh, T * n, dk)
    b = (g[..., None] * k).reshape(nh, T * n, dk)
    return d, kt, b, v.reshape(nh, T * n, -1)


# --------------------------------------------------------------------------
# Equation 1, explicit stepping.
# --------------------------------------------------------------------------

def eq1_steps(S0, d, kt, b, v, q=None):
    """n steps of S_t = S_{t-1} Diag(d_t) + (v_t - S_{t-1} b_t) k~_t^T, o_t = S_t q_t.

    S0 [nh, dv, dk]; d [nh, n, 1 or dk]; kt, b, q [nh, n, dk]; v [nh, n, dv].
    Returns (o [nh, n, dv] or None, S_n [nh, dv, dk]) in FP64."""
    S = _c(S0, np.float64).copy()
    nh, dv, dk = S.shape
    kt = _c(kt, np.float64)
    n = kt.shape[1]
    d = _c(np.broadcast_to(np.asarray(d, np.float64), (nh, n, dk)), np.float64)
    b = _c(b, np.float64)
    v = _c(v, np.float64)
    qq = None if q is None else _c(q, np.float64)
    o = None if q is None else np.zeros((nh, n, dv), np.float64)
    _load().lqo_eq1_steps(nh, dv, dk, n, _p(S), _p(d), _p(kt), _p(b), _p(v), _p(qq), _p(o))
    return o, S


# --------------------------------------------------------------------------
# Snapshot: quantize / dequantize.
# --------------------------------------------------------------------------

class Snapshot(dict):
    """codes int8 [nh,dv,dk], row_scale f32 [nh,dv], col_smooth f32 [nh,dk],
    comp_row i32 [nh,r], comp_val f32 [nh,r,dk] (+ row_norm f64 [nh,dv] when
    produced by quantize); a BF16 state (bits = 16) also holds dense f32
    [nh,dv,dk], the BF16-rounded residual, which replaces codes x scales;
    the rank-r SVD compensator rule also holds comp_u f32 [nh,r,dv]: the
    compensators are then the rank-one terms comp_u[c] comp_val[c]^T instead
    of the rows comp_row[c] = comp_val[c]."""

    @property
    def n_comp(self):
        return self["comp_row"].shape[1]


BITS = (8, 6, 4, 16)  # code widths: q_max = 2^(bits-1) - 1 = 127, 31, 7; 16 = BF16 state


def svd_compensators(S, r: int):
    """The rank-r SVD compensator rule (the scope table's variant of the
    row rule): for each head the r largest singular triplets of the FP32
    state (an FP64 SVD), u_c = s_c U_c and k~_c = V_c, the sign chosen so that
    the largest-magnitude entry of k~_c is positive, both rounded to FP32.
    Returns (u [nh, r, dv], k~ [nh, r, dk], singular values [nh, min(dv, dk)])."""
    S = _c(S, np.float32)
    nh, dv, dk = S.shape
    cu = np.zeros((nh, r, dv), np.float32)
    ck = np.zeros((nh, r, dk), np.float32)
    sv_all = np.zeros((nh, min(dv, dk)))
    for h in range(nh):
        U, sv, Vt = np.linalg.svd(S[h].astype(np.float64))
        sv_all[h] = sv
        for c in range(r):
            u, v = U[:, c] * sv[c], Vt[c]
            if v[np.argmax(np.abs(v))] < 0:
                u, v = -u, -v
            cu[h, c], ck[h, c] = u, v
    return cu, ck, sv_all


def quantize(S, n_comp: int, smoothing: bool = True, bits: int = 8, rule: str = "rows") -> Snapshot:
    """Compensator selection, residual smoothing and per-row codes of an FP32
    state ``S`` [nh, dv, dk] (rounded to FP32 first if it is not); the codes
    are ``bits`` wide (8, or the 6- and 4-bit widths of the lower-precision
    groups of [LQ] Table 1) and returned one per int8.  ``bits = 16`` is the
    BF16 state of [LQ] Table 2: compensators as above, the residual rounded
    to BF16 into ``dense`` (no smoothing, unit scales, zero codes).
    ``rule = "svd"`` takes the compensators by :func:`svd_compensators` and
    quantizes the residual S - sum_c u_c k~_c^T (rounded to FP32) with the
    same C3-C4."""
    S = _c(S, np.float32)
    nh, dv, dk = S.shape
    assert 0 <= n_comp <= dv
    assert bits in BITS and rule in ("rows", "svd")
    if rule == "svd":
        cu, ck, sv = svd_compensators(S, n_comp)
        R = S.astype(np.float64) - np.einsum("hci,hcj->hij", cu.astype(np.float64), ck.astype(np.float64))
        out = quantize(R.astype(np.float32), 0, smoothing, bits)
        out["comp_row"] = np.zeros((nh, n_comp), np.int32)
        out["comp_val"] = ck
        out["comp_u"] = cu
        out["singular_values"] = sv
        return out
    out = Snapshot(
        codes=np.zeros((nh, dv, dk), np.int8),
        row_scale=np.zeros((nh, dv), np.float32),
        col_smooth=np.zeros((nh, dk), np.float32),
        comp_row=np.zeros((nh, n_comp), np.int32),
        comp_val=np.zeros((nh, n_comp, dk), np.float32),
        row_norm=np.zeros((nh, dv), np.float64),
    )
    if bits == 16:
        out["dense"] = np.zeros((nh, dv, dk), np.float32)
    _load().lqo_quantize(nh, dv, dk, n_comp, int(bool(smoothing)), int(bits), _p(S), _p(out["codes"]),
                         _p(out["row_scale"]), _p(out["col_smooth"]), _p(out["comp_row"]),
                         _p(out["comp_val"]), _p(out["row_norm"]), _p(out.get("dense")))
    return out


def _snap_arrays(snap):
    codes = _c(snap["codes"], np.int8)
    nh, dv, dk = codes.shape
    comp_row = _c(snap["comp_row"], np.int32).reshape(nh, -1)
    r = comp_row.shape[1]
    dense = snap.get("dense")
    dense = None if dense is None else _c(dense, np.float32)
    cu = snap.get("comp_u")
    cu = None if cu is None else _c(cu, np.float32).reshape(nh, r, dv)
    return (codes, _c(snap["row_scale"], np.float32), _c(snap["col_smooth"], np.float32),
            comp_row, _c(snap["comp_val"], np.float32).reshape(nh, r, dk), dense, cu, nh, dv, dk, r)


def dequantize(snap) -> np.ndarray:
    """S^_0 = Diag(sigma) Q Diag(c) (or the BF16 residual) + compensator rows,
    FP64 [nh, dv, dk]."""
    codes, rs, cs, cr, cv, dn, cu, nh, dv, dk, r = _snap_arrays(snap)
    out = np.zeros((nh, dv, dk), np.float64)
    _load().lqo_dequantize(nh, dv, dk, r, _p(codes), _p(rs), _p(cs), _p(cr), _p(cv), _p(dn), _p(cu),
                           _p(out))
    return out


# --------------------------------------------------------------------------
# Per-window decode (buffered form), rebuild and commit.
# --------------------------------------------------------------------------

class Records(dict):
    """Window buffer: L [nh, W, gdim] (cumulative log gate), k [nh, W, dk]
    (k~), u [nh, W, dv]; positions 1..pos are filled.  FP64 arrays holding
    FP32 values (unless produced with exact=True)."""


def empty_records(nh: int, W: int, dk: int, dv: int, gdim: int) -> Records:
    return Records(L=np.zeros((nh, W, gdim)), k=np.zeros((nh, W, dk)), u=np.zeros((nh, W, dv)))


def window(snap, records: Records, pos: int, d, kt, b, v, q, exact: bool = False):
    """Decode n tokens at window positions pos+1..pos+n from the fixed
    boundary snapshot and the buffered records (updated in place).

    d [nh, n, gdim] (gdim 1 = scalar gate, d_k = diagonal gate); kt, b, q
    [nh, n, dk]; v [nh, n, dv].  Returns o [nh, n, dv] (FP64)."""
    codes, rs, cs, cr, cv, dn, cu, nh, dv, dk, r = _snap_arrays(snap)
    W = records["k"].shape[1]
    gdim = records["L"].shape[2]
    d = _c(d, np.float64)
    n = d.shape[1]
    assert d.shape == (nh, n, gdim)
    assert 0 <= pos and pos + n <= W
    for key in ("L", "k", "u"):
        records[key] = _c(records[key], np.float64)
    kt, b, v, q = (_c(a, np.float64) for a in (kt, b, v, q))
    o = np.zeros((nh, n, dv), np.float64)
    _load().lqo_window(nh, dv, dk, r, gdim, W, pos, n, int(bool(exact)), _p(codes), _p(rs), _p(cs),
                       _p(cr), _p(cv), _p(dn), _p(cu), _p(records["L"]), _p(records["k"]), _p(records["u"]),
                       _p(d), _p(kt), _p(b), _p(v), _p(q), _p(o))
    return o


def rebuild(snap, records: Records, n: int) -> np.ndarray:
    """S_n = S^_0 D_{1..n} + sum_{m<=n} u_m (D_{m+1..n} k~_m)^T, FP64 [nh, dv, dk]."""
    codes, rs, cs, cr, cv, dn, cu, nh, dv, dk, r = _snap_arrays(snap)
    W = records["k"].shape[1]
    gdim = records["L"].shape[2]
    assert 0 <= n <= W
    L, K, U = (_c(records[key], np.float64) for key in ("L", "k", "u"))
    out = np.zeros((nh, dv, dk), np.float64)
    _load().lqo_rebuild(nh, dv, dk, r, gdim, W, n, _p(codes), _p(rs), _p(cs), _p(cr), _p(cv),
                        _p(dn), _p(cu), _p(L), _p(K), _p(U), _p(out))
    return out


def commit(snap, records: Records, n: int, n_comp: int, smoothing: bool = True, bits: int = 8,
           rule: str = "rows"):
    """Window commit: rebuild S_n (kept as an FP32 state), then quantize.

    Returns (new snapshot, S_n as float32)."""
    S = rebuild(snap, records, n).astype(np.float32)
    return quantize(S, n_comp, smoothing, bits, rule), S


def decode_run(snap, d, kt, b, v, q, W: int, n_comp: int, smoothing: bool = True,
               on_commit=None, bits: int = 8):
    """Free-running per-window decode of T tokens: windows of W tokens, each
    committed at its end (the last, possibly short, window too).

    ``on_commit(window_index, snapshot)`` is called after each commit.
    Returns (o [nh, T, dv], final snapshot)."""
    nh, T = np.asarray(kt).shape[:2]
    dv = np.asarray(v).shape[2]
    dk = np.asarray(kt).shape[2]
    gdim = np.asarray(d).shape[2]
    o = np.zeros((nh, T, dv))
    widx = 0
    for t0 in range(0, T, W):
        t1 = min(T, t0 + W)
        rec = empty_records(nh, W, dk, dv, gdim)
        sl = slice(t0, t1)
        o[:, sl] = window(snap, rec, 0, d[:, sl], kt[:, sl], b[:, sl], v[:, sl], q[:, sl])
        snap, _ = commit(snap, rec, t1 - t0, n_comp, smoothing, bits)
        if on_commit is not None:
            on_commit(widx, snap)
        widx += 1
    return o, snap


def prefill(S0, d, kt, b, v, q, snapshot_every: int, n_comp: int, smoothing: bool = True,
            bits: int = 8):
    """Prefill by the token recurrence (equation 1, FP64 state) with a
    quantized snapshot of the state, rounded to FP32, after every
    ``snapshot_every`` tokens (one state per that many cached tokens).

    Returns (o [nh, T, dv], list of snapshots, final FP64 state)."""
    S = _c(S0, np.float64)
    nh, T = np.asarray(kt).shape[:2]
    dv = S.shape[1]
    o = np.zeros((nh, T, dv))
    snaps = []
    for t0 in range(0, T, snapshot_every):
        t1 = min(T, t0 + snapshot_every)
        sl = slice(t0, t1)
        o[:, sl], S = eq1_steps(S, d[:, sl], kt[:, sl], b[:, sl], v[:, sl], q[:, sl])
        if t1 - t0 == snapshot_every:
            snaps.append(quantize(S.astype(np.float32), n_comp, smoothing, bits))
    return o, snaps, S
