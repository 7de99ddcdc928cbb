"""Helpers for the GPU parity tests: inputs, oracle runs and comparisons.

Parity is checked window by window and anchored on the ORACLE: for each
window both sides start from the oracle's snapshot (uploaded to the device
with lq_state_restore), decode the window's tokens from the same seeded
inputs, and commit.  Outputs, buffered records and the next snapshot are then
compared.  Anchoring keeps two free-running chains from drifting apart after a
legitimate +-1 LSB code flip; no value produced by the CUDA path is ever fed
to the oracle.

Tolerances (ours, from the arithmetic):
  outputs   l2-relative per output vector <= 1e-3 (FP32 io), 2e-2 (BF16 io)
  codes     within +-1 LSB (a BF16 residual: one BF16 step plus 1e-5 of its
            row's largest magnitude, the FP32 rebuild's absolute error)
  scales, smoothing, compensators   within 1e-5 relative (compensators
            relative to the largest magnitude of their row)
  compensator rows  equal, except near-ties (norms within 1e-5 relative of
            the r-th largest), where the reconstructions are compared instead.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import linear_attention_recurrent_int8_b200 as lq
from linear_attention_recurrent_int8_b200 import synth

OUT_TOL = {"fp32": 1e-3, "bf16": 2e-2}
SCALE_RTOL = 1e-5
NEAR_TIE = 1e-5


def io_dtype(io):
    return torch.bfloat16 if io == "bf16" else torch.float32


def make_config(wl: synth.DecodeWorkload, **over) -> lq.Config:
    c = lq.Config(batch=wl.batch, heads=wl.heads, d_k=wl.d_k, d_v=wl.d_v, window=wl.window,
                  n_comp=wl.n_comp, gate=lq.LQ_GATE_DIAG if wl.gate == "diag" else lq.LQ_GATE_SCALAR,
                  io_dtype=lq.LQ_BF16 if wl.io == "bf16" else lq.LQ_F32,
                  smoothing=int(wl.smoothing), auto_commit=1, delta=wl.delta)
    for k, v in over.items():
        setattr(c, k, v)
    return c


def heads_major(x):
    """[B, T, H, ...] -> [B*H, T, ...]"""
    x = np.asarray(x)
    B, T, H = x.shape[:3]
    return np.ascontiguousarray(np.swapaxes(x, 1, 2).reshape((B * H, T) + x.shape[3:]))


def oracle_tokens(tok: dict, gate: str, delta: int = 1):
    """Oracle-side (d, k~, b, v, q) [nh, n, ...] from synth.tokens output."""
    q, k, v = heads_major(tok["q"]), heads_major(tok["k"]), heads_major(tok["v"])
    alpha, beta = heads_major(tok["alpha"]), heads_major(tok["beta"])
    if not delta:
        d, kt, b = oracle.gated_linear_instance(alpha, beta, k, gate == "diag")
    elif gate == "diag":
        d, kt, b = oracle.kda_instance(alpha, beta, k)
    else:
        d, kt, b = oracle.gdn_instance(alpha, beta, k)
    return d, kt, b, v, q


def to_device_tokens(tok: dict, io: str, device="cuda"):
    dt = io_dtype(io)
    out = {}
    for key in ("q", "k", "v"):
        out[key] = torch.from_numpy(np.ascontiguousarray(tok[key])).to(device=device, dtype=dt)
    for key in ("alpha", "beta"):
        out[key] = torch.from_numpy(np.ascontiguousarray(tok[key])).to(device=device,
                                                                       dtype=torch.float32)
    return out


def pack_codes4(codes) -> np.ndarray:
    """int8 codes [..., d_k] with |Q| <= 7 -> bytes [..., d_k / 2] in the
    4-bit storage format that lq.h states for lq_snapshot.codes: in each group
    of 8 key channels 8g..8g+7, byte 4g+b holds channel 8g+b in its low nibble
    and 8g+4+b in its high nibble, two's complement."""
    c = np.asarray(codes).astype(np.int16)
    g = c.reshape(c.shape[:-1] + (-1, 2, 4))  # [..., group, half, b]
    lo, hi = g[..., 0, :] & 0xF, g[..., 1, :] & 0xF
    return (lo | (hi << 4)).astype(np.uint8).reshape(c.shape[:-1] + (-1,))


def unpack_codes4(packed) -> np.ndarray:
    """Inverse of pack_codes4: bytes [..., d_k / 2] -> int8 codes [..., d_k]."""
    p = np.asarray(packed).astype(np.uint8)
    g = p.reshape(p.shape[:-1] + (-1, 4)).astype(np.int16)  # [..., group, b]
    nib = np.stack([g & 0xF, g >> 4], axis=-2)             # [..., group, half, b]
    nib = np.where(nib >= 8, nib - 16, nib)
    return nib.reshape(p.shape[:-1] + (-1,)).astype(np.int8)


def codes_to_device_format(cfg: lq.Config, codes) -> np.ndarray:
    return pack_codes4(codes) if cfg.bits == 4 else np.asarray(codes, np.int8)


def codes_from_device_format(cfg: lq.Config, codes) -> np.ndarray:
    return unpack_codes4(codes) if cfg.bits == 4 else np.asarray(codes)


def residual_to_device(cfg: lq.Config, snap: dict, device="cuda") -> torch.Tensor:
    """The snapshot's residual in the device format: codes, packed codes, or
    the BF16 values (exact: the oracle's dense residual is BF16-valued)."""
    if cfg.bits == 16:
        return torch.from_numpy(np.ascontiguousarray(snap["dense"])).to(device).to(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(codes_to_device_format(cfg, snap["codes"]))).to(device)


def upload_snapshot(cfg: lq.Config, snap: dict, device="cuda") -> lq.Snapshot:
    t = dict(codes=residual_to_device(cfg, snap, device),
             row_scale=torch.from_numpy(np.ascontiguousarray(snap["row_scale"])).to(device),
             col_smooth=torch.from_numpy(np.ascontiguousarray(snap["col_smooth"])).to(device),
             comp_row=torch.from_numpy(np.ascontiguousarray(snap["comp_row"], np.int32)).to(device),
             comp_val=torch.from_numpy(np.ascontiguousarray(snap["comp_val"])).to(device))
    return lq.Snapshot(cfg, device, t)


def snapshot_to_host(cfg: lq.Config, snap: lq.Snapshot) -> dict:
    """A device snapshot as numpy arrays, codes one int8 per code (a BF16
    residual as ``dense`` float32 with zero codes, the oracle's form)."""
    out = {k: v.detach().cpu().float().numpy() if v.dtype == torch.bfloat16 else v.detach().cpu().numpy()
           for k, v in snap.t.items()}
    if cfg.bits == 16:
        out["dense"] = out["codes"].astype(np.float32)
        out["codes"] = np.zeros(out["dense"].shape, np.int8)
    else:
        out["codes"] = codes_from_device_format(cfg, out["codes"])
    return out


def download_snapshot(st: lq.State) -> dict:
    return snapshot_to_host(st.cfg, st.snap)


def rel_l2(a, b, axis=-1):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    num = np.linalg.norm(a - b, axis=axis)
    den = np.maximum(np.linalg.norm(b, axis=axis), 1e-30)
    return num / den


def compare_outputs(o_gpu, o_ref, io, what="outputs"):
    r = rel_l2(o_gpu, o_ref)
    worst = float(r.max()) if r.size else 0.0
    assert worst <= OUT_TOL[io], f"{what}: worst l2-relative error {worst:.3e} > {OUT_TOL[io]}"
    return worst


def compare_snapshots(gpu: dict, ref: dict, ref_norms=None, heads=None, exact_codes=False):
    """Compares a device snapshot with the oracle's, head by head.

    Returns a dict of statistics.  ``ref_norms`` [nh, dv] (oracle row norms
    of the state that was quantized) enables the near-tie rule."""
    nh = ref["codes"].shape[0]
    heads = range(nh) if heads is None else heads
    stats = dict(code_flips=0, near_ties=0, heads=0)
    for h in heads:
        stats["heads"] += 1
        rc_g = [int(x) for x in gpu["comp_row"][h]]
        rc_r = [int(x) for x in ref["comp_row"][h]]
        if rc_g != rc_r:
            # several results correct: rows whose norms tie (within 1e-5) with the r-th largest
            assert ref_norms is not None, f"head {h}: compensator rows {rc_g} != {rc_r}"
            norms = ref_norms[h]
            r = len(rc_r)
            kth = np.sort(norms)[::-1][r - 1]
            for row in set(rc_g) ^ set(rc_r):
                assert abs(norms[row] - kth) <= NEAR_TIE * kth, \
                    f"head {h}: compensator rows {rc_g} != {rc_r} and row {row} is not a near-tie"
            stats["near_ties"] += 1
            sg = oracle.dequantize({k: v[h:h + 1] for k, v in gpu.items()})[0]
            sr = oracle.dequantize({k: v[h:h + 1] for k, v in ref.items()})[0]
            step = (ref["row_scale"][h][:, None].astype(np.float64) * ref["col_smooth"][h][None, :]
                    + gpu["row_scale"][h][:, None] * gpu["col_smooth"][h][None, :])
            assert np.all(np.abs(sg - sr) <= 1.5 * step + 1e-6 * np.abs(sr).max()), \
                f"head {h}: reconstructions differ beyond one code step"
            continue
        np.testing.assert_allclose(gpu["row_scale"][h], ref["row_scale"][h], rtol=SCALE_RTOL,
                                   atol=0, err_msg=f"row_scale head {h}")
        np.testing.assert_allclose(gpu["col_smooth"][h], ref["col_smooth"][h], rtol=SCALE_RTOL,
                                   atol=0, err_msg=f"col_smooth head {h}")
        if len(rc_r):
            cv_g = gpu["comp_val"][h].astype(np.float64)
            cv_r = ref["comp_val"][h].astype(np.float64)
            scale = np.abs(cv_r).max(axis=1, keepdims=True)
            assert np.all(np.abs(cv_g - cv_r) <= SCALE_RTOL * scale), f"comp_val head {h}"
        if "dense" in ref:
            # BF16 residual: one BF16 step (2^-7 of the larger magnitude) plus
            # the FP32 rebuild's error, which is absolute -- relative to the
            # row's magnitude, the same 1e-5 as for the scales -- and which a
            # floating format does not absorb near zero the way a code step
            # relative to the row maximum does
            g = gpu["dense"][h].astype(np.float64)
            r_ = ref["dense"][h].astype(np.float64)
            dd = np.abs(g - r_)
            if exact_codes:
                assert dd.max() == 0, f"BF16 residual differs in head {h}"
            rowmax = np.maximum(np.abs(g).max(axis=1, keepdims=True), np.abs(r_).max(axis=1, keepdims=True))
            assert np.all(dd <= 2.0 ** -7 * np.maximum(np.abs(g), np.abs(r_)) + SCALE_RTOL * rowmax), \
                f"BF16 residual differs by more than one step in head {h}"
            stats["code_flips"] += int((dd > 0).sum())
            continue
        d = np.abs(gpu["codes"][h].astype(np.int32) - ref["codes"][h].astype(np.int32))
        if exact_codes:
            assert d.max() == 0, f"codes differ in head {h}"
        assert d.max() <= 1, f"codes differ by {d.max()} LSB in head {h}"
        stats["code_flips"] += int((d > 0).sum())
    return stats


class AnchoredRun:
    """Runs a workload on the device window by window, anchored on the
    oracle, and checks every window."""

    def __init__(self, wl: synth.DecodeWorkload, cfg: lq.Config | None = None,
                 steps_per_call: int = 1, commit_mode: str = "auto", device="cuda"):
        self.wl = wl
        self.cfg = cfg or make_config(wl)
        if commit_mode != "auto":
            self.cfg.auto_commit = 0
        self.steps_per_call = steps_per_call
        self.commit_mode = commit_mode  # "auto" | "explicit"
        self.device = device
        self.st = lq.State(self.cfg, device)
        self.bs = np.arange(wl.batch)
        self.hs = np.arange(wl.heads)
        self.stats = dict(windows=0, worst_out=0.0, code_flips=0, near_ties=0)

    def init(self):
        wl, cfg = self.wl, self.cfg
        S0 = synth.initial_state(wl.seed, self.bs, self.hs, wl.d_k, wl.d_v, wl.outlier_rows,
                                 wl.outlier_cols, wl.outlier_scale)
        S0 = S0.reshape(wl.nh, wl.d_v, wl.d_k)
        lq.lq_state_init(self.st, torch.from_numpy(S0).to(self.device))
        torch.cuda.synchronize()
        ref = oracle.quantize(S0, cfg.n_comp, bool(cfg.smoothing), cfg.bits)
        st = compare_snapshots(download_snapshot(self.st), ref, ref["row_norm"], exact_codes=True)
        self.stats["near_ties"] += st["near_ties"]
        self.snap = ref
        return ref

    def window(self, w: int, ntok: int | None = None):
        """Runs window w (tokens w*W .. w*W+ntok-1) from the oracle's snapshot."""
        wl, cfg = self.wl, self.cfg
        W = cfg.window
        ntok = W if ntok is None else ntok
        t0 = w * W
        lq.lq_state_restore(self.st, upload_snapshot(cfg, self.snap, self.device))
        tok = synth.tokens(wl.seed, self.bs, self.hs, t0, t0 + ntok, wl.d_k, wl.d_v, wl.gate, wl.io)
        dev = to_device_tokens(tok, wl.io, self.device)
        o = torch.empty((wl.batch, ntok, wl.heads, wl.d_v), dtype=io_dtype(wl.io), device=self.device)
        s = 0
        while s < ntok:
            n = min(self.steps_per_call, ntok - s)
            sl = slice(s, s + n)
            args = [dev[key][:, sl].contiguous() for key in ("q", "k", "v", "alpha", "beta")]
            out = torch.empty((wl.batch, n, wl.heads, wl.d_v), dtype=io_dtype(wl.io),
                              device=self.device)
            lq.lq_decode_window(self.st, *args, n, out)
            o[:, sl] = out
            s += n
        if self.commit_mode == "explicit" or ntok < W:
            lq.lq_window_commit(self.st)
        torch.cuda.synchronize()
        assert self.st.pos == 0

        d, kt, b, v, q = oracle_tokens(tok, wl.gate, wl.delta)
        rec = oracle.empty_records(wl.nh, W, wl.d_k, wl.d_v, cfg.gdim)
        o_ref = oracle.window(self.snap, rec, 0, d, kt, b, v, q)
        new_snap, S_n = oracle.commit(self.snap, rec, ntok, cfg.n_comp, bool(cfg.smoothing), cfg.bits)

        o_gpu = heads_major(o.float().cpu().numpy())
        worst = compare_outputs(o_gpu, o_ref, wl.io, f"outputs window {w}")
        # buffered records (FP32) against the oracle's
        bk = self.st.buf_k.cpu().numpy()[:, :ntok]
        bu = self.st.buf_u.cpu().numpy()[:, :ntok]
        bL = self.st.buf_gate.cpu().numpy()[:, :ntok]
        assert rel_l2(bk, rec["k"][:, :ntok]).max() < 1e-6, "buffered k~ differ"
        assert rel_l2(bu, rec["u"][:, :ntok]).max() < 1e-3, "buffered u differ"
        np.testing.assert_allclose(bL, rec["L"][:, :ntok], rtol=1e-5, atol=1e-5)
        st = compare_snapshots(download_snapshot(self.st), new_snap, new_snap["row_norm"])
        self.stats["windows"] += 1
        self.stats["worst_out"] = max(self.stats["worst_out"], worst)
        self.stats["code_flips"] += st["code_flips"]
        self.stats["near_ties"] += st["near_ties"]
        self.snap = new_snap
        return o_gpu, o_ref


class SampledRun:
    """Full-size run on the device (every sequence and head, the launch
    configuration the benchmark times) with the oracle following a seeded
    sample of (sequence, head) pairs.

    Device inputs for all heads are drawn on the device with the same integer
    streams; the sampled heads' inputs (and initial states) are overwritten
    with the numpy draws that the oracle consumes, so both sides see identical
    values there.  At each window start the sampled heads' snapshots are set
    to the oracle's (anchoring); the other heads run free and are not checked
    (every head is checked by AnchoredRun in the first windows).  Nothing the
    device computes is given to the oracle."""

    def __init__(self, wl: synth.DecodeWorkload, n_sample: int, seed: int = 1234, device="cuda",
                 bits: int = 8):
        self.wl, self.device = wl, device
        self.cfg = make_config(wl, bits=bits)
        self.st = lq.State(self.cfg, device)
        rng = np.random.default_rng(seed)
        self.sample = np.sort(rng.choice(wl.nh, size=min(n_sample, wl.nh), replace=False))
        self.sb, self.sh = self.sample // wl.heads, self.sample % wl.heads
        self.idx = torch.from_numpy(self.sample).to(device)
        self.stats = dict(windows=0, worst_out=0.0, code_flips=0, near_ties=0)

    def _sample_tokens(self, t0, t1):
        wl = self.wl
        per = [synth.tokens(wl.seed, [b], [h], t0, t1, wl.d_k, wl.d_v, wl.gate, wl.io)
               for b, h in zip(self.sb, self.sh)]
        return {k: np.concatenate([p[k] for p in per], axis=2) for k in per[0]}  # [1, T, ns, ...]

    def _sampled_snapshot(self):
        sub = lq.Snapshot(self.cfg, self.device,
                          {k: v.index_select(0, self.idx) for k, v in self.st.snap.t.items()})
        return snapshot_to_host(self.cfg, sub)

    def init(self):
        wl, dev = self.wl, self.device
        S = synth.torch_initial_state(wl.seed, np.arange(wl.batch), np.arange(wl.heads), wl.d_k, wl.d_v,
                                      wl.outlier_rows, wl.outlier_cols, wl.outlier_scale, dev)
        S = S.reshape(wl.nh, wl.d_v, wl.d_k)
        S_s = np.concatenate([synth.initial_state(wl.seed, [b], [h], wl.d_k, wl.d_v, wl.outlier_rows,
                                                  wl.outlier_cols, wl.outlier_scale)[0]
                              for b, h in zip(self.sb, self.sh)], axis=0)
        S[self.idx] = torch.from_numpy(S_s).to(dev)
        lq.lq_state_init(self.st, S)
        torch.cuda.synchronize()
        del S
        ref = oracle.quantize(S_s, self.cfg.n_comp, bool(self.cfg.smoothing), self.cfg.bits)
        compare_snapshots(self._sampled_snapshot(), ref, ref["row_norm"], exact_codes=True)
        self.snap = ref

    def _anchor(self):
        for key in ("codes", "row_scale", "col_smooth", "comp_row", "comp_val"):
            if self.st.snap.t[key].numel():
                if key == "codes":
                    src = residual_to_device(self.cfg, self.snap, self.device)
                else:
                    src = torch.from_numpy(np.ascontiguousarray(self.snap[key])).to(self.device)
                self.st.snap.t[key][self.idx] = src.to(self.st.snap.t[key].dtype)

    def window(self, w: int):
        wl, cfg, dev = self.wl, self.cfg, self.device
        W = cfg.window
        t0 = w * W
        self._anchor()
        dev_tok = synth.torch_tokens(wl.seed, wl.batch, wl.heads, t0, t0 + W, wl.d_k, wl.d_v, wl.gate,
                                     wl.io, dev)
        tok_s = self._sample_tokens(t0, t0 + W)
        bi = torch.from_numpy(self.sb).to(dev)
        hi = torch.from_numpy(self.sh).to(dev)
        for k in ("q", "k", "v", "alpha", "beta"):
            vals = torch.from_numpy(np.ascontiguousarray(np.swapaxes(tok_s[k][0], 0, 1))).to(dev)
            dev_tok[k][bi, :, hi] = vals.to(dev_tok[k].dtype)
        o = torch.empty((wl.batch, W, wl.heads, wl.d_v), dtype=io_dtype(wl.io), device=dev)
        out = torch.empty((wl.batch, 1, wl.heads, wl.d_v), dtype=io_dtype(wl.io), device=dev)
        for t in range(W):
            args = [dev_tok[k][:, t:t + 1].contiguous() for k in ("q", "k", "v", "alpha", "beta")]
            lq.lq_decode_window(self.st, *args, 1, out)
            o[:, t:t + 1] = out
        torch.cuda.synchronize()
        assert self.st.pos == 0
        d, kt, b, v, q = oracle_tokens(tok_s, wl.gate, wl.delta)
        rec = oracle.empty_records(len(self.sample), W, wl.d_k, wl.d_v, cfg.gdim)
        o_ref = oracle.window(self.snap, rec, 0, d, kt, b, v, q)
        new_snap, _ = oracle.commit(self.snap, rec, W, cfg.n_comp, bool(cfg.smoothing), cfg.bits)
        o_gpu = o[bi, :, hi].float().cpu().numpy()  # [ns, W, dv]
        worst = compare_outputs(o_gpu, o_ref, wl.io, f"outputs window {w}")
        st = compare_snapshots(self._sampled_snapshot(), new_snap, new_snap["row_norm"])
        self.stats["windows"] += 1
        self.stats["worst_out"] = max(self.stats["worst_out"], worst)
        self.stats["code_flips"] += st["code_flips"]
        self.stats["near_ties"] += st["near_ties"]
        self.snap = new_snap
