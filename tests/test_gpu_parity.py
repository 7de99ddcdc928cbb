"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Every window is anchored on the oracle (see lqtest.py): both sides start from
the oracle's snapshot, decode the same seeded tokens and commit; outputs,
records and the committed snapshot are compared with the stated tolerances.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import linear_attention_recurrent_int8_b200 as lq
from linear_attention_recurrent_int8_b200 import synth

from lqtest import (AnchoredRun, compare_outputs, compare_snapshots, download_snapshot,
                    heads_major, io_dtype, make_config, oracle_tokens, rel_l2, to_device_tokens)

pytestmark = pytest.mark.gpu


def _wl(name, **over):
    return dataclasses.replace(synth.WORKLOADS[name], **over)


def _check_no_device_errors():
    assert lq.lq_device_errors() == 0


# --------------------------------------------------------------------------
# Init (I1): quantizing the same FP32 state gives bit-identical codes
# --------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["gdn_1x1_d64_fp32", "gdn_64x16_d128_bf16"])
def test_state_init_bit_exact(name):
    run = AnchoredRun(synth.WORKLOADS[name])
    run.init()  # asserts exact codes, scales and compensators
    _check_no_device_errors()


@pytest.mark.parametrize("dk,dv,r", [(128, 128, 4), (64, 128, 16), (128, 64, 0), (64, 64, 1)])
def test_state_init_zero_and_random(dk, dv, r):
    cfg = lq.Config(batch=3, heads=5, d_k=dk, d_v=dv, window=8, n_comp=r)
    st = lq.State(cfg)
    lq.lq_state_init(st, None)
    ref = oracle.quantize(np.zeros((15, dv, dk), np.float32), r)
    compare_snapshots(download_snapshot(st), ref, ref["row_norm"], exact_codes=True)
    rng = np.random.default_rng(dk + dv + r)
    S = (rng.standard_normal((15, dv, dk)) * rng.uniform(0.01, 100, size=(15, dv, 1))).astype(np.float32)
    lq.lq_state_init(st, torch.from_numpy(S).cuda())
    ref = oracle.quantize(S, r)
    compare_snapshots(download_snapshot(st), ref, ref["row_norm"], exact_codes=True)
    # smoothing off
    cfg.smoothing = 0
    st2 = lq.State(cfg)
    lq.lq_state_init(st2, torch.from_numpy(S).cuda())
    ref = oracle.quantize(S, r, smoothing=False)
    compare_snapshots(download_snapshot(st2), ref, ref["row_norm"], exact_codes=True)
    assert np.all(download_snapshot(st2)["col_smooth"] == 1.0)


# --------------------------------------------------------------------------
# Single GDN head, d = 64, 256 steps, W = 16, r = 4, FP32 io: every window
# --------------------------------------------------------------------------

def test_single_head_all_windows():
    wl = synth.WORKLOADS["gdn_1x1_d64_fp32"]
    run = AnchoredRun(wl)
    run.init()
    for w in range(wl.steps // wl.window):
        run.window(w)
    assert run.stats["windows"] == 16
    _check_no_device_errors()


@pytest.mark.parametrize("steps_per_call,commit_mode", [(5, "auto"), (16, "auto"), (3, "explicit"),
                                                        (16, "explicit")])
def test_single_head_call_shapes(steps_per_call, commit_mode):
    """Several tokens per launch, and commit as a separate call."""
    wl = synth.WORKLOADS["gdn_1x1_d64_fp32"]
    run = AnchoredRun(wl, steps_per_call=steps_per_call, commit_mode=commit_mode)
    run.init()
    for w in range(3):
        run.window(w)


@pytest.mark.parametrize("ntok", [1, 7, 15])
def test_commit_before_window_end(ntok):
    wl = synth.WORKLOADS["gdn_1x1_d64_fp32"]
    run = AnchoredRun(wl, steps_per_call=4, commit_mode="explicit")
    run.init()
    run.window(0, ntok=ntok)
    run.window(1)


# --------------------------------------------------------------------------
# Head sizes, gates, io types, window lengths, compensator counts, ragged
# batch x heads (not a multiple of anything), smoothing on / off
# --------------------------------------------------------------------------

VARIANTS = [
    # dk, dv, gate, io, W, r, smoothing, B, H
    (128, 128, "scalar", "bf16", 16, 4, True, 3, 5),
    (128, 128, "diag", "bf16", 16, 8, True, 2, 3),
    (64, 128, "scalar", "fp32", 8, 16, True, 1, 7),
    (128, 64, "diag", "fp32", 32, 0, True, 2, 2),
    (64, 64, "scalar", "bf16", 1, 0, True, 5, 1),
    (64, 64, "diag", "fp32", 1, 0, False, 1, 3),
    (128, 128, "scalar", "bf16", 32, 16, False, 1, 4),
    (128, 128, "scalar", "bf16", 1, 0, False, 4, 4),
    (64, 128, "diag", "bf16", 8, 2, True, 3, 1),
]


@pytest.mark.parametrize("dk,dv,gate,io,W,r,smooth,B,H", VARIANTS)
def test_variants(dk, dv, gate, io, W, r, smooth, B, H):
    wl = synth.DecodeWorkload(f"var_{dk}_{dv}_{gate}", B, H, dk, dv, 3 * W, W, r, gate, io, smooth,
                              max(1, dv // 100), max(1, dk // 100), 30.0)
    run = AnchoredRun(wl)
    run.init()
    for w in range(3):
        run.window(w)
    _check_no_device_errors()


# --------------------------------------------------------------------------
# GDN decode B = 64, H = 16, d = 128, bf16, W = 16, r = 4: every window of
# the 1024 steps, all heads
# --------------------------------------------------------------------------

def test_gdn_64x16_all_windows():
    wl = synth.WORKLOADS["gdn_64x16_d128_bf16"]
    run = AnchoredRun(wl)
    run.init()
    for w in range(wl.steps // wl.window):
        run.window(w)
    print("stats", run.stats)
    _check_no_device_errors()


# --------------------------------------------------------------------------
# Canaries: nothing is written outside the output and state buffers
# --------------------------------------------------------------------------

def test_canaries():
    wl = _wl("gdn_64x16_d128_bf16", batch=3, heads=5)
    cfg = make_config(wl)
    st = lq.State(cfg)
    pad = 4096
    bh = wl.nh

    def padded(t, fill):
        big = torch.full((t.numel() + 2 * pad,), fill, dtype=t.dtype, device=t.device)
        view = big[pad:pad + t.numel()].view(t.shape)
        return big, view

    bigs = {}
    for key in list(st.snap.t):
        if st.snap.t[key].numel():
            bigs[key], st.snap.t[key] = padded(st.snap.t[key], 77)
    for key in ("buf_gate", "buf_k", "buf_u"):
        bigs[key], view = padded(getattr(st, key), 77)
        setattr(st, key, view)
    st.c.snap = st.snap.c()
    st.c.buf_gate, st.c.buf_k, st.c.buf_u = (st.buf_gate.data_ptr(), st.buf_k.data_ptr(),
                                             st.buf_u.data_ptr())
    S0 = synth.initial_state(0, np.arange(3), np.arange(5), 128, 128, 2, 2, 30.0).reshape(bh, 128, 128)
    lq.lq_state_init(st, torch.from_numpy(S0).cuda())
    tok = to_device_tokens(synth.tokens(0, np.arange(3), np.arange(5), 0, 16, 128, 128, "scalar", "bf16"),
                           "bf16")
    obig = torch.full((3 * 5 * 128 + 2 * pad,), 7.0, dtype=torch.bfloat16, device="cuda")
    o = obig[pad:pad + 3 * 5 * 128].view(3, 1, 5, 128)
    for t in range(16):
        args = [tok[k][:, t:t + 1].contiguous() for k in ("q", "k", "v", "alpha", "beta")]
        lq.lq_decode_window(st, *args, 1, o)
    torch.cuda.synchronize()
    for key, big in bigs.items():
        assert torch.all(big[:pad] == 77) and torch.all(big[-pad:] == 77), key
    assert torch.all(obig[:pad] == 7.0) and torch.all(obig[-pad:] == 7.0)


# --------------------------------------------------------------------------
# FP32 per-step comparator (B2): the plain recurrence on an FP32 state
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dk,dv,gate,io,n", [(128, 128, "scalar", "bf16", 1), (128, 128, "diag", "fp32", 5),
                                             (64, 128, "scalar", "fp32", 3), (128, 64, "diag", "bf16", 2),
                                             (64, 64, "scalar", "bf16", 17)])
def test_fp32_step_parity(dk, dv, gate, io, n):
    B, H = 3, 4
    cfg = lq.Config(batch=B, heads=H, d_k=dk, d_v=dv, gate=lq.LQ_GATE_DIAG if gate == "diag" else 0,
                    io_dtype=lq.LQ_BF16 if io == "bf16" else lq.LQ_F32)
    S0 = synth.initial_state(0, np.arange(B), np.arange(H), dk, dv, 1, 1, 30.0).reshape(B * H, dv, dk)
    tok = synth.tokens(0, np.arange(B), np.arange(H), 0, n, dk, dv, gate, io)
    dev = to_device_tokens(tok, io)
    S = torch.from_numpy(S0).cuda()
    o = torch.empty((B, n, H, dv), dtype=io_dtype(io), device="cuda")
    lq.lq_fp32_step(cfg, S, dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"], n, o)
    torch.cuda.synchronize()
    d, kt, b, v, q = oracle_tokens(tok, gate)
    o_ref, S_ref = oracle.eq1_steps(S0.astype(np.float64), d, kt, b, v, q)
    compare_outputs(heads_major(o.float().cpu().numpy()), o_ref, io)
    assert rel_l2(S.cpu().numpy().reshape(B * H, -1), S_ref.reshape(B * H, -1)).max() < 1e-5


# --------------------------------------------------------------------------
# Prefill (P1 + P2), small: outputs, carried FP32 state and every snapshot
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dk,dv,gate,io,T,every,r", [(128, 128, "scalar", "bf16", 256, 64, 4),
                                                     (64, 128, "diag", "fp32", 96, 32, 2),
                                                     (128, 64, "scalar", "fp32", 100, 100, 0),
                                                     (128, 128, "scalar", "bf16", 200, 64, 3)])
def test_prefill_small(dk, dv, gate, io, T, every, r):
    B, H = 2, 3
    cfg = lq.Config(batch=B, heads=H, d_k=dk, d_v=dv, window=16, n_comp=r,
                    gate=lq.LQ_GATE_DIAG if gate == "diag" else 0,
                    io_dtype=lq.LQ_BF16 if io == "bf16" else lq.LQ_F32)
    st = lq.State(cfg)
    lq.lq_state_init(st, None)
    tok = synth.tokens(0, np.arange(B), np.arange(H), 0, T, dk, dv, gate, io)
    dev = to_device_tokens(tok, io)
    S = torch.zeros((B * H, dv, dk), dtype=torch.float32, device="cuda")
    o = torch.empty((B, T, H, dv), dtype=io_dtype(io), device="cuda")
    with_snaps = T % every == 0
    snaps = [lq.Snapshot(cfg, "cuda") for _ in range(T // every)] if with_snaps else None
    lq.lq_prefill_chunk(st, S, dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"], T, every,
                        snaps, o)
    torch.cuda.synchronize()
    d, kt, b, v, q = oracle_tokens(tok, gate)
    S0 = np.zeros((B * H, dv, dk))
    o_ref, snaps_ref, S_ref = oracle.prefill(S0, d, kt, b, v, q, every, r)
    compare_outputs(heads_major(o.float().cpu().numpy()), o_ref, io)
    assert rel_l2(S.cpu().numpy().reshape(B * H, -1), S_ref.reshape(B * H, -1)).max() < 1e-5
    if with_snaps:
        assert len(snaps_ref) == len(snaps)
        for sg, sr in zip(snaps, snaps_ref):
            compare_snapshots(sg.cpu(), sr, sr["row_norm"])
    final = oracle.quantize(S_ref.astype(np.float32), r)
    compare_snapshots(download_snapshot(st), final, final["row_norm"])
    _check_no_device_errors()


def test_prefill_then_decode():
    """Decode continues from the snapshot the prefill leaves in the state."""
    wl = _wl("gdn_64x16_d128_bf16", batch=2, heads=3, outlier_rows=0, outlier_cols=0)
    cfg = make_config(wl)
    st = lq.State(cfg)
    lq.lq_state_init(st, None)
    T = 128
    tok = synth.tokens(0, np.arange(2), np.arange(3), 0, T + 16, 128, 128, "scalar", "bf16")
    pre = {k: v[:, :T] for k, v in tok.items()}
    post = {k: v[:, T:] for k, v in tok.items()}
    dev = to_device_tokens(pre, "bf16")
    S = torch.zeros((6, 128, 128), dtype=torch.float32, device="cuda")
    o = torch.empty((2, T, 3, 128), dtype=torch.bfloat16, device="cuda")
    lq.lq_prefill_chunk(st, S, dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"], T, 64, None, o)
    snap_gpu = download_snapshot(st)
    d, kt, b, v, q = oracle_tokens(pre, "scalar")
    _, _, S_ref = oracle.prefill(np.zeros((6, 128, 128)), d, kt, b, v, q, 64, cfg.n_comp)
    ref = oracle.quantize(S_ref.astype(np.float32), cfg.n_comp)
    compare_snapshots(snap_gpu, ref, ref["row_norm"])
    # one window of decode from the oracle's snapshot
    lq.lq_state_restore(st, __import__("lqtest").upload_snapshot(cfg, ref))
    devp = to_device_tokens(post, "bf16")
    og = torch.empty((2, 16, 3, 128), dtype=torch.bfloat16, device="cuda")
    for t in range(16):
        args = [devp[k][:, t:t + 1].contiguous() for k in ("q", "k", "v", "alpha", "beta")]
        out = torch.empty((2, 1, 3, 128), dtype=torch.bfloat16, device="cuda")
        lq.lq_decode_window(st, *args, 1, out)
        og[:, t:t + 1] = out
    torch.cuda.synchronize()
    d, kt, b, v, q = oracle_tokens(post, "scalar")
    rec = oracle.empty_records(6, 16, 128, 128, 1)
    o_ref = oracle.window(ref, rec, 0, d, kt, b, v, q)
    compare_outputs(heads_major(og.float().cpu().numpy()), o_ref, "bf16")


# --------------------------------------------------------------------------
# Host-side errors on a real device: nothing launched, state unchanged
# --------------------------------------------------------------------------

def test_errors_leave_state_unchanged():
    wl = _wl("gdn_64x16_d128_bf16", batch=2, heads=2, window=4)
    cfg = make_config(wl, auto_commit=0)
    st = lq.State(cfg)
    lq.lq_state_init(st, None)
    tok = to_device_tokens(synth.tokens(0, np.arange(2), np.arange(2), 0, 5, 128, 128, "scalar", "bf16"),
                           "bf16")
    o = torch.empty((2, 4, 2, 128), dtype=torch.bfloat16, device="cuda")
    args = [tok[k][:, :4].contiguous() for k in ("q", "k", "v", "alpha", "beta")]
    lq.lq_decode_window(st, *args, 4, o)
    assert st.pos == 4
    before = {k: v.clone() for k, v in st.snap.t.items()}
    with pytest.raises(lq.LQError) as e:
        lq.lq_decode_window(st, *[a[:, :1].contiguous() for a in args], 1, o[:, :1].contiguous())
    assert e.value.status == lq.LQ_ERR_WINDOW_FULL and st.pos == 4
    with pytest.raises(lq.LQError) as e:
        lq.lq_state_snapshot(st, lq.Snapshot(cfg, "cuda"))
    assert e.value.status == lq.LQ_ERR_WINDOW_OPEN
    torch.cuda.synchronize()
    for k, v in st.snap.t.items():
        assert torch.equal(v, before[k])
    lq.lq_window_commit(st)
    assert st.pos == 0
    snap = lq.Snapshot(cfg, "cuda")
    lq.lq_state_snapshot(st, snap)
    torch.cuda.synchronize()
    for k in snap.t:
        assert torch.equal(snap.t[k], st.snap.t[k])
