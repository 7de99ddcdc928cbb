"""The b = 0 rows of Table 4 (lq_config.delta = 0: linear attention, RetNet,
Mamba2 with a scalar gate, GLA with a per-channel gate): u_t = v_t.  Decode
windows anchored on the oracle, the FP32 per-step comparator and a prefill
with its snapshots, each against the oracle's gated_linear_instance."""
import numpy as np
import pytest
import torch

import oracle
import linear_attention_recurrent_int8_b200 as lq
from linear_attention_recurrent_int8_b200 import synth

from lqtest import (AnchoredRun, compare_outputs, compare_snapshots, download_snapshot, heads_major,
                    io_dtype, oracle_tokens, rel_l2, to_device_tokens)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dk,dv,gate,io,W,r,B,H", [
    (128, 128, "scalar", "bf16", 16, 4, 3, 5),   # Mamba2-like
    (128, 128, "diag", "fp32", 8, 2, 2, 3),      # GLA-like
    (64, 128, "scalar", "fp32", 1, 0, 4, 2),     # per-token
    (128, 64, "diag", "bf16", 32, 16, 1, 3),
])
def test_decode_windows_without_delta_rule(dk, dv, gate, io, W, r, B, H):
    wl = synth.DecodeWorkload(f"gl_{dk}_{dv}_{gate}", B, H, dk, dv, 3 * W, W, r, gate, io, True,
                              max(1, dv // 100), max(1, dk // 100), 30.0, delta=0)
    run = AnchoredRun(wl)
    run.init()
    for w in range(3):
        run.window(w)
    # records: u = v exactly (v as stored on the device)
    assert lq.lq_device_errors() == 0


@pytest.mark.parametrize("gate,io,n", [("scalar", "fp32", 4), ("diag", "bf16", 3)])
def test_fp32_step_without_delta_rule(gate, io, n):
    B, H, dk, dv = 2, 3, 128, 128
    cfg = lq.Config(batch=B, heads=H, d_k=dk, d_v=dv, gate=lq.LQ_GATE_DIAG if gate == "diag" else 0,
                    io_dtype=lq.LQ_BF16 if io == "bf16" else lq.LQ_F32, delta=0)
    S0 = synth.initial_state(0, np.arange(B), np.arange(H), dk, dv, 1, 1, 30.0).reshape(B * H, dv, dk)
    tok = synth.tokens(0, np.arange(B), np.arange(H), 0, n, dk, dv, gate, io)
    dev = to_device_tokens(tok, io)
    S = torch.from_numpy(S0).cuda()
    o = torch.empty((B, n, H, dv), dtype=io_dtype(io), device="cuda")
    lq.lq_fp32_step(cfg, S, dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"], n, o)
    torch.cuda.synchronize()
    d, kt, b, v, q = oracle_tokens(tok, gate, delta=0)
    o_ref, S_ref = oracle.eq1_steps(S0.astype(np.float64), d, kt, b, v, q)
    compare_outputs(heads_major(o.float().cpu().numpy()), o_ref, io)
    assert rel_l2(S.cpu().numpy().reshape(B * H, -1), S_ref.reshape(B * H, -1)).max() < 1e-5


def test_prefill_without_delta_rule():
    B, H, dk, dv, T, every, r = 2, 3, 128, 128, 192, 64, 4
    cfg = lq.Config(batch=B, heads=H, d_k=dk, d_v=dv, window=16, n_comp=r, delta=0)
    st = lq.State(cfg)
    lq.lq_state_init(st, None)
    tok = synth.tokens(0, np.arange(B), np.arange(H), 0, T, dk, dv, "scalar", "bf16")
    dev = to_device_tokens(tok, "bf16")
    S = torch.zeros((B * H, dv, dk), dtype=torch.float32, device="cuda")
    o = torch.empty((B, T, H, dv), dtype=torch.bfloat16, device="cuda")
    snaps = [lq.Snapshot(cfg, "cuda") for _ in range(T // every)]
    lq.lq_prefill_chunk(st, S, dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"], T, every,
                        snaps, o)
    torch.cuda.synchronize()
    d, kt, b, v, q = oracle_tokens(tok, "scalar", delta=0)
    o_ref, snaps_ref, S_ref = oracle.prefill(np.zeros((B * H, dv, dk)), d, kt, b, v, q, every, r)
    compare_outputs(heads_major(o.float().cpu().numpy()), o_ref, "bf16")
    assert rel_l2(S.cpu().numpy().reshape(B * H, -1), S_ref.reshape(B * H, -1)).max() < 1e-5
    for sg, sr in zip(snaps, snaps_ref):
        compare_snapshots(sg.cpu(), sr, sr["row_norm"])
    assert lq.lq_device_errors() == 0
