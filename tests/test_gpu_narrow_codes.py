"""The 6- and 4-bit code widths and the BF16 state (lq_config.bits = 6, 4,
16): the same parity bar as the 8-bit state -- initialisation bit-exact,
anchored windows (outputs, records, next snapshot with codes within one
step, a BF16 residual within one BF16 step), the prefill's snapshots,
per-sequence positions and a full-size sampled run -- against the oracle's
quantizer at the same width.  4-bit codes are packed two per byte on the
device (lq.h); the helpers unpack them before comparing."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import linear_attention_recurrent_int8_b200 as lq
from linear_attention_recurrent_int8_b200 import synth

from lqtest import (AnchoredRun, SampledRun, compare_outputs, compare_snapshots,
                    download_snapshot, heads_major, io_dtype, make_config, oracle_tokens, rel_l2,
                    snapshot_to_host, to_device_tokens)

pytestmark = pytest.mark.gpu


def _check_no_device_errors():
    assert lq.lq_device_errors() == 0


@pytest.mark.parametrize("bits", [4, 6, 16])
@pytest.mark.parametrize("name", ["gdn_1x1_d64_fp32", "gdn_64x16_d128_bf16"])
def test_state_init_bit_exact(name, bits):
    wl = synth.WORKLOADS[name]
    run = AnchoredRun(wl, cfg=make_config(wl, bits=bits))
    run.init()
    _check_no_device_errors()


VARIANTS = [
    # dk, dv, gate, io, W, r, smoothing, B, H, bits
    (128, 128, "scalar", "bf16", 16, 4, True, 3, 5, 4),
    (128, 128, "diag", "bf16", 16, 8, True, 2, 3, 4),
    (64, 128, "scalar", "fp32", 8, 16, True, 1, 7, 4),
    (128, 64, "diag", "fp32", 32, 0, True, 2, 2, 4),
    (64, 64, "scalar", "bf16", 1, 0, False, 5, 1, 4),
    (128, 128, "scalar", "fp32", 16, 4, True, 2, 3, 6),
    (64, 128, "diag", "bf16", 8, 2, True, 3, 1, 6),
    (128, 128, "scalar", "bf16", 16, 0, True, 3, 5, 16),
    (128, 128, "diag", "fp32", 8, 4, True, 2, 3, 16),
    (64, 64, "scalar", "bf16", 1, 0, True, 4, 2, 16),
    (128, 64, "scalar", "fp32", 32, 2, False, 1, 3, 16),
]


@pytest.mark.parametrize("dk,dv,gate,io,W,r,smooth,B,H,bits", VARIANTS)
def test_variants(dk, dv, gate, io, W, r, smooth, B, H, bits):
    wl = synth.DecodeWorkload(f"var{bits}_{dk}_{dv}_{gate}", B, H, dk, dv, 3 * W, W, r, gate, io,
                              smooth, max(1, dv // 100), max(1, dk // 100), 30.0)
    run = AnchoredRun(wl, cfg=make_config(wl, bits=bits))
    run.init()
    for w in range(3):
        run.window(w)
    _check_no_device_errors()


@pytest.mark.parametrize("bits", [4, 6, 16])
def test_explicit_commit_short_window(bits):
    wl = synth.WORKLOADS["gdn_1x1_d64_fp32"]
    run = AnchoredRun(wl, cfg=make_config(wl, bits=bits), steps_per_call=3, commit_mode="explicit")
    run.init()
    run.window(0, ntok=7)
    run.window(1)
    _check_no_device_errors()


@pytest.mark.parametrize("bits", [4, 6, 16])
def test_prefill_snapshots(bits):
    B, H, dk, dv, T, every, r, io = 2, 3, 128, 128, 192, 64, 4, "bf16"
    cfg = lq.Config(batch=B, heads=H, d_k=dk, d_v=dv, window=16, n_comp=r, gate=0,
                    io_dtype=lq.LQ_BF16, bits=bits)
    st = lq.State(cfg)
    lq.lq_state_init(st, None)
    tok = synth.tokens(0, np.arange(B), np.arange(H), 0, T, dk, dv, "scalar", io)
    dev = to_device_tokens(tok, io)
    S = torch.zeros((B * H, dv, dk), dtype=torch.float32, device="cuda")
    o = torch.empty((B, T, H, dv), dtype=io_dtype(io), device="cuda")
    snaps = [lq.Snapshot(cfg, "cuda") for _ in range(T // every)]
    lq.lq_prefill_chunk(st, S, dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"], T, every,
                        snaps, o)
    torch.cuda.synchronize()
    d, kt, b, v, q = oracle_tokens(tok, "scalar")
    o_ref, snaps_ref, S_ref = oracle.prefill(np.zeros((B * H, dv, dk)), d, kt, b, v, q, every, r,
                                             bits=bits)
    compare_outputs(heads_major(o.float().cpu().numpy()), o_ref, io)
    assert rel_l2(S.cpu().numpy().reshape(B * H, -1), S_ref.reshape(B * H, -1)).max() < 1e-5
    assert len(snaps_ref) == len(snaps)
    for sg, sr in zip(snaps, snaps_ref):
        compare_snapshots(snapshot_to_host(cfg, sg), sr, sr["row_norm"])
    final = oracle.quantize(S_ref.astype(np.float32), r, bits=bits)
    compare_snapshots(download_snapshot(st), final, final["row_norm"])
    _check_no_device_errors()


def test_snapshot_copy_moves_packed_bytes():
    """lq_state_snapshot / lq_state_restore move d_v d_k / 2 code bytes per head at 4 bits."""
    wl = synth.WORKLOADS["gdn_64x16_d128_bf16"]
    cfg = make_config(wl, bits=4)
    assert lq.lq_buffer_elems(cfg, 0) == wl.nh * wl.d_v * wl.d_k // 2
    run = AnchoredRun(wl, cfg=cfg)
    ref = run.init()
    dst = lq.Snapshot(cfg, "cuda")
    lq.lq_state_snapshot(run.st, dst)
    torch.cuda.synchronize()
    assert torch.equal(dst.t["codes"], run.st.snap.t["codes"])
    compare_snapshots(snapshot_to_host(cfg, dst), ref, ref["row_norm"], exact_codes=True)


def test_gdn_256x32_4bit_sampled():
    """The large-batch GDN workload (256 x 32 heads, W = 16, r = 4) at 4 bits,
    in the benchmark's launch configuration, against the oracle on a seeded
    sample of heads for 8 windows."""
    wl = synth.WORKLOADS["gdn_256x32_d128_bf16"]
    run = SampledRun(wl, n_sample=16, seed=44, bits=4)
    run.init()
    for w in range(8):
        run.window(w)
    _check_no_device_errors()


def test_snapshot_copy_moves_bf16_residual():
    wl = synth.WORKLOADS["gdn_1x1_d64_fp32"]
    cfg = make_config(wl, bits=16)
    assert lq.lq_buffer_elems(cfg, 0) == wl.nh * wl.d_v * wl.d_k  # bf16 elements
    run = AnchoredRun(wl, cfg=cfg)
    ref = run.init()
    dst = lq.Snapshot(cfg, "cuda")
    lq.lq_state_snapshot(run.st, dst)
    torch.cuda.synchronize()
    assert dst.t["codes"].dtype == torch.bfloat16
    assert torch.equal(dst.t["codes"], run.st.snap.t["codes"])
    compare_snapshots(snapshot_to_host(cfg, dst), ref, ref["row_norm"], exact_codes=True)


def test_gdn_256x32_bf16_state_sampled():
    """The large-batch GDN workload with a BF16 state and no compensators (the
    BF16 per-window row of the paper's Table 2 ablation), in the benchmark's
    launch configuration, against the oracle on a seeded sample of heads."""
    wl = dataclasses.replace(synth.WORKLOADS["gdn_256x32_d128_bf16"], n_comp=0)
    run = SampledRun(wl, n_sample=16, seed=45, bits=16)
    run.init()
    for w in range(6):
        run.window(w)
    _check_no_device_errors()
