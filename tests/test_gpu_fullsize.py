"""Parity at the workloads' full sizes, in the launch configuration the
benchmark times (every sequence and head on the device), checked against the
oracle on a seeded sample of (sequence, head) pairs in every window, and on
every head in the first windows.  See lqtest.SampledRun / AnchoredRun."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import linear_attention_recurrent_int8_b200 as lq
from linear_attention_recurrent_int8_b200 import synth

from lqtest import (AnchoredRun, SampledRun, compare_outputs, compare_snapshots, heads_major,
                    make_config, oracle_tokens, rel_l2)

pytestmark = pytest.mark.gpu


def test_kda_128x32_all_steps_sampled():
    """KDA-style per-channel gate, batch 128 x 32 heads, 2048 steps, W=16, r=8."""
    wl = synth.WORKLOADS["kda_128x32_d128_bf16"]
    run = SampledRun(wl, n_sample=24)
    run.init()
    for w in range(wl.steps // wl.window):
        run.window(w)
    print("stats", run.stats)
    assert lq.lq_device_errors() == 0


def test_kda_128x32_first_window_all_heads():
    wl = synth.WORKLOADS["kda_128x32_d128_bf16"]
    run = AnchoredRun(wl)
    run.init()
    run.window(0)


def test_gdn_256x32_all_steps_sampled():
    """Large-batch GDN decode, batch 256 x 32 heads, 4096 steps, W=16, r=4."""
    wl = synth.WORKLOADS["gdn_256x32_d128_bf16"]
    run = SampledRun(wl, n_sample=24)
    run.init()
    for w in range(wl.steps // wl.window):
        run.window(w)
    print("stats", run.stats)
    assert lq.lq_device_errors() == 0


def test_gdn_256x32_first_windows_all_heads():
    wl = synth.WORKLOADS["gdn_256x32_d128_bf16"]
    run = AnchoredRun(wl)
    run.init()
    run.window(0)
    run.window(1)


@pytest.mark.parametrize("W,r", [(1, 0), (8, 4), (32, 8), (16, 0), (16, 8), (8, 0), (32, 4)])
def test_gdn_256x32_window_and_compensator_sweep(W, r):
    """The large-batch workload's W in {1, 8, 16, 32} x r in {0, 4, 8} sweep
    (W = 1, r = 0 is per-token quantization)."""
    wl = dataclasses.replace(synth.WORKLOADS["gdn_256x32_d128_bf16"], window=W, n_comp=r)
    run = SampledRun(wl, n_sample=12, seed=W * 100 + r)
    run.init()
    for w in range(max(3, 32 // W)):
        run.window(w)


def test_per_token_without_smoothing():
    """Plain INT8 per-step (W = 1, r = 0, no smoothing)."""
    wl = dataclasses.replace(synth.WORKLOADS["gdn_256x32_d128_bf16"], window=1, n_comp=0,
                             smoothing=False)
    run = SampledRun(wl, n_sample=12, seed=7)
    run.init()
    for w in range(16):
        run.window(w)


def test_prefill_65536_then_decode_sampled():
    """Chunked GDN prefill, batch 2 x 32 heads, T = 65536, a quantized
    snapshot every 1024 tokens; then 512 decode steps from the last snapshot
    (W = 16, r = 4).  Eight sampled heads follow the oracle over all tokens."""
    P = synth.PREFILL_WORKLOAD
    B, H, dk, dv, T, every, r = P["batch"], P["heads"], P["d_k"], P["d_v"], P["T"], \
        P["snapshot_every"], P["n_comp"]
    dev = "cuda"
    cfg = lq.Config(batch=B, heads=H, d_k=dk, d_v=dv, window=P["window"], n_comp=r,
                    gate=lq.LQ_GATE_SCALAR, io_dtype=lq.LQ_BF16, smoothing=1, auto_commit=1)
    st = lq.State(cfg, dev)
    lq.lq_state_init(st, None)
    # eight sampled heads of both sequences (each head spans both value-row
    # slices of the chunked scan)
    sample = [(0, 0), (0, 5), (0, 17), (0, 31), (1, 2), (1, 13), (1, 24), (1, 30)]
    sb = np.array([s[0] for s in sample])
    sh = np.array([s[1] for s in sample])
    # device inputs for all heads, drawn in slices; sampled heads from numpy
    q = torch.empty((B, T, H, dk), dtype=torch.bfloat16, device=dev)
    k = torch.empty_like(q)
    v = torch.empty((B, T, H, dv), dtype=torch.bfloat16, device=dev)
    alpha = torch.empty((B, T, H), dtype=torch.float32, device=dev)
    beta = torch.empty_like(alpha)
    step = 4096
    for t0 in range(0, T, step):
        tok = synth.torch_tokens(P["seed"], B, H, t0, t0 + step, dk, dv, "scalar", "bf16", dev)
        q[:, t0:t0 + step], k[:, t0:t0 + step], v[:, t0:t0 + step] = tok["q"], tok["k"], tok["v"]
        alpha[:, t0:t0 + step], beta[:, t0:t0 + step] = tok["alpha"], tok["beta"]
    tok_s = [synth.tokens(P["seed"], [b], [h], 0, T, dk, dv, "scalar", "bf16") for b, h in sample]
    for i, (b, h) in enumerate(sample):
        q[b, :, h] = torch.from_numpy(tok_s[i]["q"][0, :, 0]).to(dev, torch.bfloat16)
        k[b, :, h] = torch.from_numpy(tok_s[i]["k"][0, :, 0]).to(dev, torch.bfloat16)
        v[b, :, h] = torch.from_numpy(tok_s[i]["v"][0, :, 0]).to(dev, torch.bfloat16)
        alpha[b, :, h] = torch.from_numpy(tok_s[i]["alpha"][0, :, 0]).to(dev)
        beta[b, :, h] = torch.from_numpy(tok_s[i]["beta"][0, :, 0]).to(dev)
    S = torch.zeros((B * H, dv, dk), dtype=torch.float32, device=dev)
    o = torch.empty((B, T, H, dv), dtype=torch.bfloat16, device=dev)
    snaps = [lq.Snapshot(cfg, dev) for _ in range(T // every)]
    lq.lq_prefill_chunk(st, S, q, k, v, alpha, beta, T, every, snaps, o)
    torch.cuda.synchronize()
    assert lq.lq_device_errors() == 0

    bh = sb * H + sh
    tok_o = {kk: np.concatenate([t[kk] for t in tok_s], axis=2) for kk in tok_s[0]}
    d, kt, b_, vv, qq = oracle_tokens(tok_o, "scalar")
    o_ref, snaps_ref, S_ref = oracle.prefill(np.zeros((len(sample), dv, dk)), d, kt, b_, vv, qq,
                                             every, r)
    o_gpu = torch.stack([o[b, :, h] for b, h in sample]).float().cpu().numpy()
    compare_outputs(o_gpu, o_ref, "bf16", "prefill outputs")
    S_gpu = S[torch.from_numpy(bh).to(dev)].cpu().numpy()
    assert rel_l2(S_gpu.reshape(len(sample), -1), S_ref.reshape(len(sample), -1)).max() < 1e-4
    for n, sr in enumerate(snaps_ref):
        sg = {kk: vvv[torch.from_numpy(bh).to(dev)].cpu().numpy() for kk, vvv in snaps[n].t.items()}
        compare_snapshots(sg, sr, sr["row_norm"])

    # 512 decode steps from the prefill's final snapshot, sampled heads anchored
    wl = synth.DecodeWorkload("gdn_prefill_decode", B, H, dk, dv, P["decode_steps"], P["window"], r,
                              "scalar", "bf16", True)
    run = SampledRun(wl, n_sample=0)
    run.st = st
    run.sample = bh
    run.sb, run.sh = sb, sh
    run.idx = torch.from_numpy(bh).to(dev)
    run.snap = oracle.quantize(S_ref.astype(np.float32), r)
    # decode inputs continue the prompt's token positions
    wl.seed = P["seed"]
    for w in range(P["decode_steps"] // P["window"]):
        run.window(T // P["window"] + w)
    assert lq.lq_device_errors() == 0
