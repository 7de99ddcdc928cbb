"""The chunked tensor-core prefill (scalar gate, BF16 io, d_k = 128) against
the oracle's token recurrence: outputs, the carried FP32 state and every
snapshot, for several pass sizes of the workspace (one chunk up to sixteen
per pass, and two workspace halves where the next pass is prepared while the
current one is scanned), intervals that end in a ragged tail of fewer than
64 tokens, both
value-row splits (d_v = 128: two CTAs per head; d_v = 64: one), and the b = 0
instance.  The same call without a workspace (token by token) agrees too."""
import numpy as np
import pytest
import torch

import oracle
import linear_attention_recurrent_int8_b200 as lq
from linear_attention_recurrent_int8_b200 import synth

from lqtest import (compare_outputs, compare_snapshots, download_snapshot, heads_major, oracle_tokens,
                    rel_l2, to_device_tokens)

pytestmark = pytest.mark.gpu

CHUNK_BYTES = 3 * 128 * 64 * 2  # [PT; T] of one chunk and head, three BF16 parts


def _run(B, H, dv, T, every, r, ws_chunks, delta=1, seed=0):
    dk = 128
    cfg = lq.Config(batch=B, heads=H, d_k=dk, d_v=dv, window=16, n_comp=r, gate=lq.LQ_GATE_SCALAR,
                    io_dtype=lq.LQ_BF16, delta=delta)
    st = lq.State(cfg)
    lq.lq_state_init(st, None)
    tok = synth.tokens(seed, np.arange(B), np.arange(H), 0, T, dk, dv, "scalar", "bf16")
    dev = to_device_tokens(tok, "bf16")
    S = torch.zeros((B * H, dv, dk), dtype=torch.float32, device="cuda")
    o = torch.empty((B, T, H, dv), dtype=torch.bfloat16, device="cuda")
    with_snaps = T % every == 0
    snaps = [lq.Snapshot(cfg, "cuda") for _ in range(T // every)] if with_snaps else None
    ws = None if ws_chunks == 0 else torch.empty(ws_chunks * B * H * CHUNK_BYTES, dtype=torch.uint8,
                                                 device="cuda")
    lq.lq_prefill_chunk(st, S, dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"], T, every,
                        snaps, o, workspace=ws)
    torch.cuda.synchronize()
    assert lq.lq_device_errors() == 0
    d, kt, b, v, q = oracle_tokens(tok, "scalar", delta)
    o_ref, snaps_ref, S_ref = oracle.prefill(np.zeros((B * H, dv, dk)), d, kt, b, v, q, every, r)
    compare_outputs(heads_major(o.float().cpu().numpy()), o_ref, "bf16")
    S_gpu = S.cpu().numpy()
    assert rel_l2(S_gpu.reshape(B * H, -1), S_ref.reshape(B * H, -1)).max() < 1e-5
    if with_snaps:
        for sg, sr in zip(snaps, snaps_ref):
            compare_snapshots(sg.cpu(), sr, sr["row_norm"])
    final = oracle.quantize(S_ref.astype(np.float32), r)
    compare_snapshots(download_snapshot(st), final, final["row_norm"])
    return o, S


@pytest.mark.parametrize("B,H,dv,T,every,r,ws_chunks", [
    (1, 1, 128, 64, 64, 4, 16),        # one chunk
    (1, 2, 128, 1024, 1024, 4, 16),    # one full pass of 16 chunks
    (2, 3, 64, 512, 256, 2, 3),        # d_v = 64, passes of 3 chunks
    (1, 2, 128, 320, 320, 1, 1),       # passes of one chunk
    (2, 2, 128, 200, 100, 3, 16),      # intervals of 64 + a 36-token tail on the token path
    (1, 3, 128, 2176, 2176, 4, 16),    # 34 chunks: passes of 16, 16, 2
    (1, 3, 128, 2176, 2176, 4, 32),    # the same in two workspace halves (next pass prepared during the scan)
    (2, 2, 128, 4096, 1024, 4, 32),    # two halves, four snapshot intervals of one pass each
    (2, 2, 64, 2112, 704, 2, 40),      # two halves with spare bytes; 11-chunk intervals, d_v = 64
])
def test_chunked_prefill_matches_oracle(B, H, dv, T, every, r, ws_chunks):
    _run(B, H, dv, T, every, r, ws_chunks)


def test_chunked_prefill_b0_instance():
    """delta = 0 (Mamba2 / linear attention rows of Table 4): A = 0, T = I, R = V."""
    _run(2, 2, 128, 256, 128, 2, 16, delta=0)


def test_chunked_equals_token_by_token():
    """Same inputs with and without a workspace: outputs within the bf16
    output tolerance of each other and FP32 states within 1e-5."""
    o1, S1 = _run(1, 2, 128, 384, 128, 2, 16, seed=3)
    o2, S2 = _run(1, 2, 128, 384, 128, 2, 0, seed=3)
    compare_outputs(heads_major(o1.float().cpu().numpy()), heads_major(o2.float().cpu().numpy()), "bf16")
    assert rel_l2(S1.cpu().numpy().reshape(2, -1), S2.cpu().numpy().reshape(2, -1)).max() < 1e-5
