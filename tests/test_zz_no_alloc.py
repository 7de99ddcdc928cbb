"""lq_prefill_chunk_noalloc: the prefill for callers that cannot give the
library device memory of its own (a serving engine whose pool already holds
the GPU's memory, a plug-in that only receives its input and output buffers,
code that must avoid cudaMalloc's device synchronization).  Its scratch is a
fixed array inside the library; it must give what lq_prefill_chunk gives with
a workspace, on two calls in a row (the second finds the first call's
leftovers in the array).  Collected last so that a run stopping at the first
failure has run every other test."""
import numpy as np
import pytest
import torch

import linear_attention_recurrent_int8_b200 as lq
from linear_attention_recurrent_int8_b200 import synth

from lqtest import compare_outputs, compare_snapshots, download_snapshot, heads_major, rel_l2, to_device_tokens

pytestmark = pytest.mark.gpu


def _prefill(fn, cfg, tok, T, every, **kw):
    st = lq.State(cfg)
    lq.lq_state_init(st, None)
    dev = to_device_tokens(tok, "bf16")
    S = torch.zeros((cfg.batch * cfg.heads, cfg.d_v, cfg.d_k), dtype=torch.float32, device="cuda")
    o = torch.empty((cfg.batch, T, cfg.heads, cfg.d_v), dtype=torch.bfloat16, device="cuda")
    snaps = [lq.Snapshot(cfg, "cuda") for _ in range(T // every)]
    fn(st, S, dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"], T, every, snaps, o, **kw)
    torch.cuda.synchronize()
    return o, S, [s.cpu() for s in snaps], download_snapshot(st)


def _same(a, b):
    o1, S1, sn1, f1 = a
    o2, S2, sn2, f2 = b
    compare_outputs(heads_major(o1.float().cpu().numpy()), heads_major(o2.float().cpu().numpy()), "bf16")
    n = S1.shape[0]
    assert rel_l2(S1.cpu().numpy().reshape(n, -1), S2.cpu().numpy().reshape(n, -1)).max() < 1e-5
    for x, y in zip(sn1 + [f1], sn2 + [f2]):
        compare_snapshots(x, y)


@pytest.mark.parametrize("B,H,dv,T,every", [(2, 3, 128, 320, 64), (4, 40, 64, 256, 128)])
def test_noalloc_prefill_matches_workspace_prefill_twice(B, H, dv, T, every):
    cfg = lq.Config(batch=B, heads=H, d_k=128, d_v=dv, window=16, n_comp=2, gate=lq.LQ_GATE_SCALAR,
                    io_dtype=lq.LQ_BF16)
    tok1 = synth.tokens(0, np.arange(B), np.arange(H), 0, T, 128, dv, "scalar", "bf16")
    tok2 = synth.tokens(1, np.arange(B), np.arange(H), 0, T, 128, dv, "scalar", "bf16")
    want1 = _prefill(lq.lq_prefill_chunk, cfg, tok1, T, every)
    want2 = _prefill(lq.lq_prefill_chunk, cfg, tok2, T, every)
    got1 = _prefill(lq.lq_prefill_chunk_noalloc, cfg, tok1, T, every)
    got2 = _prefill(lq.lq_prefill_chunk_noalloc, cfg, tok2, T, every)
    _same(got1, want1)
    _same(got2, want2)
    assert lq.lq_device_errors() == 0


def test_noalloc_prefill_rejects_more_heads_than_its_array_holds():
    """One chunk of scratch is 48 KB per sequence and head: 8 MiB holds 170."""
    cfg = lq.Config(batch=171, heads=1, d_k=128, d_v=64, window=16, n_comp=0, gate=lq.LQ_GATE_SCALAR,
                    io_dtype=lq.LQ_BF16)
    tok = synth.tokens(0, np.arange(171), np.arange(1), 0, 64, 128, 64, "scalar", "bf16")
    with pytest.raises(lq.LQError) as e:
        _prefill(lq.lq_prefill_chunk_noalloc, cfg, tok, 64, 64)
    assert e.value.status == lq.LQ_ERR_UNSUPPORTED
