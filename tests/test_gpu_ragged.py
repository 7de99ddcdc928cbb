"""Per-sequence window positions (lq_decode_ragged): the sequences of a batch
decode at their own window positions and commit when their own window
fills.  Checked against the oracle sequence by sequence, anchored on the
oracle's snapshot at each of the sequence's window starts (the snapshot of
that sequence's heads is written into the device state there)."""
import numpy as np
import pytest
import torch

import oracle
import linear_attention_recurrent_int8_b200 as lq
from linear_attention_recurrent_int8_b200 import synth

from lqtest import (compare_outputs, compare_snapshots, download_snapshot, heads_major, io_dtype,
                    make_config, oracle_tokens, residual_to_device)

pytestmark = pytest.mark.gpu

SENTINEL = 7.0


def _slice_snap(snap, heads):
    return {k: np.ascontiguousarray(v[heads]) for k, v in snap.items()}


def _write_heads(st, snap, heads):
    """Device state's snapshot of `heads` <- snap (oracle arrays for those heads)."""
    idx = torch.as_tensor(heads, device="cuda")
    for key in ("codes", "row_scale", "col_smooth", "comp_row", "comp_val"):
        if key == "codes":
            st.snap.t[key][idx] = residual_to_device(st.cfg, snap)
            continue
        src = np.ascontiguousarray(snap[key], np.int32 if key == "comp_row" else None)
        st.snap.t[key][idx] = torch.from_numpy(src).to("cuda")


def _run(dk, dv, gate, io, W, r, B, H, steps, start_of, bits=8, flush=False):
    wl = synth.DecodeWorkload(f"ragged_{dk}_{dv}_{gate}", B, H, dk, dv, steps, W, r, gate, io, True,
                              max(1, dv // 100), max(1, dk // 100), 30.0)
    cfg = make_config(wl, auto_commit=0, bits=bits)
    st = lq.State(cfg, "cuda")
    bs, hs = np.arange(B), np.arange(H)
    S0 = synth.initial_state(wl.seed, bs, hs, dk, dv, wl.outlier_rows, wl.outlier_cols,
                             wl.outlier_scale).reshape(B * H, dv, dk)
    lq.lq_state_init(st, torch.from_numpy(S0).to("cuda"))
    ref0 = oracle.quantize(S0, r, True, bits)
    anchor = {b: _slice_snap(ref0, np.arange(b * H, (b + 1) * H)) for b in range(B)}
    seq_pos = torch.full((B,), -1, dtype=torch.int32, device="cuda")
    count = [0] * B            # tokens decoded so far by each sequence
    outs = {b: [] for b in range(B)}
    checked = 0
    for s in range(steps):
        for b in range(B):
            if s == start_of[b]:
                seq_pos[b] = 0
        active = [b for b in range(B) if s >= start_of[b]]
        for b in active:
            if count[b] % W == 0:  # window start: anchor on the oracle
                _write_heads(st, anchor[b], np.arange(b * H, (b + 1) * H))
        # this step's inputs: sequence b's own token count[b]; idle slots get zeros
        q = torch.zeros((B, 1, H, dk), dtype=io_dtype(io), device="cuda")
        k, v = torch.zeros_like(q), torch.zeros((B, 1, H, dv), dtype=io_dtype(io), device="cuda")
        alpha = torch.ones((B, 1, H, dk) if gate == "diag" else (B, 1, H), device="cuda")
        beta = torch.zeros((B, 1, H), device="cuda")
        toks = {}
        for b in active:
            tok = synth.tokens(wl.seed, [b], hs, count[b], count[b] + 1, dk, dv, gate, io)
            toks[b] = tok
            q[b] = torch.from_numpy(np.ascontiguousarray(tok["q"][0])).to("cuda", q.dtype)
            k[b] = torch.from_numpy(np.ascontiguousarray(tok["k"][0])).to("cuda", k.dtype)
            v[b] = torch.from_numpy(np.ascontiguousarray(tok["v"][0])).to("cuda", v.dtype)
            alpha[b] = torch.from_numpy(np.ascontiguousarray(tok["alpha"][0])).to("cuda")
            beta[b] = torch.from_numpy(np.ascontiguousarray(tok["beta"][0])).to("cuda")
        o = torch.full((B, 1, H, dv), SENTINEL, dtype=io_dtype(io), device="cuda")
        lq.lq_decode_ragged(st, seq_pos, q, k, v, alpha, beta, o)
        torch.cuda.synchronize()
        o_h = o.float().cpu().numpy()
        for b in range(B):
            if b not in active:
                assert np.all(o_h[b] == SENTINEL), f"idle sequence {b} output written"
        snap_gpu = None
        for b in active:
            outs[b].append((toks[b], o_h[b:b + 1]))
            count[b] += 1
            if count[b] % W == 0:
                # the window of sequence b just filled and was committed
                win = outs[b][-W:]
                tok = {key: np.concatenate([t[key] for t, _ in win], axis=1) for key in win[0][0]}
                d, kt, bb, vv, qq = oracle_tokens(tok, gate)
                rec = oracle.empty_records(H, W, dk, dv, dk if gate == "diag" else 1)
                o_ref = oracle.window(anchor[b], rec, 0, d, kt, bb, vv, qq)
                o_gpu = heads_major(np.concatenate([x for _, x in win], axis=1))
                compare_outputs(o_gpu, o_ref, io, f"sequence {b} window ending at token {count[b]}")
                new, _ = oracle.commit(anchor[b], rec, W, r, True, bits)
                if snap_gpu is None:
                    snap_gpu = download_snapshot(st)
                compare_snapshots(_slice_snap(snap_gpu, np.arange(b * H, (b + 1) * H)), new,
                                  new["row_norm"])
                anchor[b] = new
                checked += 1
        want = [count[b] % W if s >= start_of[b] else -1 for b in range(B)]
        assert seq_pos.cpu().tolist() == want, "positions not advanced modulo W"
    if flush:
        checked += _flush_and_check(st, seq_pos, outs, count, anchor, start_of, steps, W, r, H, dk,
                                    dv, gate, bits)
    assert lq.lq_device_errors() == 0
    return checked


def _flush_and_check(st, seq_pos, outs, count, anchor, start_of, steps, W, r, H, dk, dv, gate,
                     bits):
    """lq_ragged_flush commits each sequence's open window (count % W
    records) as the oracle's commit of those records would; sequences at a
    window start and idle slots keep their snapshots; positions go to 0."""
    B = len(count)
    assert st.pos == lq.LQ_POS_PER_SEQUENCE
    with pytest.raises(lq.LQError):  # windows may be open: the synchronous calls refuse
        lq.lq_window_commit(st)
    with pytest.raises(lq.LQError):
        lq.lq_state_snapshot(st, lq.Snapshot(st.cfg, "cuda"))
    before = download_snapshot(st)
    lq.lq_ragged_flush(st, seq_pos)
    torch.cuda.synchronize()
    assert st.pos == 0
    assert seq_pos.cpu().tolist() == [0 if steps > start_of[b] else -1 for b in range(B)]
    after = download_snapshot(st)
    flushed = 0
    for b in range(B):
        heads = np.arange(b * H, (b + 1) * H)
        n = count[b] % W
        if n == 0:
            for key in before:
                np.testing.assert_array_equal(after[key][heads], before[key][heads], err_msg=key)
            continue
        win = outs[b][-n:]
        tok = {key: np.concatenate([t[key] for t, _ in win], axis=1) for key in win[0][0]}
        d, kt, bb, vv, qq = oracle_tokens(tok, gate)
        rec = oracle.empty_records(H, W, dk, dv, dk if gate == "diag" else 1)
        oracle.window(anchor[b], rec, 0, d, kt, bb, vv, qq)
        new, _ = oracle.commit(anchor[b], rec, n, r, True, bits)
        compare_snapshots(_slice_snap(after, heads), new, new["row_norm"])
        flushed += 1
    # the state is closed again: a prefix-cache snapshot is allowed
    dst = lq.Snapshot(st.cfg, "cuda")
    lq.lq_state_snapshot(st, dst)
    torch.cuda.synchronize()
    for key in dst.t:
        assert torch.equal(dst.t[key], st.snap.t[key]), key
    assert flushed >= 1
    return flushed


@pytest.mark.parametrize("dk,dv,gate,io,W,r,B,H", [
    (128, 128, "scalar", "bf16", 4, 2, 5, 3),
    (64, 128, "diag", "fp32", 3, 1, 4, 2),
    (128, 64, "scalar", "fp32", 5, 0, 3, 4),
])
def test_ragged_staggered_windows(dk, dv, gate, io, W, r, B, H):
    start_of = [b % W for b in range(B)]  # every window phase present at once
    checked = _run(dk, dv, gate, io, W, r, B, H, steps=3 * W + 2, start_of=start_of)
    assert checked >= B * 2


def test_ragged_staggered_windows_4bit():
    _run(128, 128, "scalar", "bf16", 4, 2, 5, 3, steps=3 * 4 + 2, start_of=[b % 4 for b in range(5)],
         bits=4)


def test_ragged_staggered_windows_bf16_state():
    _run(64, 128, "diag", "fp32", 3, 1, 4, 2, steps=3 * 3 + 2, start_of=[b % 3 for b in range(4)],
         bits=16)


def test_ragged_matches_synchronous_when_aligned():
    """All sequences started together: the ragged path is the synchronous one."""
    _run(128, 128, "scalar", "bf16", 4, 2, 3, 2, steps=8, start_of=[0, 0, 0])


def test_ragged_position_out_of_range_is_skipped_and_reported():
    cfg = lq.Config(batch=3, heads=2, d_k=128, d_v=128, window=4, n_comp=1, io_dtype=lq.LQ_F32)
    st = lq.State(cfg, "cuda")
    lq.lq_state_init(st, None)
    seq_pos = torch.tensor([0, 4, -1], dtype=torch.int32, device="cuda")  # 4 == W is invalid
    q = torch.randn((3, 1, 2, 128), device="cuda")
    q = q / q.norm(dim=-1, keepdim=True)
    k, v = q.clone(), torch.randn((3, 1, 2, 128), device="cuda")
    alpha, beta = torch.full((3, 1, 2), 0.9, device="cuda"), torch.full((3, 1, 2), 0.5, device="cuda")
    o = torch.full((3, 1, 2, 128), SENTINEL, device="cuda")
    lq.lq_decode_ragged(st, seq_pos, q, k, v, alpha, beta, o)
    torch.cuda.synchronize()
    assert lq.lq_device_errors() == 2  # the bad-position flag, and nothing else
    oh = o.cpu().numpy()
    assert np.all(oh[1] == SENTINEL) and np.all(oh[2] == SENTINEL)
    assert np.all(np.isfinite(oh[0])) and not np.all(oh[0] == SENTINEL)
    assert seq_pos.cpu().tolist() == [1, 4, -1]  # only valid positions advance


@pytest.mark.parametrize("bits", [8, 4])
def test_ragged_flush_commits_every_open_window(bits):
    """Staggered sequences left at positions 2, 1, 0, 3 and one idle slot:
    the flush commits 2, 1, 0 and 3 records and closes the state."""
    _run(128, 128, "scalar", "bf16", 4, 2, 5, 3, steps=6, start_of=[0, 1, 2, 3, 99], bits=bits,
         flush=True)


def test_ragged_flush_diagonal_gate_fp32():
    _run(64, 128, "diag", "fp32", 5, 1, 4, 2, steps=7, start_of=[0, 2, 4, 99], flush=True)
